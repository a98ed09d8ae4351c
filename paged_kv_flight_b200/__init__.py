"""paged_kv_flight_b200: one in-flight-batched decode step over a paged KV
cache on B200 (sm_100a).

The compute path is the C-ABI library ``libpkv.so`` (CUDA kernels built from
``csrc/``); ``paged_kv_flight_b200.pkv`` is its thin ctypes binding and loads
it on import, failing loudly when it is missing.  ``workloads`` draws seeded
synthetic inputs.  Importing this package itself loads nothing.
"""
