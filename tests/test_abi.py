"""The C-ABI library loads, exports every symbol include/*.h declares, and
rejects bad arguments on the host before any CUDA call (runs without a GPU)."""
import ctypes as C
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", h) for h in ("pkv.h", "pkv_pages.h")]


@pytest.fixture(scope="module")
def pkv():
    from paged_kv_flight_b200 import build
    build.build()
    from paged_kv_flight_b200 import pkv as mod
    return mod


def _declared():
    text = "".join(open(h).read() for h in HEADERS)
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(pkv_[a-z_]+)\s*\(", text)))


def test_header_declarations_are_all_exported(pkv):
    names = _declared()
    assert set(names) == set(pkv.EXPORTS)
    for n in names:
        assert hasattr(pkv.lib, n), n
    out = subprocess.run(["nm", "-D", "--defined-only", pkv._LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {ln.split()[-1] for ln in out.splitlines() if " T " in ln}
    assert set(names) <= exported


def test_config_struct_layout_matches_header(pkv):
    # ints, enum, then a double on an 8-byte boundary, then three ints
    assert C.sizeof(pkv.pkv_config) == 48
    assert pkv.pkv_config.rope_base.offset == 24


def _cfg(pkv, **kw):
    base = dict(num_q_heads=32, num_kv_heads=8, head_dim=128, page_size=32, kv_dtype=0,
                rope_base=5e5, max_batch=64, max_blocks_per_seq=129, num_pages=5000)
    base.update(kw)
    return pkv.make_config(**base)


@pytest.mark.parametrize("kw,status", [
    (dict(num_q_heads=30), 1),                      # Hq % Hkv != 0
    (dict(num_kv_heads=0), 1),
    (dict(head_dim=96), 2),
    (dict(head_dim=-1), 1),
    (dict(page_size=8), 2),
    (dict(page_size=0), 1),
    (dict(num_q_heads=128, num_kv_heads=8), 2),     # G = 16
    (dict(kv_dtype=7), 1),
    (dict(rope_base=1.0), 1),
    (dict(rope_base=float("nan")), 1),
    (dict(max_batch=0), 1),
    (dict(max_batch=100000), 2),
    (dict(num_pages=0), 1),
    (dict(max_blocks_per_seq=0), 1),
])
def test_create_rejects_bad_configs_on_the_host(pkv, kw, status):
    st, ctx = pkv.pkv_create(_cfg(pkv, **kw), check=False)
    assert st == status and ctx is None


def test_null_context_and_status_strings(pkv):
    assert pkv.lib.pkv_rope_append(None, None, None, None, None, None, None, None, None, 1, None, 1, None) == 1
    assert pkv.lib.pkv_decode_attn(None, None, None, None, None, None, None, 1, None, 1, None, None) == 1
    assert pkv.lib.pkv_set_workers(None, 3) == 1
    assert pkv.lib.pkv_set_tail_chunks(None, 3) == 1
    assert pkv.lib.pkv_destroy(None) == 0
    assert pkv.lib.pkv_workspace_bytes(None) == 0
    for s in range(7):
        assert pkv.pkv_status_str(s) and pkv.pkv_status_str(s) != "unknown status"
    assert pkv.pkv_status_str(99) == "unknown status"


def test_table_sync_rejects_bad_sizes_without_touching_the_device():
    """Argument checks of pkv_table_sync run on the host before any launch."""
    import torch
    from paged_kv_flight_b200 import pkv
    # host buffers through the raw C entry point: every case below returns
    # before a pointer is dereferenced or a kernel launched
    t = torch.zeros(4, 8, dtype=torch.int32)
    up = torch.zeros(64, dtype=torch.int32)
    bt, ln = torch.zeros(4, 8, dtype=torch.int32), torch.zeros(4, dtype=torch.int32)
    call = lambda n, b, P: pkv.lib.pkv_table_sync(up.data_ptr(), n, b, 4, 8, P, t.data_ptr(),   # noqa: E731
                                                  bt.data_ptr(), ln.data_ptr(), None)
    assert call(-1, 1, 16) == pkv.PKV_ERR_INVALID_ARG
    assert call(0, 5, 16) == pkv.PKV_ERR_INVALID_ARG      # batch above the table's rows
    assert call(0, 1, 0) == pkv.PKV_ERR_INVALID_ARG       # page size
    assert call(0, 0, 16) == pkv.PKV_OK                    # nothing to do


def test_binding_rejects_host_tensors_and_wrong_element_types():
    """The Python binding checks each tensor argument before the library is
    called: device memory, the element type the kernels read it as, and
    contiguity.  A host tensor or a narrower element type would have the
    kernels touch memory the caller did not mean."""
    import pytest
    import torch
    from paged_kv_flight_b200 import pkv
    q = torch.zeros(2, 8, 64, dtype=torch.bfloat16)          # on the host
    lens = torch.zeros(2, dtype=torch.int32)
    bt = torch.zeros(2, 4, dtype=torch.int32)
    with pytest.raises(ValueError, match="device tensors"):
        pkv.pkv_decode_attn(None, q, 0x1000, 0x1000, None, None, bt, lens, q)
    with pytest.raises(ValueError, match="device tensors"):
        pkv.pkv_table_sync(lens, 0, 0, bt, bt, lens, 16, stream=0)
    # raw integer pointers pass through unchecked (the C-level checks still run)
    assert pkv._ptr(0x1000, pkv._ACT, "q") == 0x1000 and pkv._ptr(None, pkv._ACT, "q") is None
    # the element-type and layout checks, on host tensors that report
    # themselves as device tensors (no CUDA context is needed)
    class _OnDevice(torch.Tensor):
        @property
        def is_cuda(self):
            return True

    class _Fake:
        pass

    dev = lambda dt, n=4: torch.zeros(n, dtype=dt).as_subclass(_OnDevice)   # noqa: E731
    for dt, kinds in ((torch.float32, pkv._ACT), (torch.float16, pkv._ACT), (torch.int64, pkv._I32),
                      (torch.int16, pkv._POOL), (torch.float64, pkv._F32)):
        with pytest.raises(TypeError, match="expected"):
            pkv._ptr(dev(dt), kinds, "arg")
    for dt, kinds in ((torch.bfloat16, pkv._ACT), (torch.uint8, pkv._POOL), (torch.float8_e4m3fn, pkv._POOL),
                      (torch.bfloat16, pkv._POOL), (torch.int32, pkv._I32), (torch.float32, pkv._F32)):
        t = dev(dt)
        assert pkv._ptr(t, kinds, "arg") == t.data_ptr()
    strided = torch.zeros(4, 4, dtype=torch.bfloat16).as_subclass(_OnDevice).t()
    with pytest.raises(ValueError, match="contiguous"):
        pkv._ptr(strided, pkv._ACT, "q")
    with pytest.raises(TypeError):
        pkv._ptr(_Fake(), pkv._ACT, "q")
    # the page allocator's change log is a host int32 buffer
    with pytest.raises(ValueError):
        pkv._hptr(torch.zeros(6, dtype=torch.int64), "out")
    assert pkv._hptr(lens, "out") == lens.data_ptr()
