"""The decode step (RoPE + append, attention, combine) captured once in a
CUDA graph and replayed: the library never synchronises with the host, so the
three kernels capture as they are; replays on fresh inputs copied into the
captured buffers match the oracle, for the two calls and for pkv_decode_step,
whose attention is a programmatic dependent of the append kernel in the graph
too ("TensorRT-LLM: NVIDIA's Optimized Inference
Engine", section "The paged KV cache, in-flight batching and CUDA graphs":
decode steps repeat the same kernels, so they are recorded once and replayed)."""
import pytest
import torch

from paged_kv_flight_b200 import workloads
from tests import _gpu
from tests._util import oracle_step

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pkv():
    from paged_kv_flight_b200 import pkv as mod
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return mod


@pytest.mark.parametrize("fused", [False, True], ids=["two_calls", "decode_step"])
@pytest.mark.parametrize("fp8", [False, True])
def test_captured_step_replays_match_oracle(pkv, fp8, fused):
    # two workloads with the same shapes and page tables, different values
    lengths = [3, 17, 64, 200, 900, 2047]
    ws = [workloads.build(f"graph{i}", 32, 8, 128, 32, fp8, 5e5, lengths, seed=40 + i) for i in range(2)]
    dv = _gpu.to_device(ws[0])
    ctx = _gpu.make_ctx(pkv, ws[0])
    out = torch.empty(ws[0].batch, 32, 128, dtype=torch.bfloat16, device="cuda")
    side = torch.cuda.Stream()
    graph = None
    try:
        # warm the library on the capture stream (tensor maps, kernel attributes)
        with torch.cuda.stream(side):
            _gpu.gpu_step(pkv, ctx, dv, out=out, fused=fused)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=side):
            _gpu.gpu_step(pkv, ctx, dv, out=out, fused=fused)
        for w in ws:
            fresh = _gpu.to_device(w)
            for k in dv:
                if dv[k] is not None:
                    dv[k].copy_(fresh[k])
            graph.replay()
            torch.cuda.synchronize()
            _, ref, st = oracle_step(w)
            assert st == 0
            mx, mean, finite = _gpu.errors(out, ref)
            t = _gpu.tol(w)
            assert finite and mx <= t["max"] and mean <= t["mean"], (w.name, mx, mean)
        assert pkv.pkv_check_device_error(ctx)[0] == pkv.PKV_OK
    finally:
        graph = None
        torch.cuda.synchronize()
        pkv.pkv_destroy(ctx)
