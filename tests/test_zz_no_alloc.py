"""pkv_decode_attn_noalloc: the decode attention for callers that cannot
allocate device memory (a runtime that reserved all memory for its own pool,
a plug-in limited to memory its host framework provides, a path that must not
pay for an allocation).  Its output must match pkv_decode_attn's, on two calls
in a row that share the library's fixed scratch array.

This file is collected last on purpose, so that a run stopping at the first
failure has already run every other test; it also passes alone in a fresh
process."""
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


def _cfg(pkv, w):
    return pkv.make_config(w.Hq, w.Hkv, w.d, w.P, "fp8" if w.kv_fp8 else "bf16", w.rope_base, w.batch,
                           w.bt_stride, w.num_pages)


@pytest.mark.parametrize("case", [
    ("bf16", 32, 8, 128, 32, False, [0, 15, 16, 100, 1000, 4095, 2500, 77]),
    ("fp8", 32, 8, 128, 32, True, [3, 40, 700, 2000]),
    ("tiny", None),
], ids=lambda c: c[0])
def test_noalloc_matches_context_entry_point_twice(pkv, case):
    if case[0] == "tiny":
        w = workloads.make("tiny")
    else:
        name, Hq, Hkv, d, P, fp8, lengths = case
        w = workloads.build(name, Hq, Hkv, d, P, fp8, 5e5, lengths, seed=21)
    _, ref, _ = oracle_step(w)
    dv = _gpu.to_device(w)
    ctx = _gpu.make_ctx(pkv, w)
    try:
        out_ctx = _gpu.gpu_step(pkv, ctx, dv)          # append + attention through the context
        assert pkv.pkv_check_device_error(ctx)[0] == pkv.PKV_OK
    finally:
        pkv.pkv_destroy(ctx)
    cfg = _cfg(pkv, w)
    t = _gpu.tol(w)
    for _ in range(2):                                   # two calls in a row, same scratch
        out = torch.full_like(out_ctx, float("nan"))
        pkv.pkv_decode_attn_noalloc(cfg, dv["q"], dv["k_pool"], dv["v_pool"], dv["k_scale"], dv["v_scale"],
                                    dv["block_tables"], dv["seq_lens"], out)
        torch.cuda.synchronize()
        diff = (out.float() - out_ctx.float()).abs()
        assert bool(torch.isfinite(out.float()).all())
        assert diff.max().item() <= t["max"] and diff.mean().item() <= t["mean"]
        mx, mean, finite = _gpu.errors(out, ref)
        assert finite and mx <= t["max"] and mean <= t["mean"]


def test_noalloc_rejects_what_does_not_fit(pkv):
    # 8192 requests x 512 kv heads of arrival counters alone fill the 16 MiB scratch
    # (rejected on the host before anything is launched or read, so small
    # stand-in buffers suffice)
    cfg = pkv.make_config(512, 512, 64, 16, "bf16", 1e4, 8192, 4, 16)
    buf = torch.zeros(4096, dtype=torch.int32, device="cuda")
    st = pkv.pkv_decode_attn_noalloc(cfg, buf, buf, buf, None, None, buf, buf, buf, batch=8192, bt_stride=4,
                                     check=False)
    assert st == pkv.PKV_ERR_UNSUPPORTED
