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


def test_noalloc_calls_of_different_shapes_in_a_row(pkv):
    """A large call (d 128, 8 requests, many split partials) and then a tiny
    one (d 64) on the same stream, with nothing cleared in between: the second
    must not pick up the first's split geometry or partials from the shared
    scratch array.  Its output buffer starts as NaN."""
    big = workloads.build("bf16", 32, 8, 128, 32, False, 5e5, [0, 15, 16, 100, 1000, 4095, 2500, 77], seed=21)
    tiny = workloads.make("tiny")
    outs = {}
    for w in (big, tiny):
        _, ref, _ = oracle_step(w)
        dv = _gpu.to_device(w)
        ctx = _gpu.make_ctx(pkv, w)
        try:
            pkv.pkv_rope_append(ctx, dv["q"], dv["k_new"], dv["v_new"], dv["k_pool"], dv["v_pool"], dv["k_scale"],
                                dv["v_scale"], dv["block_tables"], dv["seq_lens"])
            assert pkv.pkv_check_device_error(ctx)[0] == pkv.PKV_OK
        finally:
            pkv.pkv_destroy(ctx)
        out = torch.full((w.batch, w.Hq, w.d), float("nan"), dtype=torch.bfloat16, device="cuda")
        pkv.pkv_decode_attn_noalloc(_cfg(pkv, w), dv["q"], dv["k_pool"], dv["v_pool"], dv["k_scale"],
                                    dv["v_scale"], dv["block_tables"], dv["seq_lens"], out)
        outs[w.name] = (out, ref)
    torch.cuda.synchronize()
    for name, (out, ref) in outs.items():
        mx, mean, finite = _gpu.errors(out, ref)
        assert finite and mx <= _gpu.TOL_BF16["max"] and mean <= _gpu.TOL_BF16["mean"], (name, mx, mean)


def test_noalloc_rejects_bad_calls_before_launching(pkv):
    # every case is refused on the host, before anything is launched or read
    w = workloads.build("rej", 8, 2, 64, 16, False, 1e4, [5, 9], seed=2)
    dv = _gpu.to_device(w)
    cfg = _cfg(pkv, w)
    args = [dv["k_pool"], dv["v_pool"], None, None, dv["block_tables"], dv["seq_lens"]]
    out = torch.empty(w.batch, w.Hq, w.d, dtype=torch.bfloat16, device="cuda")
    assert pkv.pkv_decode_attn_noalloc(cfg, dv["q"], *args, out, batch=w.batch + 1,
                                       check=False) == pkv.PKV_ERR_INVALID_ARG
    assert pkv.pkv_decode_attn_noalloc(cfg, dv["q"].data_ptr() + 2, *args, out,
                                       check=False) == pkv.PKV_ERR_INVALID_ARG
    bad = pkv.make_config(w.Hq, w.Hkv, 96, w.P, "bf16", 1e4, w.batch, w.bt_stride, w.num_pages)
    assert pkv.pkv_decode_attn_noalloc(bad, dv["q"], *args, out, check=False) == pkv.PKV_ERR_UNSUPPORTED
    assert pkv.pkv_decode_attn_noalloc(cfg, dv["q"], *args, out, batch=0, check=False) == pkv.PKV_OK
