"""GPU parity for several new tokens per request (speculative-decode
verification): pkv_rope_append_tokens + pkv_decode_attn_tokens, called
through the C ABI, against the CPU oracle's rope_append_tokens +
decode_attn_tokens on the same seeded inputs.

Bars as for one new token: appended V bit-exact and nothing else touched,
appended K and rotated q within 1 bf16 ulp, attention max abs error <= 1e-2
and mean <= 1e-3 (bf16 KV)."""
import numpy as np
import pytest
import torch

import oracle
from paged_kv_flight_b200 import workloads
from tests import _gpu
from tests._util import bf16_ordinal, bits16, host_inputs, oracle_attn_threaded, oracle_cfg

pytestmark = pytest.mark.gpu

CASES = [
    # name, Hq, Hkv, d, P, q_len, lengths
    ("g4_q4_d128_p32", 32, 8, 128, 32, 4, [0, 1, 12, 13, 27, 28, 100, 509, 2000]),
    ("g8_q2_d128_p16", 64, 8, 128, 16, 2, [0, 14, 15, 16, 300, 1025]),
    ("g4_q3_d64_p16", 8, 2, 64, 16, 3, [2, 13, 29, 77, 400]),
    ("g1_q8_d64_p16", 4, 4, 64, 16, 8, [0, 8, 9, 250]),
    ("g2_q5_d128_p64", 16, 8, 128, 64, 5, [59, 60, 64, 700]),
    ("g4_q1_d128_p32", 32, 8, 128, 32, 1, [0, 31, 32, 999]),
]


@pytest.fixture(scope="module")
def pkv():
    from paged_kv_flight_b200 import pkv as mod
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return mod


def _build(case, seed=31):
    name, Hq, Hkv, d, P, q_len, lengths = case
    return workloads.build(name, Hq, Hkv, d, P, False, 5e5 if d == 128 else 1e4, lengths, seed,
                           device="cpu", q_len=q_len)


def _q3(t, w):
    """q / k_new / v_new with an explicit token axis (q_len = 1 has none)."""
    return t if w.q_len > 1 else t[:, None]


def _gpu_tokens(pkv, ctx, w, dv, workers=None):
    out = torch.empty(w.batch, w.q_len, w.Hq, w.d, dtype=torch.bfloat16, device="cuda")
    q, kn, vn = (_q3(dv[k], w).contiguous() for k in ("q", "k_new", "v_new"))
    pkv.pkv_rope_append_tokens(ctx, q, kn, vn, dv["k_pool"], dv["v_pool"], None, None, dv["block_tables"],
                               dv["seq_lens"], q_len=w.q_len)
    if workers is not None:
        pkv.pkv_set_workers(ctx, workers)
    pkv.pkv_decode_attn_tokens(ctx, q, dv["k_pool"], dv["v_pool"], None, None, dv["block_tables"],
                               dv["seq_lens"], out, q_len=w.q_len)
    return q, out


def _oracle_tokens(w):
    h = host_inputs(w)
    for k in ("q", "k_new", "v_new"):
        if w.q_len == 1:
            h[k] = h[k][:, None].copy()
    cfg = oracle_cfg(w)
    assert oracle.rope_append_tokens(cfg, h["q"], h["k_new"], h["v_new"], h["k_pool"], h["v_pool"], None, None,
                                     h["block_tables"], h["seq_lens"]) == 0
    out, st = oracle.decode_attn_tokens(cfg, h["q"], h["k_pool"], h["v_pool"], None, None, h["block_tables"],
                                        h["seq_lens"])
    assert st == 0
    return h, out


@pytest.mark.parametrize("case", CASES, ids=lambda c: c[0])
def test_small_tokens_step_matches_oracle(pkv, case):
    w = _build(case)
    dv = _gpu.to_device(w)
    ctx = _gpu.make_ctx(pkv, w)
    try:
        q, out = _gpu_tokens(pkv, ctx, w, dv)
        assert pkv.pkv_check_device_error(ctx)[0] == pkv.PKV_OK
    finally:
        pkv.pkv_destroy(ctx)
    h, ref = _oracle_tokens(w)
    # append: q within 1 ulp, V bit-exact, K within 1 ulp at the landing slots only
    assert np.abs(bf16_ordinal(bits16(q)) - bf16_ordinal(h["q"])).max() <= 1
    gv, gk = bits16(dv["v_pool"]), bits16(dv["k_pool"])
    assert np.array_equal(gv, h["v_pool"])
    diff = gk != h["k_pool"]
    if diff.any():
        landing = {(int(w.block_tables[b, (L + t) // w.P]), kvh, int((L + t) % w.P))
                   for b, L in enumerate(w.seq_lens) for t in range(w.q_len) for kvh in range(w.Hkv)}
        assert {tuple(r[:3]) for r in np.argwhere(diff)} <= landing
        assert np.abs(bf16_ordinal(gk[diff]) - bf16_ordinal(h["k_pool"][diff])).max() <= 1
    mx, mean, finite = _gpu.errors(out, ref)
    assert finite and mx <= _gpu.TOL_BF16["max"] and mean <= _gpu.TOL_BF16["mean"], (mx, mean)


def test_tokens_split_count_invariance(pkv):
    w = _build(CASES[0])
    dv = _gpu.to_device(w)
    ctx = _gpu.make_ctx(pkv, w)
    outs = []
    try:
        for workers in (1, 2, 7, 100, 0):
            dv2 = _gpu.to_device(w)
            _, out = _gpu_tokens(pkv, ctx, w, dv2, workers=workers)
            outs.append(out.float())
        assert pkv.pkv_check_device_error(ctx)[0] == pkv.PKV_OK
    finally:
        pkv.pkv_destroy(ctx)
    _, ref = _oracle_tokens(w)
    for o in outs:
        mx, mean, _ = _gpu.errors(o, ref)
        assert mx <= _gpu.TOL_BF16["max"] and mean <= _gpu.TOL_BF16["mean"]


def test_full_size_spec4_whole_batch_matches_oracle(pkv):
    """The spec4 workload (the llama8b batch, 4 new tokens each) in the
    benchmark's launch configuration: the oracle recomputes the whole step
    from the generator's original inputs; every output element, q and both
    whole pools are compared."""
    w = workloads.make("spec4", device="cuda")
    h = host_inputs(w)                       # original inputs, before the step
    dv = _gpu.to_device(w)
    w.k_pool = w.v_pool = None               # the device keeps one copy of the pools
    ctx = _gpu.make_ctx(pkv, w)
    try:
        q, out = _gpu_tokens(pkv, ctx, w, dv)
        assert pkv.pkv_check_device_error(ctx)[0] == pkv.PKV_OK
    finally:
        pkv.pkv_destroy(ctx)
    assert oracle.rope_append_tokens(oracle_cfg(w), h["q"], h["k_new"], h["v_new"], h["k_pool"], h["v_pool"],
                                     None, None, h["block_tables"], h["seq_lens"]) == 0
    ref, st = oracle_attn_threaded(w, h)
    assert st == 0
    assert np.abs(bf16_ordinal(bits16(q)) - bf16_ordinal(h["q"])).max() <= 1
    gv, gk = bits16(dv["v_pool"]), bits16(dv["k_pool"])
    assert np.array_equal(gv, h["v_pool"])
    diff = gk != h["k_pool"]
    if diff.any():
        landing = {(int(w.block_tables[b, (L + t) // w.P]), kvh, int((L + t) % w.P))
                   for b, L in enumerate(w.seq_lens) for t in range(w.q_len) for kvh in range(w.Hkv)}
        assert {tuple(r[:3]) for r in np.argwhere(diff)} <= landing
        assert np.abs(bf16_ordinal(gk[diff]) - bf16_ordinal(h["k_pool"][diff])).max() <= 1
    mx, mean, finite = _gpu.errors(out, ref)
    print(f"\nspec4: attention output vs the oracle over the whole batch: max abs {mx:.3e}, mean abs {mean:.3e}")
    assert finite and mx <= _gpu.TOL_BF16["max"] and mean <= _gpu.TOL_BF16["mean"], (mx, mean)


@pytest.mark.parametrize("case", [CASES[0], CASES[1], ("spec4",)], ids=lambda c: c[0])
def test_decode_step_with_several_tokens_equals_the_two_calls(pkv, case):
    """pkv_decode_step with q_len > 1 against pkv_rope_append_tokens followed
    by pkv_decode_attn_tokens on the same inputs: bit-identical q, pools and
    output (the same kernels; the attention is a programmatic dependent of
    the append in the one call)."""
    w = workloads.make("spec4", device="cuda") if len(case) == 1 else _build(case)
    results = []
    for fused in (False, True):
        dv = _gpu.to_device(w)
        ctx = _gpu.make_ctx(pkv, w)
        try:
            if fused:
                q, kn, vn = (_q3(dv[k], w).contiguous() for k in ("q", "k_new", "v_new"))
                out = torch.empty(w.batch, w.q_len, w.Hq, w.d, dtype=torch.bfloat16, device="cuda")
                pkv.pkv_decode_step(ctx, q, kn, vn, dv["k_pool"], dv["v_pool"], None, None, dv["block_tables"],
                                    dv["seq_lens"], out, q_len=w.q_len)
            else:
                q, out = _gpu_tokens(pkv, ctx, w, dv)
            assert pkv.pkv_check_device_error(ctx)[0] == pkv.PKV_OK
        finally:
            pkv.pkv_destroy(ctx)
        results.append((q, out, dv["k_pool"], dv["v_pool"]))
    for a, b in zip(*results):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_tokens_host_side_rejections(pkv):
    w = _build(CASES[0])                     # G = 4
    dv = _gpu.to_device(w)
    ctx = _gpu.make_ctx(pkv, w)
    out = torch.empty(w.batch, 8, w.Hq, w.d, dtype=torch.bfloat16, device="cuda")
    q = torch.zeros(w.batch, 8, w.Hq, w.d, dtype=torch.bfloat16, device="cuda")
    try:
        # G x q_len = 4 x 5 > 16 rows
        st = pkv.pkv_decode_attn_tokens(ctx, q, dv["k_pool"], dv["v_pool"], None, None, dv["block_tables"],
                                        dv["seq_lens"], out, q_len=5, check=False)
        assert st == pkv.PKV_ERR_UNSUPPORTED
        st = pkv.pkv_decode_attn_tokens(ctx, q, dv["k_pool"], dv["v_pool"], None, None, dv["block_tables"],
                                        dv["seq_lens"], out, q_len=0, check=False)
        assert st == pkv.PKV_ERR_INVALID_ARG
        st = pkv.pkv_rope_append_tokens(ctx, q, q, q, dv["k_pool"], dv["v_pool"], None, None, dv["block_tables"],
                                        dv["seq_lens"], q_len=0, check=False)
        assert st == pkv.PKV_ERR_INVALID_ARG
    finally:
        pkv.pkv_destroy(ctx)
    wf = workloads.build("f", 32, 8, 128, 32, True, 5e5, [10, 20], 3, device="cpu", q_len=2)
    dvf = _gpu.to_device(wf)
    ctx = _gpu.make_ctx(pkv, wf)
    try:
        outf = torch.empty(2, 2, 32, 128, dtype=torch.bfloat16, device="cuda")
        st = pkv.pkv_decode_attn_tokens(ctx, dvf["q"], dvf["k_pool"], dvf["v_pool"], None, None,
                                        dvf["block_tables"], dvf["seq_lens"], outf, q_len=2, check=False)
        assert st == pkv.PKV_ERR_INVALID_ARG                 # E4M3 pools need their scales
    finally:
        pkv.pkv_destroy(ctx)


E4M3_CASES = [
    # name, Hq, Hkv, d, P, q_len, lengths (P >= 32: the 16-row maps of this path)
    ("f8_g4_q4_d128_p32", 32, 8, 128, 32, 4, [0, 15, 16, 31, 100, 900]),
    ("f8_g8_q2_d128_p16", 64, 8, 128, 16, 2, [3, 14, 300]),
    ("f8_g2_q8_d64_p64", 8, 4, 64, 64, 8, [0, 63, 64, 500]),
]


@pytest.mark.parametrize("case", E4M3_CASES, ids=lambda c: c[0])
def test_e4m3_tokens_step_matches_oracle(pkv, case):
    """Several new tokens with E4M3 pools: V codes bit-exact, K codes within
    one step, q within 1 ulp, attention within the E4M3 tolerances against
    the oracle fed the same codes and scales."""
    name, Hq, Hkv, d, P, q_len, lengths = case
    w = workloads.build(name, Hq, Hkv, d, P, True, 5e5 if d == 128 else 1e4, lengths, 33, device="cpu",
                        q_len=q_len)
    dv = _gpu.to_device(w)
    ctx = _gpu.make_ctx(pkv, w)
    try:
        out = torch.empty(w.batch, q_len, Hq, d, dtype=torch.bfloat16, device="cuda")
        q, kn, vn = (dv[k].contiguous() for k in ("q", "k_new", "v_new"))
        pkv.pkv_rope_append_tokens(ctx, q, kn, vn, dv["k_pool"], dv["v_pool"], dv["k_scale"], dv["v_scale"],
                                   dv["block_tables"], dv["seq_lens"], q_len=q_len)
        pkv.pkv_decode_attn_tokens(ctx, q, dv["k_pool"], dv["v_pool"], dv["k_scale"], dv["v_scale"],
                                   dv["block_tables"], dv["seq_lens"], out, q_len=q_len)
        assert pkv.pkv_check_device_error(ctx)[0] == pkv.PKV_OK
    finally:
        pkv.pkv_destroy(ctx)
    h = host_inputs(w)
    cfg = oracle_cfg(w)
    assert oracle.rope_append_tokens(cfg, h["q"], h["k_new"], h["v_new"], h["k_pool"], h["v_pool"], h["k_scale"],
                                     h["v_scale"], h["block_tables"], h["seq_lens"]) == 0
    ref, st = oracle.decode_attn_tokens(cfg, h["q"], h["k_pool"], h["v_pool"], h["k_scale"], h["v_scale"],
                                        h["block_tables"], h["seq_lens"])
    assert st == 0
    assert np.abs(bf16_ordinal(bits16(q)) - bf16_ordinal(h["q"])).max() <= 1
    assert np.array_equal(dv["v_pool"].cpu().numpy(), h["v_pool"])
    assert np.abs(dv["k_pool"].cpu().numpy().astype(int) - h["k_pool"].astype(int)).max() <= 1
    mx, mean, finite = _gpu.errors(out, ref)
    assert finite and mx <= _gpu.TOL_FP8["max"] and mean <= _gpu.TOL_FP8["mean"], (mx, mean)
