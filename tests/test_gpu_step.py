"""GPU parity: the CUDA path, called through the C ABI, against the CPU oracle.

Small cases (several tiles, ragged tails, every page size / head_dim / group
size / KV type) are compared element by element on the whole output and the
whole pools.  The four full-size workloads run in the benchmark's launch
configuration and are compared the same way: the oracle recomputes the whole
batch from the generator's original inputs.

Both forms of the one-token step are checked: pkv_rope_append followed by
pkv_decode_attn, and pkv_decode_step (bit-identical to the two calls).

Bars: appended V bit-exact, appended K (and rotated q) within 1 bf16 ulp /
1 E4M3 code step, every other pool byte untouched; attention max abs error
<= 1e-2 and mean <= 1e-3 for bf16 KV, <= 6e-2 / 6e-3 for E4M3 KV."""
import numpy as np
import pytest
import torch

import oracle
from paged_kv_flight_b200 import workloads
from tests import _gpu
from tests._util import bf16_ordinal, bits16, bytes8, host_inputs, oracle_attn_threaded, oracle_cfg, oracle_step

pytestmark = pytest.mark.gpu

SMALL = [
    # name, Hq, Hkv, d, P, fp8, lengths
    ("g4_d128_p32_bf16", 32, 8, 128, 32, False, [0, 1, 15, 16, 17, 31, 100, 257, 1000, 4095]),
    ("g8_d128_p16_bf16", 64, 8, 128, 16, False, [5, 64, 200, 511, 2049]),
    ("g4_d128_p64_bf16", 32, 8, 128, 64, False, [63, 64, 65, 3000]),
    ("g1_d64_p16_bf16", 4, 4, 64, 16, False, [2, 77, 300]),
    ("g2_d64_p32_bf16", 8, 4, 64, 32, False, [31, 32, 999]),
    ("g4_d128_p32_fp8", 32, 8, 128, 32, True, [0, 16, 33, 700, 2500]),
    ("g8_d128_p16_fp8", 64, 8, 128, 16, True, [7, 130, 1100]),
    ("g4_d64_p16_fp8", 8, 2, 64, 16, True, [3, 40, 500]),
    ("g2_d128_p64_fp8", 16, 8, 128, 64, True, [100, 1500]),
    ("g4_d64_p32_fp8", 8, 2, 64, 32, True, [0, 31, 32, 33, 63, 64, 999]),
]


@pytest.fixture(scope="module")
def pkv():
    from paged_kv_flight_b200 import pkv as mod
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return mod


def _small(case, seed=101):
    name, Hq, Hkv, d, P, fp8, lengths = case
    return workloads.build(name, Hq, Hkv, d, P, fp8, 5e5 if d == 128 else 1e4, lengths, seed, device="cpu")


def _check_append(w, h_oracle, dv):
    """GPU pools/q after the step against the oracle's, on host copies."""
    gq = bits16(dv["q"])
    assert np.abs(bf16_ordinal(gq) - bf16_ordinal(h_oracle["q"])).max() <= 1
    conv = bytes8 if w.kv_fp8 else bits16
    gk, gv = conv(dv["k_pool"]), conv(dv["v_pool"])
    assert np.array_equal(gv, h_oracle["v_pool"]), "appended V must be bit-exact, nothing else touched"
    diff = gk != h_oracle["k_pool"]
    if diff.any():
        rows = {tuple(r[:3]) for r in np.argwhere(diff)}
        landing = {(int(w.block_tables[b, L // w.P]), kvh, int(L % w.P))
                   for b, L in enumerate(w.seq_lens) for kvh in range(w.Hkv)}
        assert rows <= landing, "K differs outside the landing slots"
        if w.kv_fp8:
            assert np.abs(gk[diff].astype(int) - h_oracle["k_pool"][diff].astype(int)).max() <= 1
        else:
            assert np.abs(bf16_ordinal(gk[diff]) - bf16_ordinal(h_oracle["k_pool"][diff])).max() <= 1


@pytest.mark.parametrize("fused", [False, True], ids=["two_calls", "decode_step"])
@pytest.mark.parametrize("case", SMALL + [("tiny",)], ids=lambda c: c[0])
def test_small_step_matches_oracle(pkv, case, fused):
    w = workloads.make("tiny") if case[0] == "tiny" else _small(case)
    h, ref, st = oracle_step(w)
    assert st == 0
    dv = _gpu.to_device(w)
    ctx = _gpu.make_ctx(pkv, w)
    try:
        out = _gpu.gpu_step(pkv, ctx, dv, fused=fused)
        assert pkv.pkv_check_device_error(ctx)[0] == pkv.PKV_OK
    finally:
        pkv.pkv_destroy(ctx)
    _check_append(w, h, dv)
    mx, mean, finite = _gpu.errors(out, ref)
    t = _gpu.tol(w)
    print(f"\n{w.name}: attention output vs the oracle: max abs {mx:.3e}, mean abs {mean:.3e}")
    assert finite, "non-finite output: a stray read of a NaN sentinel"
    assert mx <= t["max"] and mean <= t["mean"], (mx, mean)


@pytest.mark.parametrize("name", ["llama8b", "hetero70b", "longctx", "fp8"])
def test_full_size_whole_batch_matches_oracle(pkv, name):
    """The full-size workloads in the benchmark's launch configuration: the
    oracle recomputes the whole step (append over the whole pools, attention
    of every request and kv head) from the generator's original inputs, and
    every output element, the rotated q and both whole pools are compared.
    The step is pkv_decode_step, as the benchmark times it (the two-call form
    is held to the same bits by test_decode_step_equals_the_two_calls)."""
    w = workloads.make(name, device="cuda")
    h = host_inputs(w)                                   # original inputs, before the step
    dv = _gpu.to_device(w)
    w.k_pool = w.v_pool = None                           # the device keeps one copy of the pools
    ctx = _gpu.make_ctx(pkv, w)
    try:
        out = _gpu.gpu_step(pkv, ctx, dv, fused=True)
        assert pkv.pkv_check_device_error(ctx)[0] == pkv.PKV_OK
    finally:
        pkv.pkv_destroy(ctx)
    assert oracle.rope_append(oracle_cfg(w), h["q"], h["k_new"], h["v_new"], h["k_pool"], h["v_pool"],
                              h["k_scale"], h["v_scale"], h["block_tables"], h["seq_lens"]) == 0
    ref, st = oracle_attn_threaded(w, h)
    assert st == 0
    _check_append(w, h, dv)
    mx, mean, finite = _gpu.errors(out, ref)
    t = _gpu.tol(w)
    print(f"\n{name}: attention output vs the oracle over the whole batch: max abs {mx:.3e}, mean abs {mean:.3e}")
    assert finite, "non-finite output: a stray read of a NaN sentinel"
    assert mx <= t["max"] and mean <= t["mean"], (mx, mean)


@pytest.mark.parametrize("case", SMALL + [("llama8b",), ("hetero70b",), ("fp8",), ("longctx",)],
                         ids=lambda c: c[0])
def test_decode_step_equals_the_two_calls(pkv, case):
    """pkv_decode_step (the attention launched as a programmatic dependent of
    the RoPE + append kernel): q, both pools and the output must be
    bit-identical to those of pkv_rope_append followed by pkv_decode_attn on
    the same inputs, small cases and full-size workloads alike."""
    w = workloads.make(case[0], device="cuda") if len(case) == 1 else _small(case)
    results = []
    for fused in (False, True):
        dv = _gpu.to_device(w)
        ctx = _gpu.make_ctx(pkv, w)
        try:
            out = _gpu.gpu_step(pkv, ctx, dv, fused=fused)
            assert pkv.pkv_check_device_error(ctx)[0] == pkv.PKV_OK
        finally:
            pkv.pkv_destroy(ctx)
        results.append((out, dv))
        del dv
    (o0, d0), (o1, d1) = results
    assert torch.equal(o0.view(torch.int16), o1.view(torch.int16))
    for k in ("q", "k_pool", "v_pool"):
        a, b = d0[k], d1[k]
        if a.dtype == torch.bfloat16:
            a, b = a.view(torch.int16), b.view(torch.int16)        # NaN sentinels: compare bits
        assert torch.equal(a, b), k
    if len(case) > 1:
        _, ref, _ = oracle_step(w)
        mx, mean, finite = _gpu.errors(o1, ref)
        assert finite and mx <= _gpu.tol(w)["max"] and mean <= _gpu.tol(w)["mean"], (mx, mean)


@pytest.mark.parametrize("case_name", ["g4_d128_p32_bf16", "g4_d128_p32_fp8", "llama8b"])
def test_split_count_invariance(pkv, case_name):
    if case_name == "llama8b":
        w = workloads.make("llama8b", device="cuda")
    else:
        w = _small(next(c for c in SMALL if c[0] == case_name))
    dv = _gpu.to_device(w)
    ctx = _gpu.make_ctx(pkv, w)
    outs = []
    try:
        pkv.pkv_rope_append(ctx, dv["q"], dv["k_new"], dv["v_new"], dv["k_pool"], dv["v_pool"],
                            dv["k_scale"], dv["v_scale"], dv["block_tables"], dv["seq_lens"])
        # static splits, then splits whose range tails are claimed dynamically
        for tail, workers in [(0, 1), (0, 2), (0, 7), (0, 100), (0, 0), (1, 2), (8, 1), (8, 2), (8, 7),
                              (8, 100), (8, 0)]:
            pkv.pkv_set_tail_chunks(ctx, tail)
            pkv.pkv_set_workers(ctx, workers)
            out = torch.empty(w.batch, w.Hq, w.d, dtype=torch.bfloat16, device="cuda")
            pkv.pkv_decode_attn(ctx, dv["q"], dv["k_pool"], dv["v_pool"], dv["k_scale"], dv["v_scale"],
                                dv["block_tables"], dv["seq_lens"], out)
            outs.append(out.float())
        assert pkv.pkv_check_device_error(ctx)[0] == pkv.PKV_OK
    finally:
        pkv.pkv_destroy(ctx)
    # a different split reorders fp32 sums and moves the running max, so the
    # bf16-rounded probabilities differ: bound the mutual difference at 4 bf16
    # ulps of the largest output of the same (request, head) row
    for o in outs[1:]:
        scale = torch.maximum(o.abs().amax(-1, keepdim=True), outs[0].abs().amax(-1, keepdim=True))
        diff = (o - outs[0]).abs()
        assert bool((diff <= 2.0 ** -6 * scale + 1e-6).all()), float((diff / scale).max())
    h = host_inputs(w)
    assert oracle.rope_append(oracle_cfg(w), h["q"], h["k_new"], h["v_new"], h["k_pool"], h["v_pool"],
                              h["k_scale"], h["v_scale"], h["block_tables"], h["seq_lens"]) == 0
    ref, st = oracle_attn_threaded(w, h)
    assert st == 0
    for o in outs:
        mx, mean, _ = _gpu.errors(o, ref)
        assert mx <= _gpu.tol(w)["max"] and mean <= _gpu.tol(w)["mean"]


@pytest.mark.parametrize("case_name", ["g4_d128_p32_bf16", "g2_d64_p32_bf16", "g4_d128_p32_fp8",
                                       "g4_d64_p32_fp8", "llama8b"])
def test_decode_step_under_every_split_equals_the_two_calls(pkv, case_name):
    """pkv_decode_step under static and dynamic splits of every size (fewer
    warp workers than warps included) against pkv_rope_append +
    pkv_decode_attn under the same split, on fresh inputs each time:
    bit-identical q, pools and output."""
    if case_name == "llama8b":
        w = workloads.make("llama8b", device="cuda")
    else:
        w = _small(next(c for c in SMALL if c[0] == case_name))
    ctx = _gpu.make_ctx(pkv, w)
    try:
        for tail, workers in [(0, 1), (0, 2), (0, 7), (0, 100), (0, 0), (1, 2), (8, 1), (8, 7), (8, 100), (8, 0)]:
            pkv.pkv_set_tail_chunks(ctx, tail)
            pkv.pkv_set_workers(ctx, workers)
            two, one = _gpu.to_device(w), _gpu.to_device(w)
            o2 = _gpu.gpu_step(pkv, ctx, two)
            o1 = _gpu.gpu_step(pkv, ctx, one, fused=True)
            assert torch.equal(o1.view(torch.int16), o2.view(torch.int16)), (tail, workers)
            for k in ("q", "k_pool", "v_pool"):
                a, b = two[k], one[k]
                if a.dtype == torch.bfloat16:
                    a, b = a.view(torch.int16), b.view(torch.int16)
                assert torch.equal(a, b), (k, tail, workers)
            del two, one
        assert pkv.pkv_check_device_error(ctx)[0] == pkv.PKV_OK
    finally:
        pkv.pkv_destroy(ctx)


def test_tail_chunk_setting_accepts_automatic_and_rejects_out_of_range(pkv):
    """-1 (the default) is the automatic tail, 0 .. 8 a cap; anything else
    is rejected without changing the setting."""
    w = _small(SMALL[0])
    ctx = _gpu.make_ctx(pkv, w)
    try:
        for ok in (-1, 0, 1, 8):
            assert pkv.pkv_set_tail_chunks(ctx, ok, check=False) == pkv.PKV_OK, ok
        for bad in (-2, 9):
            assert pkv.pkv_set_tail_chunks(ctx, bad, check=False) == pkv.PKV_ERR_INVALID_ARG, bad
    finally:
        pkv.pkv_destroy(ctx)


def test_a_later_context_with_a_smaller_batch_leaves_an_earlier_one_usable(pkv):
    # the attention kernels' shared-memory limit is one process-wide setting;
    # a context created later with a smaller max_batch must not lower it
    # under an earlier context that launches with more (one new token and
    # several)
    w = _small(SMALL[0])
    _, ref, _ = oracle_step(w)
    dv = _gpu.to_device(w)
    big = _gpu.make_ctx(pkv, w, max_batch=8192)
    small = _gpu.make_ctx(pkv, w, max_batch=w.batch)
    try:
        out = _gpu.gpu_step(pkv, big, dv)
        out_tok = torch.empty(w.batch, 1, w.Hq, w.d, dtype=torch.bfloat16, device="cuda")
        pkv.pkv_decode_attn_tokens(big, dv["q"][:, None].contiguous(), dv["k_pool"], dv["v_pool"], None, None,
                                   dv["block_tables"], dv["seq_lens"], out_tok, q_len=1)
        assert pkv.pkv_check_device_error(big)[0] == pkv.PKV_OK
    finally:
        pkv.pkv_destroy(small)
        pkv.pkv_destroy(big)
    for o in (out, out_tok[:, 0]):
        mx, mean, finite = _gpu.errors(o, ref)
        assert finite and mx <= _gpu.TOL_BF16["max"] and mean <= _gpu.TOL_BF16["mean"], (mx, mean)


def test_combine_merges_more_contributors_than_one_staging_block(pkv):
    # one (request, kv head) pair of 270,001 tokens over 128 warps: 16,876
    # tiles, 131 per warp range, a tail of 8 chunks per range -> 1,152 units
    # all cut from the same pair, several times what the combine stages at
    # once (256)
    w = workloads.build("one_long_pair", 8, 1, 128, 64, False, 5e5, [270000], seed=11)
    dv = _gpu.to_device(w)
    ctx = _gpu.make_ctx(pkv, w)
    try:
        pkv.pkv_set_workers(ctx, 128)
        pkv.pkv_set_tail_chunks(ctx, 8)
        out = _gpu.gpu_step(pkv, ctx, dv)
        assert pkv.pkv_check_device_error(ctx)[0] == pkv.PKV_OK
    finally:
        pkv.pkv_destroy(ctx)
    _, ref = _gpu.oracle_request(w, 0)
    mx, mean, _ = _gpu.errors(out[0:1].float(), ref[None])
    assert mx <= _gpu.TOL_BF16["max"] and mean <= _gpu.TOL_BF16["mean"], (mx, mean)


def test_warp_combine_merges_more_than_32_contributors(pkv):
    # 40 requests x 8 kv heads = 320 pairs (the combine then runs one warp per
    # pair) of about 1,000 tiles each; 1,184 warp ranges of about 270 tiles
    # with a tail of 8 chunks -> 9 units per range, about 35 per pair, more
    # than the 32 contributors one pass of the warp handles
    lengths = [16000 + 37 * i for i in range(40)]
    w = workloads.build("warp_combine", 32, 8, 128, 32, False, 5e5, lengths, seed=13, device="cuda")
    picks = (0, 17, 39)
    views = {b: _gpu.request_view(w, b) for b in picks}   # original inputs: the step rotates q in place
    dv = _gpu.to_device(w)
    ctx = _gpu.make_ctx(pkv, w)
    try:
        pkv.pkv_set_tail_chunks(ctx, 8)
        out = _gpu.gpu_step(pkv, ctx, dv)
        assert pkv.pkv_check_device_error(ctx)[0] == pkv.PKV_OK
    finally:
        pkv.pkv_destroy(ctx)
    for b in picks:
        cfg, h = views[b]
        assert oracle.rope_append(cfg, h["q"], h["k_new"], h["v_new"], h["k_pool"], h["v_pool"], None, None,
                                  h["block_tables"], h["seq_lens"]) == 0
        ref = np.full((w.Hq, w.d), np.nan)
        G = w.Hq // w.Hkv
        for kvh in range(w.Hkv):
            o, st = oracle.decode_attn_group(cfg, h["q"], h["k_pool"], h["v_pool"], None, None,
                                             h["block_tables"], h["seq_lens"], 0, kvh)
            assert st == 0
            ref[kvh * G:(kvh + 1) * G] = o
        mx, mean, _ = _gpu.errors(out[b], ref)
        assert mx <= _gpu.TOL_BF16["max"] and mean <= _gpu.TOL_BF16["mean"], (b, mx, mean)


def test_one_token_context_returns_v_exactly(pkv):
    w = workloads.build("one", 32, 8, 128, 32, False, 5e5, [0, 0, 0, 0], seed=3)
    dv = _gpu.to_device(w)
    ctx = _gpu.make_ctx(pkv, w)
    try:
        out = _gpu.gpu_step(pkv, ctx, dv)
    finally:
        pkv.pkv_destroy(ctx)
    G = w.Hq // w.Hkv
    want = w.v_new.to("cuda").repeat_interleave(G, dim=1)
    assert torch.equal(out.view(torch.int16), want.view(torch.int16))


def test_identical_keys_and_page_permutation(pkv):
    w = _small(SMALL[0], seed=7)
    dv = _gpu.to_device(w)
    gen = torch.Generator(device="cuda").manual_seed(9)
    key = torch.randn(w.Hkv, w.d, generator=gen, device="cuda").to(torch.bfloat16)
    # test-written K (identical in every attended slot) and V (random) for every attended slot
    for b, L in enumerate(w.seq_lens):
        for t in range(int(L) + 1):
            page = int(w.block_tables[b, t // w.P])
            dv["k_pool"][page, :, t % w.P, :] = key
            dv["v_pool"][page, :, t % w.P, :] = torch.randn(w.Hkv, w.d, generator=gen, device="cuda").to(torch.bfloat16)
    ctx = _gpu.make_ctx(pkv, w)
    try:
        out = torch.empty(w.batch, w.Hq, w.d, dtype=torch.bfloat16, device="cuda")
        pkv.pkv_decode_attn(ctx, dv["q"], dv["k_pool"], dv["v_pool"], None, None, dv["block_tables"],
                            dv["seq_lens"], out)
        # identical keys: the output is the mean of the values
        G = w.Hq // w.Hkv
        for b, L in enumerate(w.seq_lens):
            n = int(L) + 1
            idx = torch.arange(n)
            pages = torch.from_numpy(w.block_tables[b][(idx // w.P).numpy()]).long().cuda()
            V = dv["v_pool"][pages, :, (idx % w.P).cuda(), :].double()          # [n, Hkv, d]
            mean = V.mean(0).repeat_interleave(G, dim=0)
            assert (out[b].double() - mean).abs().max().item() <= 1e-2
        # permuting physical pages (contents moved, table rewritten) changes nothing, bit for bit
        perm = torch.randperm(w.num_pages, generator=torch.Generator().manual_seed(1)).cuda()
        k2 = torch.empty_like(dv["k_pool"]); v2 = torch.empty_like(dv["v_pool"])
        k2[perm] = dv["k_pool"]; v2[perm] = dv["v_pool"]
        bt = dv["block_tables"].long()
        bt2 = torch.where(bt >= 0, perm[bt.clamp(min=0)], bt).int().contiguous()
        out2 = torch.empty_like(out)
        pkv.pkv_decode_attn(ctx, dv["q"], k2, v2, None, None, bt2, dv["seq_lens"], out2)
        assert torch.equal(out.view(torch.int16), out2.view(torch.int16))
    finally:
        pkv.pkv_destroy(ctx)


def test_repeated_attention_is_deterministic(pkv):
    w = workloads.make("hetero70b", device="cuda")
    dv = _gpu.to_device(w)
    ctx = _gpu.make_ctx(pkv, w)
    try:
        out1 = _gpu.gpu_step(pkv, ctx, dv)
        out2 = torch.empty_like(out1)
        pkv.pkv_decode_attn(ctx, dv["q"], dv["k_pool"], dv["v_pool"], None, None, dv["block_tables"],
                            dv["seq_lens"], out2)
        assert torch.equal(out1.view(torch.int16), out2.view(torch.int16))
    finally:
        pkv.pkv_destroy(ctx)


# ---- errors: host-side rejections and device-side range checks (no trap) ------

def test_host_side_rejections(pkv):
    w = _small(SMALL[0])
    dv = _gpu.to_device(w)
    ctx = _gpu.make_ctx(pkv, w)
    out = torch.empty(w.batch, w.Hq, w.d, dtype=torch.bfloat16, device="cuda")
    try:
        args = [dv["k_pool"], dv["v_pool"], None, None, dv["block_tables"], dv["seq_lens"]]
        st = pkv.pkv_decode_attn(ctx, dv["q"].data_ptr() + 2, *args, out, check=False)
        assert st == pkv.PKV_ERR_INVALID_ARG                      # misaligned q
        st = pkv.pkv_decode_attn(ctx, dv["q"], *args, out, batch=w.batch + 1, check=False)
        assert st == pkv.PKV_ERR_INVALID_ARG                      # batch > max_batch
        st = pkv.pkv_decode_attn(ctx, dv["q"], *args, out, bt_stride=w.bt_stride + 1, check=False)
        assert st == pkv.PKV_ERR_INVALID_ARG                      # bt_stride > max
        st = pkv.pkv_decode_attn(ctx, dv["q"], *args, out, batch=0, check=False)
        assert st == pkv.PKV_OK                                   # empty batch: no-op
        st = pkv.pkv_rope_append(ctx, dv["q"], dv["k_new"], dv["v_new"], None, dv["v_pool"], None, None,
                                 dv["block_tables"], dv["seq_lens"], check=False)
        assert st == pkv.PKV_ERR_INVALID_ARG
    finally:
        pkv.pkv_destroy(ctx)
    wf = _small(SMALL[5])
    dvf = _gpu.to_device(wf)
    ctx = _gpu.make_ctx(pkv, wf)
    try:
        st = pkv.pkv_rope_append(ctx, dvf["q"], dvf["k_new"], dvf["v_new"], dvf["k_pool"], dvf["v_pool"], None,
                                 None, dvf["block_tables"], dvf["seq_lens"], check=False)
        assert st == pkv.PKV_ERR_INVALID_ARG                      # fp8 pools need scales
    finally:
        pkv.pkv_destroy(ctx)


@pytest.mark.parametrize("fused", [False, True], ids=["two_calls", "decode_step"])
@pytest.mark.parametrize("fp8", [False, True])
def test_device_range_errors_are_reported_not_trapped(pkv, fp8, fused):
    case = SMALL[5] if fp8 else SMALL[0]
    w = _small(case, seed=5)
    h, ref, _ = oracle_step(w)
    dv = _gpu.to_device(w)
    bad_page_req, bad_len_req = w.batch - 1, 1     # longest request: page 0 is resident, not landing
    # a resident page id out of range (not the landing page), and a length past the table
    dv["block_tables"][bad_page_req, 0] = w.num_pages + 5
    dv["seq_lens"][bad_len_req] = w.bt_stride * w.P
    ctx = _gpu.make_ctx(pkv, w)
    try:
        out = _gpu.gpu_step(pkv, ctx, dv, fused=fused)
        st, bits = pkv.pkv_check_device_error(ctx)
        assert st == pkv.PKV_ERR_DEVICE_BOUNDS and bits & 1 and bits & 2
        assert pkv.pkv_check_device_error(ctx) == (pkv.PKV_OK, 0)    # cleared after reading
        assert torch.count_nonzero(out[bad_len_req].float()) == 0      # impossible length -> zeros
        keep = [b for b in range(w.batch) if b not in (bad_page_req, bad_len_req)]
        mx, mean, finite = _gpu.errors(out[keep], ref[keep])
        t = _gpu.tol(w)
        assert finite and mx <= t["max"] and mean <= t["mean"]
        # the context still works afterwards
        dv2 = _gpu.to_device(w)
        out2 = _gpu.gpu_step(pkv, ctx, dv2, fused=fused)
        assert pkv.pkv_check_device_error(ctx)[0] == pkv.PKV_OK
        mx, mean, finite = _gpu.errors(out2, ref)
        assert finite and mx <= t["max"]
    finally:
        pkv.pkv_destroy(ctx)
