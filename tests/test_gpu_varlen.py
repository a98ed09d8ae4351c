"""GPU parity of the varlen step (pkv_rope_append_varlen +
pkv_decode_attn_varlen): a different number of new tokens per request,
packed, as in chunked prefill mixed with decode ("Scaling TensorRT-LLM:
Kernel Fusion and Inflight Batching in Production", section "What the
Scheduler Actually Does").  Against the oracle on the same inputs: appended V
bit-exact and K / q within 1 bf16 ulp at every landing slot, every other pool
byte untouched, attention within the bf16 tolerances; the split does not
matter beyond rounding; host rejections and device range errors."""
import numpy as np
import pytest
import torch

import oracle
from paged_kv_flight_b200 import workloads
from tests import _gpu
from tests._util import bf16_ordinal, bits16, oracle_cfg, varlen_host

pytestmark = pytest.mark.gpu

CASES = [
    # name, Hq, Hkv, d, P, lengths, new tokens per request
    ("g4_d128_p32", 32, 8, 128, 32, [100, 0, 517, 1200, 33, 64, 2000, 15], [1, 20, 1, 64, 0, 3, 1, 37]),
    ("g8_d128_p16", 64, 8, 128, 16, [5, 300, 1000], [7, 1, 33]),
    ("g2_d64_p64", 8, 4, 64, 64, [0, 63, 64, 200], [16, 1, 9, 65]),
    ("g1_d64_p16", 4, 4, 64, 16, [10, 40, 0], [50, 1, 1]),
    # longer chunks (up to 130 new tokens), prefixes of up to 3000 tokens,
    # ragged last blocks
    ("g1_d64_p16_prefill", 4, 4, 64, 16, [10, 700, 0], [100, 1, 130]),
    ("g8_d128_p16_prefill", 64, 8, 128, 16, [3000, 20, 511], [48, 1, 9]),
    ("g4_d128_p64_prefill", 32, 8, 128, 64, [2049, 0, 77, 1000], [64, 16, 1, 15]),
    # key counts that end exactly on 128-key tiles (no rows past the keys)
    # next to ragged ones, for the tensor-core prefill blocks
    ("g4_d128_p16_aligned", 32, 8, 128, 16, [100, 1000, 4064, 7], [28, 24, 32, 40]),
]


@pytest.fixture(scope="module")
def pkv():
    from paged_kv_flight_b200 import pkv as mod
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return mod


def _dev_bits(a):
    return torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16).contiguous()


def _setup(case, seed=41):
    name, Hq, Hkv, d, P, lengths, q_lens = case
    w = workloads.build(name, Hq, Hkv, d, P, False, 5e5 if d == 128 else 1e4, lengths, seed, device="cpu",
                        q_len=max(q_lens))
    h = varlen_host(w, q_lens)
    return w, h, q_lens


def _device(h):
    return dict(q=_dev_bits(h["q"]), k_new=_dev_bits(h["k_new"]), v_new=_dev_bits(h["v_new"]),
                k_pool=_dev_bits(h["k_pool"]), v_pool=_dev_bits(h["v_pool"]),
                block_tables=torch.from_numpy(h["block_tables"]).cuda(),
                seq_lens=torch.from_numpy(h["seq_lens"]).cuda(), cu_q=torch.from_numpy(h["cu_q"]).cuda())


def _oracle(w, h):
    ho = {k: (v.copy() if isinstance(v, np.ndarray) else v) for k, v in h.items()}
    cfg = oracle_cfg(w)
    assert oracle.rope_append_varlen(cfg, ho["q"], ho["k_new"], ho["v_new"], ho["k_pool"], ho["v_pool"], None,
                                     None, ho["block_tables"], ho["seq_lens"], ho["cu_q"]) == 0
    out, st = oracle.decode_attn_varlen(cfg, ho["q"], ho["k_pool"], ho["v_pool"], None, None, ho["block_tables"],
                                        ho["seq_lens"], ho["cu_q"])
    assert st == 0
    return ho, out


def _step(pkv, ctx, dv):
    out = torch.full_like(dv["q"], float("nan"))
    pkv.pkv_rope_append_varlen(ctx, dv["q"], dv["k_new"], dv["v_new"], dv["k_pool"], dv["v_pool"], None, None,
                               dv["block_tables"], dv["seq_lens"], dv["cu_q"])
    pkv.pkv_decode_attn_varlen(ctx, dv["q"], dv["k_pool"], dv["v_pool"], None, None, dv["block_tables"], dv["seq_lens"],
                               dv["cu_q"], out)
    return out


@pytest.mark.parametrize("prefill_rows", [64, 0], ids=["prefill_blocks", "token_blocks_only"])
@pytest.mark.parametrize("case", CASES, ids=lambda c: c[0])
def test_varlen_step_matches_oracle(pkv, case, prefill_rows):
    """Default: requests of >= 64 / G new tokens on the tensor-core prefill
    blocks, the rest on the several-new-tokens kernel; 0: all on the latter."""
    w, h, q_lens = _setup(case)
    ho, ref = _oracle(w, h)
    dv = _device(h)
    ctx = _gpu.make_ctx(pkv, w, max_batch=64)
    try:
        pkv.pkv_set_prefill_rows(ctx, prefill_rows)
        out = _step(pkv, ctx, dv)
        assert pkv.pkv_check_device_error(ctx)[0] == pkv.PKV_OK
    finally:
        pkv.pkv_destroy(ctx)
    # q rotated in place: within 1 ulp; pools: V bit-exact, K within 1 ulp, nothing else changed
    assert np.abs(bf16_ordinal(bits16(dv["q"])) - bf16_ordinal(ho["q"])).max() <= 1
    assert np.array_equal(bits16(dv["v_pool"]), ho["v_pool"])
    assert np.abs(bf16_ordinal(bits16(dv["k_pool"])) - bf16_ordinal(ho["k_pool"])).max() <= 1
    mx, mean, finite = _gpu.errors(out, ref)
    assert finite and mx <= _gpu.TOL_BF16["max"] and mean <= _gpu.TOL_BF16["mean"], (mx, mean)


def test_varlen_split_invariance(pkv):
    w, h, _ = _setup(CASES[0], seed=43)
    _, ref = _oracle(w, h)
    outs = []
    ctx = _gpu.make_ctx(pkv, w, max_batch=64)
    try:
        for workers in (1, 7, 0):
            pkv.pkv_set_workers(ctx, workers)
            outs.append(_step(pkv, ctx, _device(h)))
            assert pkv.pkv_check_device_error(ctx)[0] == pkv.PKV_OK
    finally:
        pkv.pkv_destroy(ctx)
    for o in outs:
        mx, mean, finite = _gpu.errors(o, ref)
        assert finite and mx <= _gpu.TOL_BF16["max"] and mean <= _gpu.TOL_BF16["mean"]


def test_varlen_rejections_and_range_errors(pkv):
    w, h, q_lens = _setup(CASES[1], seed=45)
    dv = _device(h)
    out = torch.empty_like(dv["q"])
    ctx = _gpu.make_ctx(pkv, w, max_batch=4)          # room for 16 blocks of 2 tokens
    try:
        # 41 new tokens in blocks of 2 (G = 8): 3 + 21 blocks > 16
        st = pkv.pkv_decode_attn_varlen(ctx, dv["q"], dv["k_pool"], dv["v_pool"], None, None, dv["block_tables"],
                                        dv["seq_lens"], dv["cu_q"], out, check=False)
        assert st == pkv.PKV_ERR_UNSUPPORTED
    finally:
        pkv.pkv_destroy(ctx)
    ctx = _gpu.make_ctx(pkv, w, max_batch=64)
    try:
        bad = dv["seq_lens"].clone()
        bad[1] = w.bt_stride * w.P                    # request 1's one token lies past its table
        out = torch.full_like(dv["q"], 1.0)
        pkv.pkv_decode_attn_varlen(ctx, dv["q"], dv["k_pool"], dv["v_pool"], None, None, dv["block_tables"], bad, dv["cu_q"],
                                   out)
        st, bits = pkv.pkv_check_device_error(ctx)
        assert st == pkv.PKV_ERR_DEVICE_BOUNDS and bits & 1
        i = int(h["cu_q"][1])
        assert torch.count_nonzero(out[i].float()) == 0   # its token's output is zeros
    finally:
        pkv.pkv_destroy(ctx)



def test_varlen_every_request_on_prefill_blocks(pkv):
    """prefill rows 1: every request with a new token takes the tensor-core
    blocks (the several-new-tokens kernel gets no work) — single decode tokens,
    a request with none, ragged blocks."""
    case = CASES[0]
    w, h, _ = _setup(case, seed=53)
    _, ref = _oracle(w, h)
    ctx = _gpu.make_ctx(pkv, w, max_batch=64)
    try:
        pkv.pkv_set_prefill_rows(ctx, 1)
        out = _step(pkv, ctx, _device(h))
        assert pkv.pkv_check_device_error(ctx)[0] == pkv.PKV_OK
    finally:
        pkv.pkv_destroy(ctx)
    mx, mean, finite = _gpu.errors(out, ref)
    assert finite and mx <= _gpu.TOL_BF16["max"] and mean <= _gpu.TOL_BF16["mean"], (mx, mean)


def test_varlen_prefill_blocks_rescale_when_later_keys_dominate(pkv):
    """Keys from position 256 on are scaled by 4 (exact in bf16), so a row's
    max grows by far more than 2^8 after the first 128-key tiles: the
    prefill blocks' reference max moves and O and l are rescaled in tensor
    memory.  Against the oracle on the same inputs.  The softmax is then
    sharp and an output is close to one V row, so V is scaled by 1/4 too:
    outputs stay below about 1.2, where bf16 rounding (half an ulp, <= 2^-8)
    leaves room inside the 1e-2 bar."""
    Hq, Hkv, d, P = 32, 8, 128, 16
    lengths, q_lens = [600, 300, 1000], [40, 20, 1]
    w = workloads.build("rescale", Hq, Hkv, d, P, False, 5e5, lengths, 57, device="cpu", q_len=max(q_lens))
    h = varlen_host(w, q_lens)
    kp = h["k_pool"]
    for b, L in enumerate(lengths):
        for pos in range(256, L):
            page, slot = int(h["block_tables"][b][pos // P]), pos % P
            f = (kp[page, :, slot, :].astype(np.uint16).astype(np.uint32) << 16).view(np.float32) * np.float32(4)
            kp[page, :, slot, :] = (f.view(np.uint32) >> 16).astype(kp.dtype)
    for key in ("v_pool", "v_new"):
        a = h[key]
        f = (a.astype(np.uint16).astype(np.uint32) << 16).view(np.float32) * np.float32(0.25)
        h[key] = (f.view(np.uint32) >> 16).astype(a.dtype)
    _, ref = _oracle(w, h)
    ctx = _gpu.make_ctx(pkv, w, max_batch=8)
    try:
        out = _step(pkv, ctx, _device(h))
        assert pkv.pkv_check_device_error(ctx)[0] == pkv.PKV_OK
    finally:
        pkv.pkv_destroy(ctx)
    mx, mean, finite = _gpu.errors(out, ref)
    assert finite and mx <= _gpu.TOL_BF16["max"] and mean <= _gpu.TOL_BF16["mean"], (mx, mean)


def test_prefill_rows_setting_range(pkv):
    w, _, _ = _setup(CASES[0])
    ctx = _gpu.make_ctx(pkv, w, max_batch=8)
    try:
        for ok in (0, 1, 64, 128):
            assert pkv.pkv_set_prefill_rows(ctx, ok, check=False) == pkv.PKV_OK, ok
        for bad in (-1, 129):
            assert pkv.pkv_set_prefill_rows(ctx, bad, check=False) == pkv.PKV_ERR_INVALID_ARG, bad
    finally:
        pkv.pkv_destroy(ctx)


@pytest.mark.parametrize("fault", ["length", "page"])
def test_varlen_prefill_block_range_errors(pkv, fault):
    """A prefill request whose last token lies past its block table, or
    whose table names a page outside the pool: its rows come out zero, the
    error word says which, the other requests are still right."""
    case = CASES[0]                       # request 3 prefills 64 tokens (G = 4: on the prefill blocks)
    w, h, q_lens = _setup(case, seed=55)
    _, ref = _oracle(w, h)
    dv = _device(h)
    bt, sl = dv["block_tables"].clone(), dv["seq_lens"].clone()
    if fault == "length":
        sl[3] = w.bt_stride * w.P - 10    # its 64 tokens run past the table
    else:
        bt[3, 0] = w.num_pages + 3        # its first page is outside the pool
    out = torch.full_like(dv["q"], 1.0)
    ctx = _gpu.make_ctx(pkv, w, max_batch=64)
    try:
        # the append with the good tables, the attention with the bad ones
        pkv.pkv_rope_append_varlen(ctx, dv["q"], dv["k_new"], dv["v_new"], dv["k_pool"], dv["v_pool"], None, None,
                                   dv["block_tables"], dv["seq_lens"], dv["cu_q"])
        assert pkv.pkv_check_device_error(ctx)[0] == pkv.PKV_OK
        pkv.pkv_decode_attn_varlen(ctx, dv["q"], dv["k_pool"], dv["v_pool"], None, None, bt, sl, dv["cu_q"], out)
        st, bits = pkv.pkv_check_device_error(ctx)
    finally:
        pkv.pkv_destroy(ctx)
    assert st == pkv.PKV_ERR_DEVICE_BOUNDS and bits & (1 if fault == "length" else 2), bits
    cu = h["cu_q"]
    rows = slice(int(cu[3]), int(cu[4]))
    assert torch.count_nonzero(out[rows].float()) == 0
    other = np.ones(int(cu[-1]), bool)
    other[rows] = False
    o = out.float().cpu().numpy()[other]
    assert np.abs(o - ref[other]).max() <= _gpu.TOL_BF16["max"]


def test_full_size_mixed_batch_matches_oracle(pkv):
    """The benchmark's mixed batch (llama8b lengths, 8 requests prefill a
    64-token chunk, 56 decode one token), as the benchmark runs it: RoPE +
    append, then the attention, every output row against the oracle."""
    w, q_lens = workloads.make_mixed(device="cpu")
    h = varlen_host(w, q_lens)
    ho, ref = _oracle(w, h)
    dv = _device(h)
    ctx = _gpu.make_ctx(pkv, w, max_batch=w.batch)
    try:
        out = _step(pkv, ctx, dv)
        assert pkv.pkv_check_device_error(ctx)[0] == pkv.PKV_OK
    finally:
        pkv.pkv_destroy(ctx)
    assert np.array_equal(bits16(dv["v_pool"]), ho["v_pool"])
    mx, mean, finite = _gpu.errors(out, ref)
    print(f"mixed: attention output vs the oracle over the whole batch: max abs {mx:.3e}, mean abs {mean:.3e}")
    assert finite and mx <= _gpu.TOL_BF16["max"] and mean <= _gpu.TOL_BF16["mean"], (mx, mean)


@pytest.mark.parametrize("P", [16, 32])
def test_varlen_step_with_e4m3_pools(pkv, P):
    """The varlen step with E4M3 pools (P = 32: the 16-row maps of the
    several-new-tokens path): V codes bit-exact, K codes within one step,
    attention within the E4M3 tolerances."""
    q_lens = [1, 9, 0, 4, 17]
    w = workloads.build("vf8", 32, 8, 128, P, True, 5e5, [40, 0, 7, 300, 63], 49, device="cpu",
                        q_len=max(q_lens))
    h = varlen_host(w, q_lens)
    ho = {k: (v.copy() if isinstance(v, np.ndarray) else v) for k, v in h.items()}
    cfg = oracle_cfg(w)
    assert oracle.rope_append_varlen(cfg, ho["q"], ho["k_new"], ho["v_new"], ho["k_pool"], ho["v_pool"],
                                     ho["k_scale"], ho["v_scale"], ho["block_tables"], ho["seq_lens"],
                                     ho["cu_q"]) == 0
    ref, st = oracle.decode_attn_varlen(cfg, ho["q"], ho["k_pool"], ho["v_pool"], ho["k_scale"], ho["v_scale"],
                                        ho["block_tables"], ho["seq_lens"], ho["cu_q"])
    assert st == 0
    q = _dev_bits(h["q"])
    kp, vp = torch.from_numpy(h["k_pool"]).cuda(), torch.from_numpy(h["v_pool"]).cuda()
    ks, vs = torch.from_numpy(h["k_scale"]).cuda(), torch.from_numpy(h["v_scale"]).cuda()
    bt, sl = torch.from_numpy(h["block_tables"]).cuda(), torch.from_numpy(h["seq_lens"]).cuda()
    cu = torch.from_numpy(h["cu_q"]).cuda()
    out = torch.full_like(q, float("nan"))
    ctx = _gpu.make_ctx(pkv, w, max_batch=16)
    try:
        pkv.pkv_rope_append_varlen(ctx, q, _dev_bits(h["k_new"]), _dev_bits(h["v_new"]), kp, vp, ks, vs, bt, sl, cu)
        pkv.pkv_decode_attn_varlen(ctx, q, kp, vp, ks, vs, bt, sl, cu, out)
        assert pkv.pkv_check_device_error(ctx)[0] == pkv.PKV_OK
    finally:
        pkv.pkv_destroy(ctx)
    assert np.array_equal(vp.cpu().numpy(), ho["v_pool"])
    assert np.abs(kp.cpu().numpy().astype(int) - ho["k_pool"].astype(int)).max() <= 1
    mx, mean, finite = _gpu.errors(out, ref)
    assert finite and mx <= _gpu.TOL_FP8["max"] and mean <= _gpu.TOL_FP8["mean"], (mx, mean)


def test_varlen_append_into_e4m3_pools(pkv):
    """pkv_rope_append_varlen with E4M3 pools: V codes bit-exact, K codes
    within one step, q within 1 ulp, nothing else changed."""
    q_lens = [3, 0, 1, 9]
    w = workloads.build("vl8", 8, 2, 128, 32, True, 5e5, [10, 4, 63, 100], 47, device="cpu", q_len=max(q_lens))
    h = varlen_host(w, q_lens)
    ho = {k: (v.copy() if isinstance(v, np.ndarray) else v) for k, v in h.items()}
    assert oracle.rope_append_varlen(oracle_cfg(w), ho["q"], ho["k_new"], ho["v_new"], ho["k_pool"], ho["v_pool"],
                                     ho["k_scale"], ho["v_scale"], ho["block_tables"], ho["seq_lens"],
                                     ho["cu_q"]) == 0
    dq, dk, dv_ = _dev_bits(h["q"]), _dev_bits(h["k_new"]), _dev_bits(h["v_new"])
    kp = torch.from_numpy(h["k_pool"]).cuda()
    vp = torch.from_numpy(h["v_pool"]).cuda()
    ks = torch.from_numpy(h["k_scale"]).cuda()
    vs = torch.from_numpy(h["v_scale"]).cuda()
    ctx = _gpu.make_ctx(pkv, w, max_batch=8)
    try:
        pkv.pkv_rope_append_varlen(ctx, dq, dk, dv_, kp, vp, ks, vs, torch.from_numpy(h["block_tables"]).cuda(),
                                   torch.from_numpy(h["seq_lens"]).cuda(), torch.from_numpy(h["cu_q"]).cuda())
        assert pkv.pkv_check_device_error(ctx)[0] == pkv.PKV_OK
    finally:
        pkv.pkv_destroy(ctx)
    assert np.array_equal(vp.cpu().numpy(), ho["v_pool"])
    assert np.abs(kp.cpu().numpy().astype(int) - ho["k_pool"].astype(int)).max() <= 1
    assert np.abs(bf16_ordinal(bits16(dq)) - bf16_ordinal(ho["q"])).max() <= 1
