"""GPU parity of the fused QKV projection + RoPE + append
(pkv_qkv_rope_append, tcgen05 tensor cores) against the oracle: the fp64
projection rounded to bf16 (orc_project_bf16), split into q / k_new / v_new,
then the oracle's own RoPE + append (orc_rope_append).

The kernel sums the hidden-size products in fp32 on the tensor cores (each
bf16 x bf16 product is exact in fp32; the order and rounding of the sum are
the hardware's), so a projection output differs from the fp64 sum by at most
K 2^-23 S (K = hidden, S = sum_j |x_j w_j|, the worst case for fp32
accumulation in any order, truncating or rounding), which can move it to
another bf16 value; the rotation mixes the two members of a pair.  The bar:
every element within 3 bf16 ulps of the larger magnitude of its rotation
pair plus K 2^-23 S of the pair's features; at least 97% of the elements
bit-identical; E4M3 codes within one step; every pool byte outside the
landing slots untouched.  The same projection from the tiled weight layout
(pkv_qkv_pack_weight) must give the same bytes as from the row-major one, and
every split of the hidden dimension over a cluster (1 .. 4 CTAs, reduced
through distributed shared memory) must meet the same bar."""
import numpy as np
import pytest
import torch

import oracle
from paged_kv_flight_b200 import workloads
from tests import _gpu
from tests._util import bits16, bytes8, host_inputs, oracle_cfg

pytestmark = pytest.mark.gpu

CASES = [
    # name, Hq, Hkv, d, P, hidden, lengths, fp8
    ("small_d128", 8, 2, 128, 16, 256, [0, 5, 17, 40, 100], False),
    ("llama8b_like", 32, 8, 128, 32, 4096, list(range(100, 100 + 64 * 37, 37)), False),
    ("two_m_tiles_d64", 16, 4, 64, 16, 512, [3 * i for i in range(130)], False),
    ("fp8_pools", 8, 2, 128, 32, 512, [1, 31, 32, 77, 300, 600, 1000], True),
]


@pytest.fixture(scope="module")
def pkv():
    from paged_kv_flight_b200 import pkv as mod
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return mod


def _f(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def pair_max(a):
    half = a.shape[-1] // 2
    m = np.maximum(a[..., :half], a[..., half:])
    return np.concatenate([m, m], axis=-1)


def close_pairs(got_bits, ref_bits, acc_err, ulps=3):
    """|got - ref| <= ulps 2^-8 max(|ref_i|, |ref_{i+d/2}|) + the pair's accumulation bound."""
    g, r = _f(got_bits), _f(ref_bits)
    tol = ulps * 2.0 ** -8 * np.maximum(pair_max(np.abs(r)), 2.0 ** -20) + pair_max(acc_err)
    return bool((np.abs(g - r) <= tol).all())


def _inputs(B, N, hidden, seed=5):
    gen = torch.Generator().manual_seed(seed)
    x = torch.randn(B, hidden, generator=gen).to(torch.bfloat16)
    wq = (torch.randn(N, hidden, generator=gen) / hidden ** 0.5).to(torch.bfloat16)
    return x, wq


@pytest.mark.parametrize("case", CASES, ids=lambda c: c[0])
def test_fused_projection_matches_oracle(pkv, case):
    name, Hq, Hkv, d, P, hidden, lengths, fp8 = case
    w = workloads.build(name, Hq, Hkv, d, P, fp8, 5e5 if d == 128 else 1e4, lengths, 17, device="cpu")
    B, N = w.batch, (Hq + 2 * Hkv) * d
    x, wq = _inputs(B, N, hidden)

    xd, wd = x.cuda(), wq.cuda()
    wt = torch.empty_like(wd)
    # (split, layout) runs: automatic split from both layouts, then every split
    runs = [(0, pkv.PKV_W_ROWS), (0, pkv.PKV_W_TILED)] + [(sp, pkv.PKV_W_TILED) for sp in (1, 2, 3, 4)]
    results = []
    ctx = _gpu.make_ctx(pkv, w)
    try:
        pkv.pkv_qkv_pack_weight(ctx, wd, wt)
        for sp, layout in runs:
            dv = _gpu.to_device(w)
            q_out = torch.empty(B, Hq, d, dtype=torch.bfloat16, device="cuda")
            pkv.pkv_set_qkv_split(ctx, sp)
            pkv.pkv_qkv_rope_append(ctx, xd, wt if layout == pkv.PKV_W_TILED else wd, q_out, dv["k_pool"],
                                    dv["v_pool"], dv["k_scale"], dv["v_scale"], dv["block_tables"], dv["seq_lens"],
                                    w_layout=layout)
            assert pkv.pkv_check_device_error(ctx)[0] == pkv.PKV_OK
            results.append((sp, layout, q_out.cpu(), dv["k_pool"].cpu(), dv["v_pool"].cpu()))
    finally:
        pkv.pkv_destroy(ctx)
    # the tiled layout holds the same values in another order (a permutation,
    # checked byte for byte), and the kernel's sums run in the same order
    perm = wq.view(Hq + 2 * Hkv, d, hidden // 64, 64).permute(0, 2, 1, 3).contiguous()
    assert torch.equal(wt.cpu().view(torch.int16), perm.reshape(N, hidden).view(torch.int16))
    for a, b in zip(results[0][2:], results[1][2:]):
        assert torch.equal(a.view(torch.uint8), b.view(torch.uint8))

    # oracle: fp64 projection -> bf16, then the oracle's RoPE + append
    y = oracle.project_bf16(bits16(x), bits16(wq))
    # fp32 accumulation bound per (token, feature): K 2^-23 sum_j |x_j w_j|
    acc = hidden * 2.0 ** -23 * (np.abs(x.double().numpy()) @ np.abs(wq.double().numpy()).T)
    h = host_inputs(w)
    h["q"] = np.ascontiguousarray(y[:, :Hq * d].reshape(B, Hq, d))
    h["k_new"] = np.ascontiguousarray(y[:, Hq * d:(Hq + Hkv) * d].reshape(B, Hkv, d))
    h["v_new"] = np.ascontiguousarray(y[:, (Hq + Hkv) * d:].reshape(B, Hkv, d))
    assert oracle.rope_append(oracle_cfg(w), h["q"], h["k_new"], h["v_new"], h["k_pool"], h["v_pool"],
                              h["k_scale"], h["v_scale"], h["block_tables"], h["seq_lens"]) == 0

    acc_q = acc[:, :Hq * d].reshape(B, Hq, d)
    acc_k = acc[:, Hq * d:(Hq + Hkv) * d].reshape(B, Hkv, d)
    acc_v = acc[:, (Hq + Hkv) * d:].reshape(B, Hkv, d)
    landing = {(int(w.block_tables[b, L // P]), kvh, int(L % P)) for b, L in enumerate(w.seq_lens)
               for kvh in range(Hkv)}
    order = sorted((int(w.block_tables[b, L // P]), kvh, int(L % P), b) for b, L in enumerate(w.seq_lens)
                   for kvh in range(Hkv))
    conv = bytes8 if fp8 else bits16
    for sp, layout, q_out, k_pool, v_pool in results:
        gq = bits16(q_out)
        assert close_pairs(gq, h["q"], acc_q), (sp, layout)
        same = [np.mean(gq == h["q"])]
        for key, pool in (("k_pool", k_pool), ("v_pool", v_pool)):
            got, ref = conv(pool), h[key]
            diff = got != ref
            rows = {tuple(map(int, r[:3])) for r in np.argwhere(diff)}
            assert rows <= landing, f"{key}: bytes changed outside the landing slots (split {sp})"
            gl = np.stack([got[pg, kvh, sl] for pg, kvh, sl, _ in order])
            rl = np.stack([ref[pg, kvh, sl] for pg, kvh, sl, _ in order])
            ae = np.stack([(acc_k if key == "k_pool" else acc_v)[b, kvh] for _, kvh, _, b in order])
            if fp8:
                assert np.abs(gl.astype(int) - rl.astype(int)).max() <= 1      # one E4M3 code step
            else:
                assert close_pairs(gl, rl, ae, ulps=3 if key == "k_pool" else 1), (sp, key)
            same.append(np.mean(gl == rl))
        assert min(same) >= 0.97, (sp, layout, same)


@pytest.mark.parametrize("fp8", [False, True])
def test_device_range_errors_skip_the_token(pkv, fp8):
    """A length past the block table (error bit 1) and an out-of-range landing
    page id (bit 2) are the kernel's own checks: the token with the bad length
    stores nothing, the one with the bad page stores its q but no k / v, every
    other token is stored as the oracle says, and the context keeps working."""
    Hq, Hkv, d, P, hidden = 8, 2, 128, 16, 512
    lengths = [0, 5, 17, 40, 100, 63]
    w = workloads.build("qkv_err", Hq, Hkv, d, P, fp8, 5e5, lengths, 23, device="cpu")
    B, N = w.batch, (Hq + 2 * Hkv) * d
    x, wq = _inputs(B, N, hidden, seed=9)
    bad_len, bad_page = 1, 3
    lp = lengths[bad_page] // P
    y = oracle.project_bf16(bits16(x), bits16(wq))
    acc = hidden * 2.0 ** -23 * (np.abs(x.double().numpy()) @ np.abs(wq.double().numpy()).T)
    h = host_inputs(w)
    pool0 = {key: h[key].copy() for key in ("k_pool", "v_pool")}
    h["q"] = np.ascontiguousarray(y[:, :Hq * d].reshape(B, Hq, d))
    h["k_new"] = np.ascontiguousarray(y[:, Hq * d:(Hq + Hkv) * d].reshape(B, Hkv, d))
    h["v_new"] = np.ascontiguousarray(y[:, (Hq + Hkv) * d:].reshape(B, Hkv, d))
    assert oracle.rope_append(oracle_cfg(w), h["q"], h["k_new"], h["v_new"], h["k_pool"], h["v_pool"],
                              h["k_scale"], h["v_scale"], h["block_tables"], h["seq_lens"]) == 0
    good = [b for b in range(B) if b not in (bad_len, bad_page)]
    conv = bytes8 if fp8 else bits16
    sentinel = torch.full((B, Hq, d), 7.0, dtype=torch.bfloat16)
    ctx = _gpu.make_ctx(pkv, w)
    try:
        for sp in (0, 1, 3):
            dv = _gpu.to_device(w)
            dv["seq_lens"][bad_len] = w.bt_stride * P
            dv["block_tables"][bad_page, lp] = w.num_pages + 5
            q_out = sentinel.cuda()
            pkv.pkv_set_qkv_split(ctx, sp)
            pkv.pkv_qkv_rope_append(ctx, x.cuda(), wq.cuda(), q_out, dv["k_pool"], dv["v_pool"], dv["k_scale"],
                                    dv["v_scale"], dv["block_tables"], dv["seq_lens"])
            st, bits = pkv.pkv_check_device_error(ctx)
            assert st == pkv.PKV_ERR_DEVICE_BOUNDS and bits & 1 and bits & 2, (sp, st, bits)
            gq = bits16(q_out)
            assert (gq[bad_len] == bits16(sentinel)[bad_len]).all(), sp        # nothing stored
            ok_q = [b for b in range(B) if b != bad_len]
            assert close_pairs(gq[ok_q], h["q"][ok_q], acc[ok_q, :Hq * d].reshape(len(ok_q), Hq, d)), sp
            for key in ("k_pool", "v_pool"):
                got, ref, base = conv(dv[key].cpu()), h[key], pool0[key]
                slots = {(int(w.block_tables[b, lengths[b] // P]), kvh, lengths[b] % P) for b in good
                         for kvh in range(Hkv)}
                for idx in map(tuple, np.argwhere((got != base).any(axis=-1))):
                    assert idx in slots, (sp, key, idx)                      # only good tokens' slots
                for b in good:
                    pg = int(w.block_tables[b, lengths[b] // P])
                    off = Hq * d if key == "k_pool" else (Hq + Hkv) * d
                    for kvh in range(Hkv):
                        g_, r_ = got[pg, kvh, lengths[b] % P], ref[pg, kvh, lengths[b] % P]
                        if fp8:
                            assert np.abs(g_.astype(int) - r_.astype(int)).max() <= 1
                        else:
                            a_ = acc[b, off + kvh * d: off + (kvh + 1) * d]
                            assert close_pairs(g_[None], r_[None], a_[None]), (sp, key, b)
        # the context still works afterwards
        dv = _gpu.to_device(w)
        pkv.pkv_set_qkv_split(ctx, 0)
        q_out = torch.empty(B, Hq, d, dtype=torch.bfloat16, device="cuda")
        pkv.pkv_qkv_rope_append(ctx, x.cuda(), wq.cuda(), q_out, dv["k_pool"], dv["v_pool"], dv["k_scale"],
                                dv["v_scale"], dv["block_tables"], dv["seq_lens"])
        assert pkv.pkv_check_device_error(ctx)[0] == pkv.PKV_OK
        assert close_pairs(bits16(q_out), h["q"], acc[:, :Hq * d].reshape(B, Hq, d))
    finally:
        pkv.pkv_destroy(ctx)


def test_host_side_rejections(pkv):
    w = workloads.build("qkv_rej", 8, 2, 128, 16, False, 5e5, [3, 9], 3, device="cpu")
    dv = _gpu.to_device(w)
    x = torch.zeros(w.batch, 256, dtype=torch.bfloat16, device="cuda")
    wq = torch.zeros(12 * 128, 256, dtype=torch.bfloat16, device="cuda")
    q_out = torch.empty(w.batch, 8, 128, dtype=torch.bfloat16, device="cuda")
    ctx = _gpu.make_ctx(pkv, w)
    try:
        args = (dv["k_pool"], dv["v_pool"], None, None, dv["block_tables"], dv["seq_lens"])
        x96 = torch.zeros(w.batch, 96, dtype=torch.bfloat16, device="cuda")   # hidden not a multiple of 64
        assert pkv.pkv_qkv_rope_append(ctx, x96, wq, q_out, *args, check=False) == pkv.PKV_ERR_UNSUPPORTED
        assert pkv.pkv_qkv_rope_append(ctx, x, wq, q_out, *args, check=False, w_layout=2) == pkv.PKV_ERR_INVALID_ARG
        assert pkv.pkv_set_qkv_split(ctx, 5, check=False) == pkv.PKV_ERR_INVALID_ARG
        assert pkv.pkv_qkv_pack_weight(ctx, wq, wq, check=False) == pkv.PKV_ERR_INVALID_ARG      # overlap
        shape = pkv.pkv_qkv_launch_shape(ctx, w.batch, 256)
        assert 1 <= shape["split"] <= 4 and shape["stages"] >= 2 and shape["smem_bytes"] > 0
    finally:
        pkv.pkv_destroy(ctx)

