"""Pins for the oracle's append placement and decode attention.

Each test checks the oracle against something outside it: the closed-form
slot placement, independent numpy RoPE, a library SDPA in fp64 on a numpy
gather, an explicit brute-force loop, and the closed-form special cases the
method has (one-token context returns v exactly; identical keys or a zero
query give the mean of the values; adding one vector to every key, which adds
one constant to every score, changes nothing; permuting physical pages changes
nothing)."""
import math

import numpy as np
import pytest
import torch

import oracle
from paged_kv_flight_b200 import workloads
from tests._util import bits16, host_inputs, oracle_attn_threaded, oracle_cfg, bf16_ordinal
from tests.test_oracle_rope import _complex_rope


def _tiny():
    return workloads.make("tiny", device="cpu")


def _small(kv_fp8=False, lengths=(0, 5, 31, 32, 77), Hq=8, Hkv=2, d=64, P=16, seed=11):
    return workloads.build("small", Hq, Hkv, d, P, kv_fp8, 1e4, lengths, seed, device="cpu")


def _gather(h, w, b, kvh, n, pool_key, scale_key):
    """numpy fancy-index gather of n tokens of (b, kvh), dequantised."""
    t = np.arange(n)
    pages = h["block_tables"][b, t // w.P]
    raw = h[pool_key][pages, kvh, t % w.P, :]
    if w.kv_fp8:
        vals = torch.from_numpy(raw.copy()).view(torch.float8_e4m3fn).double().numpy()
        return vals * h[scale_key][pages, kvh][:, None].astype(np.float64)
    return (raw.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


# ---- append ----------------------------------------------------------------

def test_append_touches_exactly_the_landing_slots_bf16():
    w = _tiny()
    h = host_inputs(w)
    k0, v0 = h["k_pool"].copy(), h["v_pool"].copy()
    st = oracle.rope_append(oracle_cfg(w), h["q"], h["k_new"], h["v_new"], h["k_pool"],
                            h["v_pool"], None, None, h["block_tables"], h["seq_lens"])
    assert st == 0
    changed_k = np.argwhere((h["k_pool"] != k0).any(-1))
    changed_v = np.argwhere((h["v_pool"] != v0).any(-1))
    expect = set()
    for b, L in enumerate(w.seq_lens):
        page = w.block_tables[b, L // w.P]
        for kvh in range(w.Hkv):
            expect.add((int(page), kvh, int(L % w.P)))
            # v copied bit for bit
            assert np.array_equal(h["v_pool"][page, kvh, L % w.P], h["v_new"][b, kvh])
    assert {tuple(map(int, r)) for r in changed_v} == expect
    assert {tuple(map(int, r)) for r in changed_k} <= expect
    # slot cases of the tiny config: 17 -> slot 1, 64 -> fresh page slot 0,
    # 100 -> slot 4, 255 -> last slot 15
    assert [int(L % w.P) for L in w.seq_lens] == [1, 0, 4, 15]


def test_append_k_and_q_are_rope_rounded_to_bf16():
    w = _tiny()
    h = host_inputs(w)
    q_in, k_in = h["q"].copy(), h["k_new"].copy()
    oracle.rope_append(oracle_cfg(w), h["q"], h["k_new"], h["v_new"], h["k_pool"], h["v_pool"],
                       None, None, h["block_tables"], h["seq_lens"])
    f = lambda bits: (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    for b, L in enumerate(w.seq_lens):
        q_ref = _complex_rope(f(q_in[b]), int(L), w.rope_base)
        k_ref = _complex_rope(f(k_in[b]), int(L), w.rope_base)
        q_ref_bits = torch.from_numpy(q_ref).float().to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        k_ref_bits = torch.from_numpy(k_ref).float().to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        # torch's double->bf16 goes through float (two roundings), so allow one step
        assert np.abs(bf16_ordinal(h["q"][b]) - bf16_ordinal(q_ref_bits)).max() <= 1
        page = w.block_tables[b, L // w.P]
        got_k = h["k_pool"][page, :, L % w.P, :]
        assert np.abs(bf16_ordinal(got_k) - bf16_ordinal(k_ref_bits)).max() <= 1


def test_append_fp8_codes_match_library_cast():
    w = _small(kv_fp8=True, lengths=(3, 40, 64, 90), Hq=4, Hkv=2, d=64, P=32)
    h = host_inputs(w)
    k_in = h["k_new"].copy()
    st = oracle.rope_append(oracle_cfg(w), h["q"], h["k_new"], h["v_new"], h["k_pool"],
                            h["v_pool"], h["k_scale"], h["v_scale"], h["block_tables"],
                            h["seq_lens"])
    assert st == 0
    f = lambda bits: (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    for b, L in enumerate(w.seq_lens):
        page = w.block_tables[b, L // w.P]
        for kvh in range(w.Hkv):
            sv = float(h["v_scale"][page, kvh])
            sk = float(h["k_scale"][page, kvh])
            v32 = (f(h["v_new"][b, kvh]) / sv).astype(np.float32)
            v_ref = torch.from_numpy(np.clip(v32, -448, 448)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
            assert np.array_equal(h["v_pool"][page, kvh, L % w.P], v_ref)
            k32 = (_complex_rope(f(k_in[b, kvh]), int(L), w.rope_base) / sk).astype(np.float32)
            k_ref = torch.from_numpy(np.clip(k32, -448, 448)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
            got = h["k_pool"][page, kvh, L % w.P]
            # independent RoPE may differ in the last fp64 bit: at most one code step
            assert np.abs(got.astype(int) - k_ref.astype(int)).max() <= 1


# ---- attention ---------------------------------------------------------------

@pytest.mark.parametrize("kv_fp8", [False, True])
def test_attention_matches_library_sdpa_fp64(kv_fp8):
    w = _small(kv_fp8=kv_fp8)
    h = host_inputs(w)
    cfg = oracle_cfg(w)
    oracle.rope_append(cfg, h["q"], h["k_new"], h["v_new"], h["k_pool"], h["v_pool"],
                       h["k_scale"], h["v_scale"], h["block_tables"], h["seq_lens"])
    out, st = oracle.decode_attn(cfg, h["q"], h["k_pool"], h["v_pool"], h["k_scale"],
                                 h["v_scale"], h["block_tables"], h["seq_lens"])
    assert st == 0
    G = w.Hq // w.Hkv
    qf = (h["q"].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    for b, L in enumerate(w.seq_lens):
        n = int(L) + 1
        K = np.stack([_gather(h, w, b, kvh, n, "k_pool", "k_scale") for kvh in range(w.Hkv)])
        V = np.stack([_gather(h, w, b, kvh, n, "v_pool", "v_scale") for kvh in range(w.Hkv)])
        Kt = torch.from_numpy(K).repeat_interleave(G, dim=0)    # [Hq, n, d], head h -> kv h // G
        Vt = torch.from_numpy(V).repeat_interleave(G, dim=0)
        qt = torch.from_numpy(qf[b])[:, None, :]                 # [Hq, 1, d]
        ref = torch.nn.functional.scaled_dot_product_attention(qt, Kt, Vt)[:, 0, :].numpy()
        assert np.allclose(out[b], ref, rtol=1e-12, atol=1e-13)


def test_attention_matches_brute_force_loops():
    w = _small(lengths=(2, 9), Hq=4, Hkv=2, d=8, P=4)
    h = host_inputs(w)
    cfg = oracle_cfg(w)
    oracle.rope_append(cfg, h["q"], h["k_new"], h["v_new"], h["k_pool"], h["v_pool"],
                       None, None, h["block_tables"], h["seq_lens"])
    out, st = oracle.decode_attn(cfg, h["q"], h["k_pool"], h["v_pool"], None, None,
                                 h["block_tables"], h["seq_lens"])
    assert st == 0
    dec = lambda u: float(np.array([u], np.uint32).__lshift__(16).view(np.float32)[0])
    G = w.Hq // w.Hkv
    for b in range(w.batch):
        n = int(w.seq_lens[b]) + 1
        for hh in range(w.Hq):
            kvh = hh // G
            scores = []
            for t in range(n):
                page = int(h["block_tables"][b][t // w.P])
                s = 0.0
                for j in range(w.d):
                    s += dec(h["q"][b][hh][j]) * dec(h["k_pool"][page][kvh][t % w.P][j])
                scores.append(s / math.sqrt(w.d))
            m = max(scores)
            e = [math.exp(s - m) for s in scores]
            for j in range(w.d):
                num = sum(e[t] * dec(h["v_pool"][int(h["block_tables"][b][t // w.P])][kvh][t % w.P][j])
                          for t in range(n))
                ref = num / sum(e)
                assert abs(out[b, hh, j] - ref) <= 1e-12 * max(1.0, abs(ref))


@pytest.mark.parametrize("kv_fp8", [False, True])
def test_one_token_context_returns_v_exactly(kv_fp8):
    w = _small(kv_fp8=kv_fp8, lengths=(0, 0, 0))
    h = host_inputs(w)
    cfg = oracle_cfg(w)
    oracle.rope_append(cfg, h["q"], h["k_new"], h["v_new"], h["k_pool"], h["v_pool"],
                       h["k_scale"], h["v_scale"], h["block_tables"], h["seq_lens"])
    out, st = oracle.decode_attn(cfg, h["q"], h["k_pool"], h["v_pool"], h["k_scale"],
                                 h["v_scale"], h["block_tables"], h["seq_lens"])
    assert st == 0
    G = w.Hq // w.Hkv
    for b in range(w.batch):
        page = w.block_tables[b, 0]
        for hh in range(w.Hq):
            v = _gather(h, w, b, hh // G, 1, "v_pool", "v_scale")[0]
            assert np.array_equal(out[b, hh], v)
        if not kv_fp8:
            # and that stored value is v_new itself, bit for bit
            assert np.array_equal(oracle.bf16_encode(out[b].reshape(w.Hkv, G, w.d)[:, 0]),
                                  h["v_new"][b])
            assert np.array_equal(h["v_pool"][page, :, 0], h["v_new"][b])


def _write_identical_keys(h, w, key_bits):
    for b, L in enumerate(w.seq_lens):
        for t in range(int(L) + 1):
            page = w.block_tables[b, t // w.P]
            h["k_pool"][page, :, t % w.P, :] = key_bits


def test_identical_keys_give_mean_of_values():
    w = _small(lengths=(6, 33, 70))
    h = host_inputs(w)
    cfg = oracle_cfg(w)
    oracle.rope_append(cfg, h["q"], h["k_new"], h["v_new"], h["k_pool"], h["v_pool"],
                       None, None, h["block_tables"], h["seq_lens"])
    # identical post-RoPE keys written straight into every attended slot
    key = bits16(torch.randn(w.Hkv, w.d, generator=torch.Generator().manual_seed(5)).to(torch.bfloat16))
    _write_identical_keys(h, w, key)
    out, st = oracle.decode_attn(cfg, h["q"], h["k_pool"], h["v_pool"], None, None,
                                 h["block_tables"], h["seq_lens"])
    assert st == 0
    G = w.Hq // w.Hkv
    for b, L in enumerate(w.seq_lens):
        for hh in range(w.Hq):
            V = _gather(h, w, b, hh // G, int(L) + 1, "v_pool", None)
            assert np.allclose(out[b, hh], V.mean(0), rtol=0, atol=1e-13)


def test_zero_query_gives_mean_of_values():
    w = _small(lengths=(1, 15, 16, 47))
    h = host_inputs(w)
    cfg = oracle_cfg(w)
    oracle.rope_append(cfg, h["q"], h["k_new"], h["v_new"], h["k_pool"], h["v_pool"],
                       None, None, h["block_tables"], h["seq_lens"])
    h["q"][:] = 0
    out, _ = oracle.decode_attn(cfg, h["q"], h["k_pool"], h["v_pool"], None, None,
                                h["block_tables"], h["seq_lens"])
    G = w.Hq // w.Hkv
    for b, L in enumerate(w.seq_lens):
        for hh in range(w.Hq):
            V = _gather(h, w, b, hh // G, int(L) + 1, "v_pool", None)
            assert np.allclose(out[b, hh], V.mean(0), rtol=0, atol=1e-13)


def _encode_exact(vals, kv_fp8):
    """Pool codes of values that both formats hold exactly (multiples of 1/4
    within +-1.5)."""
    t = torch.from_numpy(np.ascontiguousarray(vals, np.float32))
    if kv_fp8:
        return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    return bits16(t.to(torch.bfloat16))


@pytest.mark.parametrize("kv_fp8", [False, True])
def test_common_key_offset_shifts_scores_and_changes_nothing(kv_fp8):
    """softmax(s + c) = softmax(s): keys K_t and K_t + u (the same u for every
    token of a kv head) give scores that differ by the constant q.u / sqrt(d),
    so the output must not move beyond fp64 rounding."""
    w = _small(kv_fp8=kv_fp8, lengths=(5, 40, 70))
    h = host_inputs(w)
    cfg = oracle_cfg(w)
    oracle.rope_append(cfg, h["q"], h["k_new"], h["v_new"], h["k_pool"], h["v_pool"],
                       h["k_scale"], h["v_scale"], h["block_tables"], h["seq_lens"])
    rng = np.random.default_rng(9)
    if kv_fp8:                                    # unit scales: codes are the values themselves
        h["k_scale"][:] = 1.0
    base = rng.integers(-2, 3, size=h["k_pool"].shape) / 4.0           # K'  in {-0.5 .. 0.5}
    u = rng.integers(-4, 5, size=(w.Hkv, w.d)) / 4.0                   # u   in {-1 .. 1}
    shifted = base + u[None, :, None, :]                                # |K' + u| <= 1.5, exact
    h["k_pool"][:] = _encode_exact(base, kv_fp8)
    out0, st0 = oracle.decode_attn(cfg, h["q"], h["k_pool"], h["v_pool"], h["k_scale"], h["v_scale"],
                                   h["block_tables"], h["seq_lens"])
    h["k_pool"][:] = _encode_exact(shifted, kv_fp8)
    out1, st1 = oracle.decode_attn(cfg, h["q"], h["k_pool"], h["v_pool"], h["k_scale"], h["v_scale"],
                                   h["block_tables"], h["seq_lens"])
    assert st0 == 0 and st1 == 0
    # the offset really moves the scores (by q.u / sqrt(d), a few units here)
    qf = (h["q"].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    G = w.Hq // w.Hkv
    shift = np.einsum("bhd,hd->bh", qf, np.repeat(u, G, axis=0)) / math.sqrt(w.d)
    assert np.abs(shift).max() > 1.0
    assert np.allclose(out0, out1, rtol=0, atol=1e-12)
    assert np.abs(out0).max() > 0.1


@pytest.mark.parametrize("kv_fp8", [False, True])
def test_permuting_physical_pages_changes_nothing(kv_fp8):
    w = _small(kv_fp8=kv_fp8, lengths=(10, 50, 95))
    h = host_inputs(w)
    cfg = oracle_cfg(w)
    oracle.rope_append(cfg, h["q"], h["k_new"], h["v_new"], h["k_pool"], h["v_pool"],
                       h["k_scale"], h["v_scale"], h["block_tables"], h["seq_lens"])
    out, _ = oracle.decode_attn(cfg, h["q"], h["k_pool"], h["v_pool"], h["k_scale"],
                                h["v_scale"], h["block_tables"], h["seq_lens"])
    perm = np.random.default_rng(4).permutation(w.num_pages)      # old page p -> new perm[p]
    k2, v2 = np.empty_like(h["k_pool"]), np.empty_like(h["v_pool"])
    k2[perm], v2[perm] = h["k_pool"], h["v_pool"]
    bt2 = np.where(h["block_tables"] >= 0, perm[np.maximum(h["block_tables"], 0)], -1).astype(np.int32)
    ks2 = vs2 = None
    if kv_fp8:
        ks2, vs2 = np.empty_like(h["k_scale"]), np.empty_like(h["v_scale"])
        ks2[perm], vs2[perm] = h["k_scale"], h["v_scale"]
    out2, _ = oracle.decode_attn(cfg, h["q"], k2, v2, ks2, vs2, bt2, h["seq_lens"])
    assert np.array_equal(out, out2)


def test_out_of_range_requests_are_reported_and_skipped():
    w = _small(lengths=(5, 20))
    h = host_inputs(w)
    cfg = oracle_cfg(w)
    bad_len = h["seq_lens"].copy()
    bad_len[1] = w.bt_stride * w.P                 # past the block table
    k0 = h["k_pool"].copy()
    st = oracle.rope_append(cfg, h["q"], h["k_new"], h["v_new"], h["k_pool"], h["v_pool"],
                            None, None, h["block_tables"], bad_len)
    assert st == oracle.ORC_ERR_RANGE
    changed = np.argwhere((h["k_pool"] != k0).any(-1))
    assert len(changed) == w.Hkv                    # only request 0 appended
    bt = h["block_tables"].copy()
    bt[0, 0] = w.num_pages                          # page id out of range
    _, st = oracle.decode_attn(cfg, h["q"], h["k_pool"], h["v_pool"], None, None, bt, h["seq_lens"])
    assert st == oracle.ORC_ERR_RANGE


def test_tiny_regression_fixture():
    """The oracle still reproduces tests/golden/tiny_oracle.txt (written by
    tests/golden/make_golden.py, which calls only the generator and oracle/)."""
    import os
    from tests.golden.make_golden import rows
    path = os.path.join(os.path.dirname(__file__), "golden", "tiny_oracle.txt")
    with open(path) as f:
        stored = [ln.rstrip("\n") for ln in f if not ln.startswith("#")]
    assert rows() == stored


@pytest.mark.parametrize("kv_fp8,q_len", [(False, 1), (True, 1), (False, 3)])
def test_threaded_whole_batch_helper_equals_the_batch_call(kv_fp8, q_len):
    # the GPU tests' whole-batch oracle runs one C call per (request, new
    # token, kv head) on host threads; it must give exactly the batch call
    w = workloads.build("thr", 16, 4, 64, 16, kv_fp8, 1e4, [0, 15, 16, 200, 77, 513], seed=5, device="cpu",
                        q_len=q_len)
    h = host_inputs(w)
    cfg = oracle_cfg(w)
    if q_len == 1:
        assert oracle.rope_append(cfg, h["q"], h["k_new"], h["v_new"], h["k_pool"], h["v_pool"], h["k_scale"],
                                  h["v_scale"], h["block_tables"], h["seq_lens"]) == 0
        ref, st = oracle.decode_attn(cfg, h["q"], h["k_pool"], h["v_pool"], h["k_scale"], h["v_scale"],
                                     h["block_tables"], h["seq_lens"])
    else:
        assert oracle.rope_append_tokens(cfg, h["q"], h["k_new"], h["v_new"], h["k_pool"], h["v_pool"],
                                         h["k_scale"], h["v_scale"], h["block_tables"], h["seq_lens"]) == 0
        ref, st = oracle.decode_attn_tokens(cfg, h["q"], h["k_pool"], h["v_pool"], h["k_scale"], h["v_scale"],
                                            h["block_tables"], h["seq_lens"])
    assert st == 0
    out, st2 = oracle_attn_threaded(w, h, threads=4)
    assert st2 == 0
    assert out.shape == ref.shape and np.array_equal(out, ref)
