"""Pins for the oracle's several-new-tokens step (speculative-decode
verification: a draft proposes tokens and the target checks all of them in
one pass, "Scaling TensorRT-LLM: Kernel Fusion and Inflight Batching in
Production", section "3. Speculative Decoding for Tail Latency";
"TensorRT-LLM Guide: High-Throughput GPU Inference Engine", section
"2. Pipelined Speculative Decoding").

New token t of request b sits at position L_b + t and attends tokens
0 .. L_b + t.  The pins reach outside the oracle: slot placement from the
position arithmetic, an independent numpy complex rotation, an explicit
numpy softmax over a numpy gather, causality (tokens after t cannot move
token t's output), the identical-keys closed form, and reduction to the
single-token oracle (itself pinned elsewhere) when q_len = 1."""
import numpy as np
import pytest
import torch

import oracle
from paged_kv_flight_b200 import workloads
from tests._util import bf16_ordinal, bits16, host_inputs, oracle_cfg
from tests.test_oracle_rope import _complex_rope


def _tok(q_len=3, lengths=(0, 5, 14, 15, 31, 40), Hq=8, Hkv=2, d=64, P=16, seed=21, fp8=False):
    return workloads.build("tok", Hq, Hkv, d, P, fp8, 1e4, lengths, seed, device="cpu", q_len=q_len)


def _append(w, h):
    return oracle.rope_append_tokens(oracle_cfg(w), h["q"], h["k_new"], h["v_new"], h["k_pool"], h["v_pool"],
                                     h["k_scale"], h["v_scale"], h["block_tables"], h["seq_lens"])


def _f64(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def test_generator_gives_pages_for_every_new_token():
    w = _tok(q_len=4, lengths=(12, 13, 15, 28), P=16)
    for b, L in enumerate(w.seq_lens):
        need = (int(L) + 4 + w.P - 1) // w.P
        assert (w.block_tables[b, :need] >= 0).all()
    assert tuple(w.q.shape) == (4, 4, 8, 64) and tuple(w.k_new.shape) == (4, 4, 2, 64)


def test_append_places_each_new_token_at_its_position():
    w = _tok(q_len=3)
    h = host_inputs(w)
    k0, v0 = h["k_pool"].copy(), h["v_pool"].copy()
    assert _append(w, h) == 0
    expect = set()
    for b, L in enumerate(w.seq_lens):
        for t in range(3):
            pos = int(L) + t
            page = int(w.block_tables[b, pos // w.P])
            for kvh in range(w.Hkv):
                expect.add((page, kvh, pos % w.P))
                assert np.array_equal(h["v_pool"][page, kvh, pos % w.P], h["v_new"][b, t, kvh])
                # k: the independent complex rotation at position L + t, within 1 bf16 ulp
                ref = _complex_rope(_f64(bits16(w.k_new[b, t, kvh])), pos, w.rope_base)
                got = _f64(h["k_pool"][page, kvh, pos % w.P])
                ref_bits = bits16(torch.from_numpy(ref).to(torch.bfloat16))
                assert np.abs(bf16_ordinal(h["k_pool"][page, kvh, pos % w.P]) - bf16_ordinal(ref_bits)).max() <= 1
                assert np.isfinite(got).all()
    changed_v = {tuple(map(int, r)) for r in np.argwhere((h["v_pool"] != v0).any(-1))}
    changed_k = {tuple(map(int, r)) for r in np.argwhere((h["k_pool"] != k0).any(-1))}
    assert changed_v == expect and changed_k <= expect


def test_q_rotated_at_each_tokens_position():
    w = _tok(q_len=2)
    h = host_inputs(w)
    q0 = h["q"].copy()
    assert _append(w, h) == 0
    for b, L in enumerate(w.seq_lens):
        for t in range(2):
            ref = _complex_rope(_f64(q0[b, t]), int(L) + t, w.rope_base)
            ref_bits = bits16(torch.from_numpy(ref).to(torch.bfloat16))
            assert np.abs(bf16_ordinal(h["q"][b, t]) - bf16_ordinal(ref_bits)).max() <= 1


@pytest.mark.parametrize("fp8", [False, True])
def test_one_new_token_is_the_single_token_step(fp8):
    # same draws through the single-token generator path and a token axis of 1
    w1 = workloads.build("one", 8, 2, 64, 16, fp8, 1e4, [3, 17, 40], 5, device="cpu")
    h1 = host_inputs(w1)
    ht = {k: (v.copy() if isinstance(v, np.ndarray) else v) for k, v in h1.items()}
    for k in ("q", "k_new", "v_new"):
        ht[k] = ht[k][:, None].copy()
    cfg = oracle_cfg(w1)
    assert oracle.rope_append(cfg, h1["q"], h1["k_new"], h1["v_new"], h1["k_pool"], h1["v_pool"], h1["k_scale"],
                              h1["v_scale"], h1["block_tables"], h1["seq_lens"]) == 0
    assert oracle.rope_append_tokens(cfg, ht["q"], ht["k_new"], ht["v_new"], ht["k_pool"], ht["v_pool"],
                                     ht["k_scale"], ht["v_scale"], ht["block_tables"], ht["seq_lens"]) == 0
    assert np.array_equal(h1["k_pool"], ht["k_pool"]) and np.array_equal(h1["v_pool"], ht["v_pool"])
    o1, s1 = oracle.decode_attn(cfg, h1["q"], h1["k_pool"], h1["v_pool"], h1["k_scale"], h1["v_scale"],
                                h1["block_tables"], h1["seq_lens"])
    ot, st = oracle.decode_attn_tokens(cfg, ht["q"], ht["k_pool"], ht["v_pool"], ht["k_scale"], ht["v_scale"],
                                       ht["block_tables"], ht["seq_lens"])
    assert s1 == 0 and st == 0
    assert np.array_equal(o1, ot[:, 0])


def test_brute_force_softmax_over_the_causal_prefix():
    w = _tok(q_len=3, lengths=(0, 7, 16, 33))
    h = host_inputs(w)
    assert _append(w, h) == 0
    out, st = oracle.decode_attn_tokens(oracle_cfg(w), h["q"], h["k_pool"], h["v_pool"], None, None,
                                        h["block_tables"], h["seq_lens"])
    assert st == 0
    G = w.Hq // w.Hkv
    for b, L in enumerate(w.seq_lens):
        for t in range(3):
            n = int(L) + t + 1
            tok = np.arange(n)
            pages = h["block_tables"][b, tok // w.P]
            for kvh in range(w.Hkv):
                K = _f64(h["k_pool"][pages, kvh, tok % w.P])
                V = _f64(h["v_pool"][pages, kvh, tok % w.P])
                for g in range(G):
                    qv = _f64(h["q"][b, t, kvh * G + g])
                    s = K @ qv / np.sqrt(w.d)
                    p = np.exp(s - s.max())
                    ref = (p / p.sum()) @ V
                    np.testing.assert_allclose(out[b, t, kvh * G + g], ref, rtol=0, atol=1e-12)


def test_tokens_after_t_do_not_move_token_t():
    w = _tok(q_len=4, lengths=(3, 20, 47))
    h = host_inputs(w)
    h2 = {k: (v.copy() if isinstance(v, np.ndarray) else v) for k, v in h.items()}
    # different k/v for the last two new tokens only
    rng = np.random.default_rng(3)
    for key in ("k_new", "v_new"):
        noise = torch.from_numpy(rng.standard_normal(h2[key][:, 2:].shape)).to(torch.bfloat16)
        h2[key][:, 2:] = bits16(noise)
    assert _append(w, h) == 0 and _append(w, h2) == 0
    cfg = oracle_cfg(w)
    o1, _ = oracle.decode_attn_tokens(cfg, h["q"], h["k_pool"], h["v_pool"], None, None,
                                      h["block_tables"], h["seq_lens"])
    o2, _ = oracle.decode_attn_tokens(cfg, h2["q"], h2["k_pool"], h2["v_pool"], None, None,
                                      h2["block_tables"], h2["seq_lens"])
    assert np.array_equal(o1[:, :2], o2[:, :2])          # tokens 0, 1 cannot see tokens 2, 3
    assert not np.allclose(o1[:, 2:], o2[:, 2:])          # tokens 2, 3 see themselves


def test_identical_keys_give_the_mean_of_the_visible_values():
    w = _tok(q_len=3, lengths=(4, 30))
    h = host_inputs(w)
    assert _append(w, h) == 0
    key = bits16(torch.randn(w.Hkv, w.d, generator=torch.Generator().manual_seed(2)).to(torch.bfloat16))
    for b, L in enumerate(w.seq_lens):
        for tpos in range(int(L) + 3):
            page = h["block_tables"][b, tpos // w.P]
            h["k_pool"][page, :, tpos % w.P] = key
    out, st = oracle.decode_attn_tokens(oracle_cfg(w), h["q"], h["k_pool"], h["v_pool"], None, None,
                                        h["block_tables"], h["seq_lens"])
    assert st == 0
    G = w.Hq // w.Hkv
    for b, L in enumerate(w.seq_lens):
        for t in range(3):
            n = int(L) + t + 1
            tok = np.arange(n)
            pages = h["block_tables"][b, tok // w.P]
            for kvh in range(w.Hkv):
                mean = _f64(h["v_pool"][pages, kvh, tok % w.P]).mean(0)
                for g in range(G):
                    np.testing.assert_allclose(out[b, t, kvh * G + g], mean, rtol=0, atol=1e-12)


def test_position_past_the_block_table_is_a_range_error():
    w = _tok(q_len=2, lengths=(15,), P=16)           # tokens at 15 and 16: two pages
    h = host_inputs(w)
    bt = h["block_tables"][:, :1].copy()             # a table of one page: position 16 has no page
    st = oracle.rope_append_tokens(oracle_cfg(w), h["q"], h["k_new"], h["v_new"], h["k_pool"], h["v_pool"],
                                   None, None, bt, h["seq_lens"])
    assert st == oracle.ORC_ERR_RANGE
