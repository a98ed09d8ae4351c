"""Pins for the oracle's varlen step: a different number of new tokens per
request, packed (chunked prefill mixed with decode in one batch, "Scaling
TensorRT-LLM: Kernel Fusion and Inflight Batching in Production", section
"What the Scheduler Actually Does").  Token i of request b sits at position
L_b + i - cu_q[b] and attends tokens 0 .. that position.

The oracle composes the several-new-tokens functions request by request; the
pins reach outside that composition: every request decoding one token is the
single-token step (other C functions), equal counts are the batched
several-new-tokens call (one call over the whole batch, not per request), an
explicit numpy softmax over a numpy gather of the causal prefix on a mixed
batch, and a request with no new token changes nothing."""
import numpy as np

import oracle
from paged_kv_flight_b200 import workloads
from tests._util import host_inputs, oracle_cfg, varlen_host


def _f64(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _w(q_len, lengths, seed=31, Hq=8, Hkv=2, d=64, P=16):
    return workloads.build("vl", Hq, Hkv, d, P, False, 1e4, lengths, seed, device="cpu", q_len=q_len)


def _run(w, h):
    cfg = oracle_cfg(w)
    st = oracle.rope_append_varlen(cfg, h["q"], h["k_new"], h["v_new"], h["k_pool"], h["v_pool"], None, None,
                                   h["block_tables"], h["seq_lens"], h["cu_q"])
    out, st2 = oracle.decode_attn_varlen(cfg, h["q"], h["k_pool"], h["v_pool"], None, None, h["block_tables"],
                                         h["seq_lens"], h["cu_q"])
    return out, st | st2


def test_one_token_each_is_the_single_token_step():
    w1 = workloads.build("one", 8, 2, 64, 16, False, 1e4, [3, 17, 40, 0], 5, device="cpu")
    h1 = host_inputs(w1)
    hv = {k: (v.copy() if isinstance(v, np.ndarray) else v) for k, v in h1.items()}
    hv["cu_q"] = np.arange(w1.batch + 1, dtype=np.int32)
    cfg = oracle_cfg(w1)
    assert oracle.rope_append(cfg, h1["q"], h1["k_new"], h1["v_new"], h1["k_pool"], h1["v_pool"], None, None,
                              h1["block_tables"], h1["seq_lens"]) == 0
    o1, s1 = oracle.decode_attn(cfg, h1["q"], h1["k_pool"], h1["v_pool"], None, None, h1["block_tables"],
                                h1["seq_lens"])
    ov, sv = _run(w1, hv)
    assert s1 == 0 and sv == 0
    assert np.array_equal(h1["k_pool"], hv["k_pool"]) and np.array_equal(h1["v_pool"], hv["v_pool"])
    assert np.array_equal(h1["q"], hv["q"]) and np.array_equal(o1, ov)


def test_equal_counts_are_the_batched_tokens_step():
    w = _w(3, [0, 9, 30, 47])
    h = host_inputs(w)
    hv = varlen_host(w, [3, 3, 3, 3])
    cfg = oracle_cfg(w)
    assert oracle.rope_append_tokens(cfg, h["q"], h["k_new"], h["v_new"], h["k_pool"], h["v_pool"], None, None,
                                     h["block_tables"], h["seq_lens"]) == 0
    ob, sb = oracle.decode_attn_tokens(cfg, h["q"], h["k_pool"], h["v_pool"], None, None, h["block_tables"],
                                       h["seq_lens"])
    ov, sv = _run(w, hv)
    assert sb == 0 and sv == 0
    assert np.array_equal(h["k_pool"], hv["k_pool"]) and np.array_equal(h["v_pool"], hv["v_pool"])
    assert np.array_equal(ob.reshape(-1, w.Hq, w.d), ov)


def test_mixed_counts_against_a_numpy_softmax():
    q_lens = [1, 5, 0, 16, 2]
    w = _w(16, [4, 0, 11, 30, 63])
    h = varlen_host(w, q_lens)
    out, st = _run(w, h)
    assert st == 0
    G = w.Hq // w.Hkv
    for b, L in enumerate(w.seq_lens):
        for t in range(q_lens[b]):
            i = int(h["cu_q"][b]) + t
            n = int(L) + t + 1
            tok = np.arange(n)
            pages = h["block_tables"][b, tok // w.P]
            for kvh in range(w.Hkv):
                K = _f64(h["k_pool"][pages, kvh, tok % w.P])
                V = _f64(h["v_pool"][pages, kvh, tok % w.P])
                for g in range(G):
                    qv = _f64(h["q"][i, kvh * G + g])
                    s = K @ qv / np.sqrt(w.d)
                    p = np.exp(s - s.max())
                    np.testing.assert_allclose(out[i, kvh * G + g], (p / p.sum()) @ V, rtol=0, atol=1e-12)


def test_a_request_without_new_tokens_changes_nothing():
    w = _w(4, [5, 18, 33])
    h0 = varlen_host(w, [2, 4, 3])
    h1 = varlen_host(w, [2, 0, 3])
    k_before = h1["k_pool"].copy()
    _run(w, h0)
    out1, st = _run(w, h1)
    assert st == 0
    # request 1's landing slots keep their (NaN sentinel) contents
    for t in range(4):
        pos = int(w.seq_lens[1]) + t
        page = int(w.block_tables[1, pos // w.P])
        assert np.array_equal(h1["k_pool"][page, :, pos % w.P], k_before[page, :, pos % w.P])
    # the other requests' tokens are what they are with request 1 decoding
    a0, a2 = slice(0, 2), slice(6, 9)
    assert np.array_equal(out1[0:2], _run(w, varlen_host(w, [2, 4, 3]))[0][a0])
    assert np.array_equal(out1[2:5], _run(w, varlen_host(w, [2, 4, 3]))[0][a2])


def test_e4m3_append_one_token_each_is_the_single_token_append():
    w1 = workloads.build("onef", 8, 2, 64, 16, True, 1e4, [3, 17, 40, 0], 6, device="cpu")
    h1 = host_inputs(w1)
    hv = {k: (v.copy() if isinstance(v, np.ndarray) else v) for k, v in h1.items()}
    cfg = oracle_cfg(w1)
    assert oracle.rope_append(cfg, h1["q"], h1["k_new"], h1["v_new"], h1["k_pool"], h1["v_pool"], h1["k_scale"],
                              h1["v_scale"], h1["block_tables"], h1["seq_lens"]) == 0
    assert oracle.rope_append_varlen(cfg, hv["q"], hv["k_new"], hv["v_new"], hv["k_pool"], hv["v_pool"],
                                     hv["k_scale"], hv["v_scale"], hv["block_tables"], hv["seq_lens"],
                                     np.arange(w1.batch + 1, dtype=np.int32)) == 0
    assert np.array_equal(h1["k_pool"], hv["k_pool"]) and np.array_equal(h1["v_pool"], hv["v_pool"])
    assert np.array_equal(h1["q"], hv["q"])
