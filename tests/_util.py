"""Helpers shared by the tests: marshal a generated workload into the numpy
arrays the oracle takes, and compare results.  No step arithmetic here."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from paged_kv_flight_b200.workloads import Workload


def bits16(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> uint16 bit patterns (host copy)."""
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16).copy()


def bytes8(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().cpu().numpy().view(np.uint8).copy()


def pool_np(w: Workload, t: torch.Tensor) -> np.ndarray:
    return bytes8(t) if w.kv_fp8 else bits16(t)


def oracle_cfg(w: Workload) -> oracle.OracleConfig:
    return oracle.OracleConfig(w.Hq, w.Hkv, w.d, w.P, w.kv_fp8, w.num_pages, w.rope_base)


def host_inputs(w: Workload) -> dict:
    """Fresh host copies of every input of the step, in oracle form."""
    return dict(
        q=bits16(w.q), k_new=bits16(w.k_new), v_new=bits16(w.v_new),
        k_pool=pool_np(w, w.k_pool), v_pool=pool_np(w, w.v_pool),
        k_scale=None if w.k_scale is None else w.k_scale.detach().cpu().numpy().copy(),
        v_scale=None if w.v_scale is None else w.v_scale.detach().cpu().numpy().copy(),
        block_tables=np.ascontiguousarray(w.block_tables, np.int32),
        seq_lens=np.ascontiguousarray(w.seq_lens, np.int32),
    )


def oracle_step(w: Workload, h: dict | None = None):
    """Run the oracle's append + attention on host copies; returns (h, out, st)."""
    h = host_inputs(w) if h is None else h
    cfg = oracle_cfg(w)
    st1 = oracle.rope_append(cfg, h["q"], h["k_new"], h["v_new"], h["k_pool"], h["v_pool"],
                             h["k_scale"], h["v_scale"], h["block_tables"], h["seq_lens"])
    out, st2 = oracle.decode_attn(cfg, h["q"], h["k_pool"], h["v_pool"], h["k_scale"],
                                  h["v_scale"], h["block_tables"], h["seq_lens"])
    return h, out, max(st1, st2)


def bf16_ordinal(bits: np.ndarray) -> np.ndarray:
    """Monotone integer image of bf16 bit patterns (sign-magnitude -> ordinal),
    so that |ordinal(a) - ordinal(b)| counts representable steps."""
    b = bits.astype(np.int64)
    mag = b & 0x7FFF
    return np.where(b & 0x8000, -mag, mag)


def f64_of_bf16_tensor(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def varlen_host(w: Workload, q_lens) -> dict:
    """Host inputs of a varlen step from a several-new-tokens workload (token
    axis of at least max(q_lens), pages for them): request b keeps its first
    q_lens[b] new tokens, packed in request order, and cu_q [batch + 1]."""
    h = host_inputs(w)
    q_lens = np.asarray(q_lens, np.int64)
    assert len(q_lens) == w.batch and (q_lens <= w.q_len).all()
    cu = np.zeros(w.batch + 1, np.int32)
    cu[1:] = np.cumsum(q_lens)
    for key in ("q", "k_new", "v_new"):
        h[key] = np.ascontiguousarray(np.concatenate([h[key][b, :int(q)] for b, q in enumerate(q_lens)]))
    h["cu_q"] = cu
    return h


def oracle_attn_threaded(w: Workload, h: dict, threads: int | None = None):
    """The oracle's attention of the whole batch, every (request, new token,
    kv head) group in its own call of the single-threaded C functions, the
    calls spread over host threads (the C library keeps no state and ctypes
    releases the GIL), longest requests first.  Returns (out, status) like
    oracle.decode_attn / decode_attn_tokens: [batch, Hq, d] for one new token
    per request, [batch, q_len, Hq, d] for several."""
    import os
    from concurrent.futures import ThreadPoolExecutor

    cfg = oracle_cfg(w)
    G = w.Hq // w.Hkv
    tok = w.q_len > 1
    shape = (w.batch, w.q_len, w.Hq, w.d) if tok else (w.batch, w.Hq, w.d)
    out = np.full(shape, np.nan)
    order = np.argsort(-np.asarray(w.seq_lens, np.int64), kind="stable")
    jobs = [(int(b), t, kvh) for b in order for t in range(w.q_len) for kvh in range(w.Hkv)]

    def run(job):
        b, t, kvh = job
        if tok:
            o, st = oracle.decode_attn_tokens_group(cfg, h["q"], h["k_pool"], h["v_pool"], h["k_scale"],
                                                    h["v_scale"], h["block_tables"], h["seq_lens"], b, t, kvh)
            out[b, t, kvh * G:(kvh + 1) * G] = o
        else:
            o, st = oracle.decode_attn_group(cfg, h["q"], h["k_pool"], h["v_pool"], h["k_scale"], h["v_scale"],
                                             h["block_tables"], h["seq_lens"], b, kvh)
            out[b, kvh * G:(kvh + 1) * G] = o
        return st

    n = threads or max(1, min(32, (os.cpu_count() or 1)))
    with ThreadPoolExecutor(max_workers=n) as ex:
        status = max(ex.map(run, jobs), default=0)
    return out, status
