"""CPU fp64 oracle for the paged-KV decode step (test infrastructure only).

Only the test suite, ``__graft_entry__.smoke()`` and the benchmark's
CPU-baseline / reference legs may import this package.  It wraps the plain C
library built from ``oracle/pkv_oracle.c`` (single-threaded, fp64) through
ctypes and numpy; it imports nothing from the GPU package and the GPU package
imports nothing from it.

Arrays are numpy: bf16 tensors as uint16 bit patterns, E4M3 as uint8 codes,
pools ``[num_pages, Hkv, P, d]``, block tables ``[batch, bt_stride]`` int32,
``seq_lens[b]`` = tokens cached before the step, scales
``[num_pages, Hkv]`` float32.
"""
from __future__ import annotations

import ctypes as C
from dataclasses import dataclass

import numpy as np

from . import build as _build

ORC_OK, ORC_ERR_ARG, ORC_ERR_RANGE = 0, 1, 2


class _Cfg(C.Structure):
    _fields_ = [("num_q_heads", C.c_int), ("num_kv_heads", C.c_int),
                ("head_dim", C.c_int), ("page_size", C.c_int),
                ("kv_fp8", C.c_int), ("num_pages", C.c_int),
                ("rope_base", C.c_double)]


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = C.CDLL(_build.build())
        P = C.c_void_p
        lib.orc_bf16_decode_n.argtypes = [P, P, C.c_longlong]
        lib.orc_bf16_encode_rne_n.argtypes = [P, P, C.c_longlong]
        lib.orc_e4m3_decode_n.argtypes = [P, P, C.c_longlong]
        lib.orc_e4m3_encode_satfinite_n.argtypes = [P, P, C.c_longlong]
        for f in (lib.orc_bf16_decode_n, lib.orc_bf16_encode_rne_n,
                  lib.orc_e4m3_decode_n, lib.orc_e4m3_encode_satfinite_n):
            f.restype = None
        lib.orc_rope_f64.argtypes = [P, P, C.c_int, C.c_double, C.c_double]
        lib.orc_rope_f64.restype = None
        lib.orc_rope_append.argtypes = [C.POINTER(_Cfg), P, P, P, P, P, P, P, P,
                                        C.c_int, P, C.c_int]
        lib.orc_rope_append.restype = C.c_int
        lib.orc_decode_attn_group.argtypes = [C.POINTER(_Cfg), P, P, P, P, P, P,
                                              C.c_int, P, C.c_int, C.c_int, P]
        lib.orc_decode_attn_group.restype = C.c_int
        lib.orc_decode_attn.argtypes = [C.POINTER(_Cfg), P, P, P, P, P, P, C.c_int,
                                        P, C.c_int, P]
        lib.orc_decode_attn.restype = C.c_int
        lib.orc_rope_append_tokens.argtypes = [C.POINTER(_Cfg), P, P, P, P, P, P, P, P,
                                               C.c_int, P, C.c_int, C.c_int]
        lib.orc_rope_append_tokens.restype = C.c_int
        lib.orc_decode_attn_tokens_group.argtypes = [C.POINTER(_Cfg), P, P, P, P, P, P, C.c_int, P,
                                                     C.c_int, C.c_int, C.c_int, C.c_int, P]
        lib.orc_decode_attn_tokens_group.restype = C.c_int
        lib.orc_decode_attn_tokens.argtypes = [C.POINTER(_Cfg), P, P, P, P, P, P, C.c_int, P,
                                               C.c_int, C.c_int, P]
        lib.orc_decode_attn_tokens.restype = C.c_int
        lib.orc_project_bf16.argtypes = [P, P, C.c_int, C.c_int, C.c_int, P]
        lib.orc_project_bf16.restype = C.c_int
        _lib = lib
    return _lib


@dataclass(frozen=True)
class OracleConfig:
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    page_size: int
    kv_fp8: bool
    num_pages: int
    rope_base: float

    def _c(self) -> _Cfg:
        return _Cfg(self.num_q_heads, self.num_kv_heads, self.head_dim, self.page_size,
                    int(bool(self.kv_fp8)), self.num_pages, float(self.rope_base))


def _ptr(a):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def _need(a, dtype, name):
    if not isinstance(a, np.ndarray) or a.dtype != dtype or not a.flags.c_contiguous:
        raise TypeError(f"{name}: expected a C-contiguous numpy {np.dtype(dtype)} array")
    return a


# ---- codecs ---------------------------------------------------------------

def bf16_decode(bits: np.ndarray) -> np.ndarray:
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    out = np.empty(bits.shape, np.float64)
    _load().orc_bf16_decode_n(_ptr(bits), _ptr(out), bits.size)
    return out


def bf16_encode(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float64)
    out = np.empty(x.shape, np.uint16)
    _load().orc_bf16_encode_rne_n(_ptr(x), _ptr(out), x.size)
    return out


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    out = np.empty(codes.shape, np.float64)
    _load().orc_e4m3_decode_n(_ptr(codes), _ptr(out), codes.size)
    return out


def e4m3_encode(x: np.ndarray) -> np.ndarray:
    """E4M3 RNE with saturation to +-448; the input is taken as float32."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, np.uint8)
    _load().orc_e4m3_encode_satfinite_n(_ptr(x), _ptr(out), x.size)
    return out


# ---- RoPE -----------------------------------------------------------------

def rope(x: np.ndarray, pos: float, base: float) -> np.ndarray:
    """Rotate-half RoPE of the last axis of x (fp64) at position pos."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    d = x.shape[-1]
    out = np.empty_like(x)
    flat_in, flat_out = x.reshape(-1, d), out.reshape(-1, d)
    lib = _load()
    for r in range(flat_in.shape[0]):
        lib.orc_rope_f64(_ptr(flat_in[r]), _ptr(flat_out[r]), d, float(pos), float(base))
    return out


# ---- the step ---------------------------------------------------------------

def _pool_dtype(cfg: OracleConfig):
    return np.uint8 if cfg.kv_fp8 else np.uint16


def rope_append(cfg: OracleConfig, q, k_new, v_new, k_pool, v_pool, k_scale, v_scale,
                block_tables, seq_lens) -> int:
    """In place: rotates q, writes k/v of the new token into the pools.

    Returns the oracle status (0 ok, 2 if a request's length or page id is out
    of range; such requests are skipped)."""
    _need(q, np.uint16, "q"); _need(k_new, np.uint16, "k_new"); _need(v_new, np.uint16, "v_new")
    _need(k_pool, _pool_dtype(cfg), "k_pool"); _need(v_pool, _pool_dtype(cfg), "v_pool")
    _need(block_tables, np.int32, "block_tables"); _need(seq_lens, np.int32, "seq_lens")
    if cfg.kv_fp8:
        _need(k_scale, np.float32, "k_scale"); _need(v_scale, np.float32, "v_scale")
    c = cfg._c()
    return _load().orc_rope_append(C.byref(c), _ptr(q), _ptr(k_new), _ptr(v_new),
                                   _ptr(k_pool), _ptr(v_pool), _ptr(k_scale), _ptr(v_scale),
                                   _ptr(block_tables), block_tables.shape[1],
                                   _ptr(seq_lens), seq_lens.shape[0])


def decode_attn_group(cfg: OracleConfig, q, k_pool, v_pool, k_scale, v_scale,
                      block_tables, seq_lens, b: int, kvh: int):
    """fp64 output [G, d] of request b, kv head kvh; (out, status)."""
    G = cfg.num_q_heads // cfg.num_kv_heads
    out = np.zeros((G, cfg.head_dim), np.float64)
    c = cfg._c()
    st = _load().orc_decode_attn_group(C.byref(c), _ptr(q), _ptr(k_pool), _ptr(v_pool),
                                       _ptr(k_scale), _ptr(v_scale), _ptr(block_tables),
                                       block_tables.shape[1], _ptr(seq_lens), int(b), int(kvh),
                                       _ptr(out))
    return out, st


def decode_attn(cfg: OracleConfig, q, k_pool, v_pool, k_scale, v_scale, block_tables,
                seq_lens):
    """fp64 output [batch, Hq, d]; (out, status)."""
    _need(q, np.uint16, "q")
    _need(k_pool, _pool_dtype(cfg), "k_pool"); _need(v_pool, _pool_dtype(cfg), "v_pool")
    _need(block_tables, np.int32, "block_tables"); _need(seq_lens, np.int32, "seq_lens")
    B = seq_lens.shape[0]
    out = np.zeros((B, cfg.num_q_heads, cfg.head_dim), np.float64)
    c = cfg._c()
    st = _load().orc_decode_attn(C.byref(c), _ptr(q), _ptr(k_pool), _ptr(v_pool),
                                 _ptr(k_scale), _ptr(v_scale), _ptr(block_tables),
                                 block_tables.shape[1], _ptr(seq_lens), B, _ptr(out))
    return out, st


# ---- several new tokens per request (speculative-decode verification) ------

def rope_append_tokens(cfg: OracleConfig, q, k_new, v_new, k_pool, v_pool, k_scale, v_scale,
                       block_tables, seq_lens) -> int:
    """In place, for q [batch, q_len, Hq, d] and k_new / v_new [batch, q_len,
    Hkv, d]: new token t of request b is rotated at position L_b + t and its
    k / v stored in that position's page slot.  Returns the oracle status."""
    _need(q, np.uint16, "q"); _need(k_new, np.uint16, "k_new"); _need(v_new, np.uint16, "v_new")
    _need(k_pool, _pool_dtype(cfg), "k_pool"); _need(v_pool, _pool_dtype(cfg), "v_pool")
    _need(block_tables, np.int32, "block_tables"); _need(seq_lens, np.int32, "seq_lens")
    if cfg.kv_fp8:
        _need(k_scale, np.float32, "k_scale"); _need(v_scale, np.float32, "v_scale")
    B, Q = q.shape[0], q.shape[1]
    c = cfg._c()
    return _load().orc_rope_append_tokens(C.byref(c), _ptr(q), _ptr(k_new), _ptr(v_new),
                                          _ptr(k_pool), _ptr(v_pool), _ptr(k_scale), _ptr(v_scale),
                                          _ptr(block_tables), block_tables.shape[1],
                                          _ptr(seq_lens), B, Q)


def decode_attn_tokens_group(cfg: OracleConfig, q, k_pool, v_pool, k_scale, v_scale,
                             block_tables, seq_lens, b: int, t: int, kvh: int):
    """fp64 output [G, d] of new token t of request b, kv head kvh (it attends
    tokens 0 .. L_b + t); (out, status).  q is [batch, q_len, Hq, d]."""
    G = cfg.num_q_heads // cfg.num_kv_heads
    out = np.zeros((G, cfg.head_dim), np.float64)
    c = cfg._c()
    st = _load().orc_decode_attn_tokens_group(C.byref(c), _ptr(q), _ptr(k_pool), _ptr(v_pool),
                                              _ptr(k_scale), _ptr(v_scale), _ptr(block_tables),
                                              block_tables.shape[1], _ptr(seq_lens), q.shape[1],
                                              int(b), int(t), int(kvh), _ptr(out))
    return out, st


def decode_attn_tokens(cfg: OracleConfig, q, k_pool, v_pool, k_scale, v_scale, block_tables,
                       seq_lens):
    """fp64 output [batch, q_len, Hq, d]; (out, status)."""
    _need(q, np.uint16, "q")
    _need(k_pool, _pool_dtype(cfg), "k_pool"); _need(v_pool, _pool_dtype(cfg), "v_pool")
    _need(block_tables, np.int32, "block_tables"); _need(seq_lens, np.int32, "seq_lens")
    B, Q = q.shape[0], q.shape[1]
    out = np.zeros((B, Q, cfg.num_q_heads, cfg.head_dim), np.float64)
    c = cfg._c()
    st = _load().orc_decode_attn_tokens(C.byref(c), _ptr(q), _ptr(k_pool), _ptr(v_pool),
                                        _ptr(k_scale), _ptr(v_scale), _ptr(block_tables),
                                        block_tables.shape[1], _ptr(seq_lens), B, Q, _ptr(out))
    return out, st


# ---- several new tokens, a different number per request (varlen) ---------------
#
# Packed new tokens: cu_q [batch + 1], request b's tokens are rows
# cu_q[b] .. cu_q[b+1] - 1, token i at position L_b + i - cu_q[b].  By
# definition this is, request by request, the several-new-tokens case with
# that request's own count, so the oracle is that composition ("Scaling
# TensorRT-LLM: Kernel Fusion and Inflight Batching in Production", section
# "What the Scheduler Actually Does": prefill chunks and decode tokens in one
# batch).

def rope_append_varlen(cfg: OracleConfig, q, k_new, v_new, k_pool, v_pool, k_scale, v_scale,
                       block_tables, seq_lens, cu_q) -> int:
    """In place, for q [n_tokens, Hq, d] and k_new / v_new [n_tokens, Hkv, d];
    returns the OR of the per-request statuses."""
    st = 0
    for b in range(len(seq_lens)):
        a, e = int(cu_q[b]), int(cu_q[b + 1])
        if e <= a:
            continue
        qb = np.ascontiguousarray(q[a:e][None])
        st |= rope_append_tokens(cfg, qb, np.ascontiguousarray(k_new[a:e][None]),
                                 np.ascontiguousarray(v_new[a:e][None]), k_pool, v_pool, k_scale, v_scale,
                                 np.ascontiguousarray(block_tables[b:b + 1]),
                                 np.ascontiguousarray(seq_lens[b:b + 1]))
        q[a:e] = qb[0]
    return st


def decode_attn_varlen(cfg: OracleConfig, q, k_pool, v_pool, k_scale, v_scale, block_tables, seq_lens,
                       cu_q):
    """fp64 output [n_tokens, Hq, d]; (out, OR of the per-request statuses)."""
    out = np.zeros((q.shape[0], cfg.num_q_heads, cfg.head_dim), np.float64)
    st = 0
    for b in range(len(seq_lens)):
        a, e = int(cu_q[b]), int(cu_q[b + 1])
        if e <= a:
            continue
        o, s = decode_attn_tokens(cfg, np.ascontiguousarray(q[a:e][None]), k_pool, v_pool, k_scale, v_scale,
                                  np.ascontiguousarray(block_tables[b:b + 1]),
                                  np.ascontiguousarray(seq_lens[b:b + 1]))
        out[a:e] = o[0]
        st |= s
    return out, st


# ---- the QKV projection -------------------------------------------------------

def project_bf16(x, w):
    """bf16 bits: x [T, hidden], w [N, hidden] -> out [T, N] = bf16_RNE(x w^T),
    the dot products in fp64."""
    _need(x, np.uint16, "x"); _need(w, np.uint16, "w")
    T, H = x.shape
    N = w.shape[0]
    assert w.shape[1] == H
    out = np.zeros((T, N), np.uint16)
    st = _load().orc_project_bf16(_ptr(x), _ptr(w), T, N, H, _ptr(out))
    assert st == ORC_OK
    return out
