"""Seeded synthetic workloads for one in-flight-batched decode step.

This module only draws inputs.  It holds none of the step's arithmetic (no
RoPE, no attention, no append); both the GPU path and the CPU oracle take
their inputs from here and from nowhere else.

Shapes follow the pages' workload descriptions: requests of different
lengths in one batch ("Scaling TensorRT-LLM: Kernel Fusion and Inflight
Batching in Production", section "Static vs. Dynamic vs. Inflight"), KV in
fixed-size pages of 16/32/64 tokens named by a per-request block table
(same page, section "The Paged KV-Cache"; "TensorRT-LLM Guide:
High-Throughput GPU Inference Engine", section "2. Paged KV Cache & Memory
Virtualization").

Recipe (all seeded):
  * lengths L_b (tokens cached before the step) per configuration, drawn
    with numpy ``default_rng(seed)``;
  * each request owns ceil((L_b + q_len) / P) pages, the last ones holding
    the slots the q_len new tokens land in (q_len = 1 for the five decode
    configurations, 4 for the speculative-verification one); physical page
    ids are the first
    sum(pages) entries of a seeded permutation of the pool, handed out in
    logical order; the pool has 10% free pages (64 pages for ``tiny``);
  * block-table entries past a request's pages are -1;
  * resident K/V values ~ N(0, 1) rounded to bf16, drawn with a seeded
    ``torch.Generator`` on the target device; q, k_new, v_new the same;
  * every slot that holds no token (the landing slot, the rest of the last
    page, every free page) holds a NaN sentinel (bf16 0x7FC0, E4M3 0x7F), so
    a stray read poisons the output;
  * fp8 pools: for every allocated page and kv head a full P x d block of
    N(0, 1) values is drawn, its scale is amax/448 in fp32, the block is cast
    by torch to float8_e4m3fn after division by the scale (clamped to +-448
    first), and the resident slots keep the first rows.  Free pages get
    scale 1.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional

import numpy as np
import torch

BF16_NAN_BITS = 0x7FC0
E4M3_NAN_CODE = 0x7F

SEED_BASE = 20260000

# name -> (index, heads, head_dim, page, kv dtype, rope base)
_SHAPES = {
    "tiny":      dict(index=0, Hq=8,  Hkv=2, d=64,  P=16, kv_fp8=False, base=1e4),
    "llama8b":   dict(index=1, Hq=32, Hkv=8, d=128, P=32, kv_fp8=False, base=5e5),
    "hetero70b": dict(index=2, Hq=64, Hkv=8, d=128, P=16, kv_fp8=False, base=5e5),
    "longctx":   dict(index=3, Hq=32, Hkv=8, d=128, P=64, kv_fp8=False, base=5e5),
    "fp8":       dict(index=4, Hq=32, Hkv=8, d=128, P=32, kv_fp8=True,  base=5e5),
    # several new tokens per request (speculative-decode verification)
    "spec4":     dict(index=5, Hq=32, Hkv=8, d=128, P=32, kv_fp8=False, base=5e5, q_len=4),
}
# the five single-token decode configurations, and the multi-token one
CONFIG_NAMES = ("tiny", "llama8b", "hetero70b", "longctx", "fp8")
TOKEN_CONFIG_NAMES = ("spec4",)

DESCRIPTIONS = {
    "tiny": "4 requests, cached lengths {17,64,100,255}, Hq 8 / Hkv 2, d 64, page 16, "
            "64-page pool, bf16 KV N(0,1), RoPE base 1e4",
    "llama8b": "Llama-3-8B-shaped layer: batch 64, cached lengths U[128,4096], Hq 32 / Hkv 8, "
               "d 128, page 32, bf16 KV N(0,1), RoPE base 5e5, pool +10%",
    "hetero70b": "70B-shaped heterogeneous in-flight batch: batch 256, Hq 64 / Hkv 8, d 128, "
                 "page 16, bf16; lengths prompt{64,128,512,2048}+U[0,500], 20% refilled at 64",
    "longctx": "long-context split-KV: batch 8, cached lengths U[32768,131072], Hq 32 / Hkv 8, "
               "d 128, page 64, bf16 KV N(0,1), RoPE base 5e5",
    "fp8": "fp8 KV: batch 128, lengths log-normal(median 1024, sigma 1) clipped [16,16384], "
           "Hq 32 / Hkv 8, d 128, page 32, E4M3 KV with per-(page, kv head) scale amax/448",
    "spec4": "speculative-decode verification on the Llama-3-8B-shaped layer: batch 64, cached "
             "lengths U[128,4096], 4 new tokens per request (positions L..L+3, causal among "
             "them), Hq 32 / Hkv 8, d 128, page 32, bf16 KV N(0,1), RoPE base 5e5, pool +10%",
}


def config_seed(name: str, offset: int = 0) -> int:
    return SEED_BASE + _SHAPES[name]["index"] + 1000 * offset


def draw_lengths(name: str, rng: np.random.Generator) -> np.ndarray:
    """Cached lengths L_b (before the step) for a named configuration."""
    if name == "tiny":
        return np.array([17, 64, 100, 255], np.int64)
    if name in ("llama8b", "spec4"):
        return rng.integers(128, 4096, size=64, endpoint=True)
    if name == "hetero70b":
        B = 256
        prompt = rng.choice(np.array([64, 128, 512, 2048]), size=B)
        progress = rng.integers(0, 500, size=B, endpoint=True)
        L = prompt + progress
        refilled = rng.permutation(B)[: int(round(0.2 * B))]
        L[refilled] = 64
        return L
    if name == "longctx":
        return rng.integers(32768, 131072, size=8, endpoint=True)
    if name == "fp8":
        z = rng.standard_normal(128)
        return np.clip(np.round(np.exp(math.log(1024.0) + 1.0 * z)), 16, 16384).astype(np.int64)
    raise KeyError(name)


@dataclass
class Workload:
    name: str
    Hq: int
    Hkv: int
    d: int
    P: int
    kv_fp8: bool
    rope_base: float
    seq_lens: np.ndarray          # [B] int32, L_b before the step
    block_tables: np.ndarray      # [B, bt_stride] int32, -1 past the used pages
    num_pages: int
    q: torch.Tensor               # [B, Hq, d] bf16; [B, q_len, Hq, d] when q_len > 1
    k_new: torch.Tensor           # [B, Hkv, d] bf16; [B, q_len, Hkv, d] when q_len > 1
    v_new: torch.Tensor           # as k_new
    k_pool: torch.Tensor          # [num_pages, Hkv, P, d] bf16 or uint8 (E4M3 codes)
    v_pool: torch.Tensor
    k_scale: Optional[torch.Tensor] = None   # [num_pages, Hkv] fp32 (fp8 only)
    v_scale: Optional[torch.Tensor] = None
    seed: int = 0
    q_len: int = 1                # new tokens per request (positions L_b .. L_b + q_len - 1)
    extra: dict = field(default_factory=dict)

    @property
    def batch(self) -> int:
        return int(self.seq_lens.shape[0])

    @property
    def bt_stride(self) -> int:
        return int(self.block_tables.shape[1])

    @property
    def kv_bytes_per_elem(self) -> int:
        return 1 if self.kv_fp8 else 2


def _assign_pages(lengths: np.ndarray, P: int, num_pages: Optional[int],
                  rng: np.random.Generator, q_len: int = 1):
    pages_needed = (lengths + q_len + P - 1) // P      # includes the landing page(s)
    total = int(pages_needed.sum())
    if num_pages is None:
        num_pages = int(math.ceil(1.1 * total))
    if total > num_pages:
        raise ValueError("pool too small for the requested lengths")
    perm = rng.permutation(num_pages).astype(np.int32)
    bt_stride = max(1, int(pages_needed.max()))
    bt = np.full((lengths.shape[0], bt_stride), -1, np.int32)
    pos = 0
    for b, n in enumerate(pages_needed):
        bt[b, :n] = perm[pos:pos + n]
        pos += n
    return bt, num_pages


def _resident_mask(lengths: np.ndarray, bt: np.ndarray, num_pages: int, P: int) -> np.ndarray:
    """[num_pages, P] bool: True where a slot holds a resident (pre-step) token."""
    mask = np.zeros((num_pages, P), bool)
    for b, L in enumerate(lengths):
        for lp in range(int((L + P - 1) // P)):
            page = bt[b, lp]
            lo = lp * P
            n_here = int(min(P, max(0, L - lo)))
            mask[page, :n_here] = True
    return mask


def build(name: str, Hq: int, Hkv: int, d: int, P: int, kv_fp8: bool, rope_base: float,
          lengths, seed: int, device="cpu", num_pages: Optional[int] = None,
          bt_stride: Optional[int] = None, q_len: int = 1) -> Workload:
    """Draw one workload with the given shapes and cached lengths; q_len new
    tokens per request (q_len > 1 gives q, k_new, v_new a token axis)."""
    lengths = np.asarray(lengths, np.int64)
    rng = np.random.default_rng(seed + 7)   # page permutation stream
    bt, num_pages = _assign_pages(lengths, P, num_pages, rng, q_len)
    if bt_stride is not None and bt_stride > bt.shape[1]:
        bt = np.concatenate([bt, np.full((bt.shape[0], bt_stride - bt.shape[1]), -1, np.int32)], 1)
    B = lengths.shape[0]
    dev = torch.device(device)
    gen = torch.Generator(device=dev)
    gen.manual_seed(seed)
    mask = torch.from_numpy(_resident_mask(lengths, bt, num_pages, P)).to(dev)
    slot_mask = mask[:, None, :, None]                          # [pages, 1, P, 1]

    def randn(*shape):
        return torch.randn(*shape, generator=gen, device=dev, dtype=torch.float32)

    k_scale = v_scale = None
    if not kv_fp8:
        nan = torch.tensor(BF16_NAN_BITS, dtype=torch.int16, device=dev).view(torch.bfloat16)
        pools = []
        for _ in range(2):
            vals = randn(num_pages, Hkv, P, d).to(torch.bfloat16)
            pools.append(torch.where(slot_mask, vals, nan))
            del vals
        k_pool, v_pool = pools
    else:
        allocated = torch.zeros(num_pages, dtype=torch.bool, device=dev)
        used = torch.from_numpy(bt[bt >= 0].astype(np.int64)).to(dev)
        allocated[used] = True
        pools, scales = [], []
        for _ in range(2):
            block = randn(num_pages, Hkv, P, d)
            amax = block.abs().amax(dim=(2, 3))                     # [pages, Hkv] fp32
            scale = torch.where(allocated[:, None], amax / 448.0, torch.ones_like(amax))
            scaled = (block / scale[:, :, None, None]).clamp_(-448.0, 448.0)
            codes = scaled.to(torch.float8_e4m3fn).view(torch.uint8)
            nan_code = torch.tensor(E4M3_NAN_CODE, dtype=torch.uint8, device=dev)
            pools.append(torch.where(slot_mask, codes, nan_code))
            scales.append(scale.contiguous())
            del block, scaled, codes
        k_pool, v_pool = pools
        k_scale, v_scale = scales

    tok = () if q_len == 1 else (q_len,)
    q = randn(B, *tok, Hq, d).to(torch.bfloat16)
    k_new = randn(B, *tok, Hkv, d).to(torch.bfloat16)
    v_new = randn(B, *tok, Hkv, d).to(torch.bfloat16)
    return Workload(name=name, Hq=Hq, Hkv=Hkv, d=d, P=P, kv_fp8=kv_fp8, rope_base=rope_base,
                    seq_lens=lengths.astype(np.int32), block_tables=bt, num_pages=num_pages,
                    q=q, k_new=k_new, v_new=v_new, k_pool=k_pool.contiguous(),
                    v_pool=v_pool.contiguous(), k_scale=k_scale, v_scale=v_scale, seed=seed,
                    q_len=q_len)


def make(name: str, device="cpu", offset: int = 0, requests: Optional[int] = None) -> Workload:
    """One of the five named workloads; ``offset`` draws an independent replica.
    ``requests`` keeps only the first that many requests of the batch (same
    shapes and lengths, a pool sized for them): a smaller case of the same
    workload, for profiler captures."""
    s = _SHAPES[name]
    seed = config_seed(name, offset)
    lengths = draw_lengths(name, np.random.default_rng(seed))
    if requests is not None:
        lengths = lengths[:max(1, int(requests))]
    w = build(name, s["Hq"], s["Hkv"], s["d"], s["P"], s["kv_fp8"], s["base"], lengths,
              seed, device=device, num_pages=64 if name == "tiny" else None, q_len=s.get("q_len", 1))
    if requests is not None:
        w.extra["requests"] = w.batch
    return w


def make_mixed(device="cpu", offset: int = 0, chunk: int = 64, prefills: int = 8):
    """Chunked prefill mixed with decode on the llama8b batch: the llama8b
    lengths and shapes, `prefills` seeded requests take a chunk of `chunk` new
    tokens, the others one.  Returns (workload with a token axis of `chunk`,
    new tokens per request); the varlen step uses the first q_lens[b] tokens
    of request b."""
    s = _SHAPES["llama8b"]
    seed = config_seed("llama8b", offset) + 31
    rng = np.random.default_rng(seed)
    lengths = draw_lengths("llama8b", np.random.default_rng(config_seed("llama8b", offset)))
    q_lens = np.ones(len(lengths), np.int64)
    q_lens[rng.choice(len(lengths), size=prefills, replace=False)] = chunk
    w = build("mixed", s["Hq"], s["Hkv"], s["d"], s["P"], s["kv_fp8"], s["base"], lengths, seed, device=device,
              q_len=chunk)
    return w, q_lens


def shape_of(name: str) -> dict:
    return dict(_SHAPES[name])
