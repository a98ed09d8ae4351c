"""GPU-test helpers: run the step through the C ABI and build the oracle's
view of sampled requests from the generator's ORIGINAL inputs (never from
anything the GPU path wrote)."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from paged_kv_flight_b200.workloads import Workload
from tests._util import bits16, bytes8

# attention-output tolerances (abs) for bf16 KV and for E4M3 KV
TOL_BF16 = dict(max=1e-2, mean=1e-3)
TOL_FP8 = dict(max=6e-2, mean=6e-3)


def tol(w: Workload):
    return TOL_FP8 if w.kv_fp8 else TOL_BF16


def to_device(w: Workload, device="cuda"):
    """Device copies of every step input (the generator may draw on the CPU).
    Always copies, also when the workload already lives on the device, so the
    step never writes into the generator's original tensors."""
    def cp(t):
        return None if t is None else t.to(device, copy=True).contiguous()
    d = dict(q=cp(w.q), k_new=cp(w.k_new), v_new=cp(w.v_new), k_pool=cp(w.k_pool), v_pool=cp(w.v_pool),
             k_scale=cp(w.k_scale), v_scale=cp(w.v_scale),
             block_tables=torch.from_numpy(w.block_tables).to(device).contiguous(),
             seq_lens=torch.from_numpy(w.seq_lens).to(device).contiguous())
    return d


def make_ctx(pkv, w: Workload, max_batch=None, max_blocks=None):
    cfg = pkv.make_config(w.Hq, w.Hkv, w.d, w.P, "fp8" if w.kv_fp8 else "bf16", w.rope_base,
                          max_batch or w.batch, max_blocks or w.bt_stride, w.num_pages)
    return pkv.pkv_create(cfg)


def gpu_step(pkv, ctx, dv: dict, out=None, check=True, fused=False):
    """The step through the C ABI: pkv_rope_append then pkv_decode_attn, or
    with fused=True the one call pkv_decode_step."""
    B = dv["seq_lens"].shape[0]
    Hq, d = dv["q"].shape[1], dv["q"].shape[2]
    if out is None:
        out = torch.empty(B, Hq, d, dtype=torch.bfloat16, device=dv["q"].device)
    if fused:
        pkv.pkv_decode_step(ctx, dv["q"], dv["k_new"], dv["v_new"], dv["k_pool"], dv["v_pool"], dv["k_scale"],
                            dv["v_scale"], dv["block_tables"], dv["seq_lens"], out, check=check)
        return out
    pkv.pkv_rope_append(ctx, dv["q"], dv["k_new"], dv["v_new"], dv["k_pool"], dv["v_pool"],
                        dv["k_scale"], dv["v_scale"], dv["block_tables"], dv["seq_lens"], check=check)
    pkv.pkv_decode_attn(ctx, dv["q"], dv["k_pool"], dv["v_pool"], dv["k_scale"], dv["v_scale"],
                        dv["block_tables"], dv["seq_lens"], out, check=check)
    return out


def request_view(w: Workload, b: int, dev_orig: dict | None = None):
    """Oracle inputs for request b alone: its pages copied out of the original
    pools into a private pool, block table renumbered 0..n-1."""
    L = int(w.seq_lens[b])
    npg = (L + w.q_len + w.P - 1) // w.P          # pages up to the last new token
    pages = w.block_tables[b, :npg].astype(np.int64)
    src = dev_orig if dev_orig is not None else dict(k_pool=w.k_pool, v_pool=w.v_pool, k_scale=w.k_scale,
                                                     v_scale=w.v_scale, q=w.q, k_new=w.k_new, v_new=w.v_new)
    idx = torch.from_numpy(pages).to(src["k_pool"].device)
    conv = bytes8 if w.kv_fp8 else bits16
    h = dict(
        q=bits16(src["q"][b:b + 1]), k_new=bits16(src["k_new"][b:b + 1]), v_new=bits16(src["v_new"][b:b + 1]),
        k_pool=conv(src["k_pool"].index_select(0, idx)), v_pool=conv(src["v_pool"].index_select(0, idx)),
        k_scale=None if w.k_scale is None else src["k_scale"].index_select(0, idx).cpu().numpy().copy(),
        v_scale=None if w.v_scale is None else src["v_scale"].index_select(0, idx).cpu().numpy().copy(),
        block_tables=np.arange(npg, dtype=np.int32)[None, :].copy(),
        seq_lens=np.array([L], np.int32),
    )
    cfg = oracle.OracleConfig(w.Hq, w.Hkv, w.d, w.P, w.kv_fp8, npg, w.rope_base)
    return cfg, h


def oracle_request(w: Workload, b: int, dev_orig: dict | None = None, kvh_list=None):
    """Oracle append + attention for request b; returns (h after append, out [Hq, d] fp64)."""
    cfg, h = request_view(w, b, dev_orig)
    st = oracle.rope_append(cfg, h["q"], h["k_new"], h["v_new"], h["k_pool"], h["v_pool"], h["k_scale"],
                            h["v_scale"], h["block_tables"], h["seq_lens"])
    assert st == 0
    G = w.Hq // w.Hkv
    out = np.full((w.Hq, w.d), np.nan)
    for kvh in (range(w.Hkv) if kvh_list is None else kvh_list):
        o, st = oracle.decode_attn_group(cfg, h["q"], h["k_pool"], h["v_pool"], h["k_scale"], h["v_scale"],
                                         h["block_tables"], h["seq_lens"], 0, kvh)
        assert st == 0
        out[kvh * G:(kvh + 1) * G] = o
    return h, out


def errors(gpu_out: torch.Tensor, ref: np.ndarray):
    g = gpu_out.float().cpu().numpy().astype(np.float64)
    m = ~np.isnan(ref)
    diff = np.abs(g[m] - ref[m])
    return float(diff.max()), float(diff.mean()), bool(np.isfinite(g).all())
