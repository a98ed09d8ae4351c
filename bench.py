#!/usr/bin/env python
"""Benchmark: one in-flight-batched decode step over a paged KV cache
(RoPE + append, then split-KV GQA decode attention), through the libpkv C ABI.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME|suite|all]
                    [--impl ours|reference]

By default every graded workload is measured in turn (llama8b, hetero70b,
fp8, spec4, then longctx), one JSON line each; the last line printed is the
long-context workload's, the largest.  One step = pkv_decode_step (RoPE +
append, then the attention as a programmatic dependent of the append kernel,
then the split combine) over the whole batch of the workload.  Inputs are resident in HBM; before every timed step, outside the
CUDA-event window, a 2x-L2 buffer is written and another 2x-L2 buffer read,
so the step finds none of its inputs in L2 and no dirty lines to write back.  The value is
whole-job HBM throughput: resident KV bytes attended plus q / out bytes, per
step, summed over ranks, divided by the max-over-ranks median step time.  Under
torchrun every rank runs an independent replica of the workload (weak
scaling; the step has no exchange between GPUs).

``--impl reference`` times the CPU oracle (plain fp64 C, one thread) on a
bounded sample of the same workload instead.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import re
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "paged-KV decode attn: HBM GB/s (% of B200 peak), request-tokens/s, step µs"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
# the default run: every graded workload, the largest (longctx) last so that
# the last line printed is the long-context one
SUITE = ("llama8b", "hetero70b", "fp8", "spec4", "longctx")
DEFAULT_CONFIG = "suite"
# sources of the kernel whose DRAM traffic a profile line records: the
# attention kernels for the attention workloads, the fused projection for qkv8b
KERNEL_SOURCES = {
    "attn": ("paged_kv_flight_b200/csrc/decode_attn.cu", "paged_kv_flight_b200/csrc/decode_attn_tokens.cu",
             "paged_kv_flight_b200/csrc/attn_common.cuh", "paged_kv_flight_b200/csrc/combine.cu",
             "paged_kv_flight_b200/csrc/pkv_device.cuh", "paged_kv_flight_b200/csrc/pkv_internal.h"),
    "qkv": ("paged_kv_flight_b200/csrc/qkv_rope_append.cu", "paged_kv_flight_b200/csrc/pkv_device.cuh",
            "paged_kv_flight_b200/csrc/umma.cuh", "paged_kv_flight_b200/csrc/pkv_internal.h"),
}
# the mixed leg's attention: the several-new-tokens kernels, the combine and
# the prefill blocks on tcgen05 (its traffic line is the three kernels' sum)
KERNEL_SOURCES["mixed"] = KERNEL_SOURCES["attn"] + ("paged_kv_flight_b200/csrc/chunk_attn.cu",
                                                    "paged_kv_flight_b200/csrc/umma.cuh")


# ---------------------------------------------------------------- accounting

def metric_bytes(seq_lens, Hq, Hkv, d, P, kv_fp8, q_len=1) -> int:
    """Resident KV attended (the new tokens included, read once per request
    and kv head) + q read + out written (+ the two fp32 scales per attended
    page and kv head for E4M3 pools)."""
    n = np.asarray(seq_lens, np.int64) + q_len
    s = 1 if kv_fp8 else 2
    kv = int((2 * Hkv * n * d * s).sum())
    qo = 2 * len(n) * q_len * Hq * d * 2
    sc = int(2 * ((n + P - 1) // P).sum() * Hkv * 4) if kv_fp8 else 0
    return kv + qo + sc


def workload_bytes(w) -> int:
    return metric_bytes(w.seq_lens, w.Hq, w.Hkv, w.d, w.P, w.kv_fp8, w.q_len)


def full_step_bytes(seq_lens, Hq, Hkv, d, P, kv_fp8, q_len=1) -> int:
    """The step's whole algorithmic traffic: the metric bytes plus what the
    RoPE + append kernel moves (q read and written back, k_new / v_new read,
    the new k / v rows written, the landing pages' scales for E4M3 pools) and
    the index reads of both kernels (block-table entries of the attended
    pages, seq_lens, the landing pages' entries).  The split partials are left
    out: how many there are is planned on the device each step."""
    n = np.asarray(seq_lens, np.int64) + q_len
    B = len(n)
    s = 1 if kv_fp8 else 2
    rope = B * q_len * (2 * Hq * d * 2 + 2 * Hkv * d * 2 + 2 * Hkv * d * s + 4)
    if kv_fp8:
        rope += B * q_len * 2 * Hkv * 4
    index = int(((n + P - 1) // P).sum()) * 4 + 2 * B * 4
    return metric_bytes(seq_lens, Hq, Hkv, d, P, kv_fp8, q_len) + rope + index


def host_cpu() -> dict:
    """The host's CPU model and hardware thread count, for the CPU baselines."""
    model = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    model = ln.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"cpu_model": model, "host_threads": os.cpu_count()}


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            v = float(json.load(f)["hbm_gbs"])
        return v, "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def source_sha(kernel: str = "attn") -> str:
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str):
    """DRAM bytes per launch of the workload's dominant kernel from a
    committed ncu summary, if it was taken on that kernel's current sources;
    otherwise None."""
    sha = source_sha({"qkv8b": "qkv", "mixed": "mixed"}.get(workload, "attn"))
    pat = re.compile(r"traffic-per-launch:\s+(\S+)\s+(\d+)\s+src=([0-9a-f]+)")
    pdir = os.path.join(ROOT, "profiles")
    if not os.path.isdir(pdir):
        return None
    for fn in sorted(os.listdir(pdir)):
        if not fn.endswith((".md", ".txt")):
            continue
        with open(os.path.join(pdir, fn)) as f:
            for m in pat.finditer(f.read()):
                if m.group(1) == workload and m.group(3) == sha:
                    return int(m.group(2))
    return None


# ---------------------------------------------------------------- ranks

def dist_info():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def max_over_ranks(x: float) -> float:
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return x
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float) -> float:
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return x
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


# ---------------------------------------------------------------- clocks

_REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
            0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
            0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}


class ClockSampler:
    """Polls the SM clock and the clock-event (throttle) reasons of this
    process's GPU through NVML while the timed region runs."""

    def __init__(self, device_index: int, period_s: float = 0.01):
        self.period = period_s
        self.samples, self.reason_bits = [], 0
        self.err = None
        self.h = None
        try:
            import pynvml
            import torch
            self.nv = pynvml
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            for cand in (uuid, "GPU-" + uuid):
                try:
                    self.h = pynvml.nvmlDeviceGetHandleByUUID(cand)
                    break
                except Exception:
                    continue
            if self.h is None:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # no NVML: report that, keep running
            self.err = f"{type(e).__name__}: {e}"
        self._stop = threading.Event()
        self._t = None

    def _reasons(self):
        f = getattr(self.nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            self.nv.nvmlDeviceGetCurrentClocksThrottleReasons
        return int(f(self.h))

    def sample(self):
        if self.h is None:
            return
        try:
            self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
            self.reason_bits |= self._reasons()
        except Exception as e:
            self.err = f"{type(e).__name__}: {e}"

    def _run(self):
        while not self._stop.is_set():
            self.sample()
            time.sleep(self.period)

    def start(self):
        self._t = threading.Thread(target=self._run, daemon=True)
        self._t.start()

    def stop(self) -> dict:
        self._stop.set()
        if self._t:
            self._t.join()
        out = {"sm_mhz": statistics.median(self.samples) if self.samples else None,
               "sm_max_mhz": getattr(self, "max_mhz", None),
               "reasons": [n for b, n in _REASONS.items() if self.reason_bits & b and b != 0x1],
               "samples": len(self.samples), "source": "nvml, polled every 10 ms during the timed steps"}
        if self.err:
            out["error"] = self.err
        return out


# ---------------------------------------------------------------- oracle leg

def _request_pages(w, b, src, cached=None):
    """Host copies (oracle form) of request b's pages, block table renumbered;
    with `cached`, the request cut to its first `cached` cached tokens (the new
    tokens then land right after them)."""
    import torch
    L = int(w.seq_lens[b]) if cached is None else min(int(cached), int(w.seq_lens[b]))
    npg = (L + w.q_len + w.P - 1) // w.P
    idx = torch.from_numpy(w.block_tables[b, :npg].astype(np.int64)).to(src["k_pool"].device)

    def b16(t):
        return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16).copy()

    def u8(t):
        return t.contiguous().cpu().numpy().copy()

    conv = u8 if w.kv_fp8 else b16
    return dict(
        npg=npg,
        q=b16(src["q"][b:b + 1]), k_new=b16(src["k_new"][b:b + 1]), v_new=b16(src["v_new"][b:b + 1]),
        k_pool=conv(src["k_pool"].index_select(0, idx)), v_pool=conv(src["v_pool"].index_select(0, idx)),
        k_scale=None if src["k_scale"] is None else src["k_scale"].index_select(0, idx).cpu().numpy().copy(),
        v_scale=None if src["v_scale"] is None else src["v_scale"].index_select(0, idx).cpu().numpy().copy(),
        block_tables=np.arange(npg, dtype=np.int32)[None, :].copy(),
        seq_lens=np.array([L], np.int32))


def oracle_step_requests(w, views):
    """The oracle's whole step (append + attention) for the given requests."""
    import oracle
    for v in views:
        cfg = oracle.OracleConfig(w.Hq, w.Hkv, w.d, w.P, w.kv_fp8, v["npg"], w.rope_base)
        q = v["q"].copy()
        kp, vp = v["k_pool"].copy(), v["v_pool"].copy()
        if w.q_len > 1:
            oracle.rope_append_tokens(cfg, q, v["k_new"], v["v_new"], kp, vp, v["k_scale"], v["v_scale"],
                                      v["block_tables"], v["seq_lens"])
            oracle.decode_attn_tokens(cfg, q, kp, vp, v["k_scale"], v["v_scale"], v["block_tables"],
                                      v["seq_lens"])
        else:
            oracle.rope_append(cfg, q, v["k_new"], v["v_new"], kp, vp, v["k_scale"], v["v_scale"],
                               v["block_tables"], v["seq_lens"])
            oracle.decode_attn(cfg, q, kp, vp, v["k_scale"], v["v_scale"], v["block_tables"], v["seq_lens"])


def sample_requests(w, token_head_budget: int):
    """Prefix of the batch whose attended token-heads stay within the budget
    (at least one request)."""
    picks, acc = [], 0
    for b, L in enumerate(w.seq_lens):
        th = (int(L) + w.q_len) * w.Hkv
        if picks and acc + th > token_head_budget:
            break
        picks.append(b)
        acc += th
    return picks


def cpu_baseline(w, src, time_budget_s: float = 20.0) -> dict:
    """Times the oracle as it stands on this host (one thread), request by
    request in batch order until the time budget is spent."""
    views, t_sum, done = [], 0.0, []
    for b in range(w.batch):
        v = _request_pages(w, b, src)
        t0 = time.perf_counter()
        oracle_step_requests(w, [v])
        t_sum += time.perf_counter() - t0
        done.append(b)
        if t_sum >= time_budget_s:
            break
    by = metric_bytes(w.seq_lens[done], w.Hq, w.Hkv, w.d, w.P, w.kv_fp8, w.q_len)
    toks = int((w.seq_lens[done].astype(np.int64) + w.q_len).sum())
    return {"value": by / t_sum / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle",
            "seconds": t_sum, **host_cpu(),
            "sample": f"requests 0..{len(done) - 1} of {w.batch} ({toks} attended tokens, "
                      f"{100.0 * by / workload_bytes(w):.1f}% of the step's bytes); plain fp64 C oracle, "
                      f"single thread, append + attention"}


# ---------------------------------------------------------------- config

L2_NOTE = "flushed before every timed step, outside the event window: write 2x L2, then read 2x L2"


def workload_config(w, name, world) -> dict:
    """The `config` object of a line: the workload alone, identical for the
    GPU arm and the reference (oracle) arm."""
    from paged_kv_flight_b200 import workloads
    return {"workload": name, "description": workloads.DESCRIPTIONS[name], "batch": w.batch,
            "tokens_attended": int((w.seq_lens.astype(np.int64) + w.q_len).sum()),
            "new_tokens_per_request": w.q_len,
            "metric_bytes_per_step": workload_bytes(w),
            "full_step_bytes": full_step_bytes(w.seq_lens, w.Hq, w.Hkv, w.d, w.P, w.kv_fp8, w.q_len),
            "l2": L2_NOTE, "replicas": world,
            **({"requests_kept": w.batch} if w.extra.get("requests") else {})}


# ---------------------------------------------------------------- GPU leg

def _device_inputs(w, device):
    import torch
    return dict(q=w.q.to(device).contiguous(), k_new=w.k_new.to(device).contiguous(),
                v_new=w.v_new.to(device).contiguous(), k_pool=w.k_pool.to(device).contiguous(),
                v_pool=w.v_pool.to(device).contiguous(),
                k_scale=None if w.k_scale is None else w.k_scale.to(device).contiguous(),
                v_scale=None if w.v_scale is None else w.v_scale.to(device).contiguous(),
                block_tables=torch.from_numpy(w.block_tables).to(device).contiguous(),
                seq_lens=torch.from_numpy(w.seq_lens).to(device).contiguous())


def run_ours(args, name, rank, world, local_rank, cpu_budget=None):
    import torch
    from paged_kv_flight_b200 import pkv, workloads

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w = workloads.make(name, device=dev, offset=rank, requests=args.requests)
    dv = _device_inputs(w, dev)
    B = w.batch
    cfg = pkv.make_config(w.Hq, w.Hkv, w.d, w.P, "fp8" if w.kv_fp8 else "bf16", w.rope_base, B,
                          w.bt_stride, w.num_pages)
    ctx = pkv.pkv_create(cfg)
    if args.tail_chunks is not None:
        pkv.pkv_set_tail_chunks(ctx, args.tail_chunks)
    tok = w.q_len > 1          # several new tokens per request: the *_tokens entry points
    out = torch.empty(B, *((w.q_len,) if tok else ()), w.Hq, w.d, dtype=torch.bfloat16, device=dev)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size

    def rope_call(x, stream=None):
        fn = pkv.pkv_rope_append_tokens if tok else pkv.pkv_rope_append
        fn(ctx, x["q"], x["k_new"], x["v_new"], dv["k_pool"], dv["v_pool"], dv["k_scale"], dv["v_scale"],
           x["block_tables"], x["seq_lens"], stream=stream)

    def attn_call(x, o, stream=None):
        fn = pkv.pkv_decode_attn_tokens if tok else pkv.pkv_decode_attn
        fn(ctx, x["q"], dv["k_pool"], dv["v_pool"], dv["k_scale"], dv["v_scale"], x["block_tables"],
           x["seq_lens"], o, stream=stream)
    flush_w = torch.empty(2 * l2, dtype=torch.uint8, device=dev)
    flush_r = torch.ones(2 * l2 // 8, dtype=torch.int64, device=dev)
    flush_sink = torch.empty((), dtype=torch.int64, device=dev)

    class _Flush:
        """Writes a buffer of 2x L2, then reads another of 2x L2, so that the
        step starts with an L2 that holds none of its inputs and no dirty
        lines whose write-back would land inside the timed window."""

        @staticmethod
        def zero_():
            flush_w.zero_()
            torch.sum(flush_r, dim=0, out=flush_sink)

    flush = _Flush()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, dv, args.cpu_budget if cpu_budget is None else cpu_budget)

    def step(x=dv, o=out, stream=None):
        """One step: pkv_decode_step (the attention a programmatic dependent
        of the append kernel), or with --two-calls the two calls."""
        if args.two_calls:
            rope_call(x, stream=stream)
            attn_call(x, o, stream=stream)
        else:
            pkv.pkv_decode_step(ctx, x["q"], x["k_new"], x["v_new"], dv["k_pool"], dv["v_pool"], dv["k_scale"],
                                dv["v_scale"], x["block_tables"], x["seq_lens"], o, q_len=w.q_len, stream=stream)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    st, bits = pkv.pkv_check_device_error(ctx)
    if st != pkv.PKV_OK:
        raise RuntimeError(f"device error during warm-up: {pkv.pkv_status_str(st)} bits={bits}")

    K = args.steps
    # the step captured once in a CUDA graph (three kernels, no host work),
    # replayed in the headline timing; the kernels inside are the same
    graph = None
    if not args.no_graph:
        side = torch.cuda.Stream(dev)
        with torch.cuda.stream(side):
            step()
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=side):
            step()
        for _ in range(args.warmup):
            flush.zero_()
            graph.replay()
        torch.cuda.synchronize()

    # timed region 1: eager steps through the C ABI, with events between the
    # two calls (rope_append; attention + combine) for the per-kernel times
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    clocks = ClockSampler(local_rank)
    barrier()
    torch.cuda.synchronize()
    clocks.start()
    for k in range(K):
        flush.zero_()                       # outside the event window
        ev[k][0].record()
        rope_call(dv)
        ev[k][1].record()
        attn_call(dv, out)
        ev[k][2].record()
    clocks.sample()
    torch.cuda.synchronize()
    barrier()

    # timed region 2: the same K steps replayed from the graph (L2 flushed
    # before each replay, outside the event window)
    graph_ms = None
    if graph is not None:
        gev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
        torch.cuda.synchronize()
        for k in range(K):
            flush.zero_()
            gev[k][0].record()
            graph.replay()
            gev[k][1].record()
        clocks.sample()
        torch.cuda.synchronize()
        barrier()
        graph_ms = [a.elapsed_time(b) for a, b in gev]
        del graph

    # timed region 3: the same K steps launched eagerly as one call each
    sev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    torch.cuda.synchronize()
    for k in range(K):
        flush.zero_()
        sev[k][0].record()
        step()
        sev[k][1].record()
    clocks.sample()
    torch.cuda.synchronize()
    barrier()
    step_call_ms = [a.elapsed_time(b) for a, b in sev]

    # the kernels' own time inside a replayed step: the two calls captured
    # in a graph with timing events recorded as graph nodes before the
    # append, between the calls and after the combine; each replay is read
    # back before the next (L2 flushed before each, outside the events)
    rope_g_ms, attn_g_ms = [], []
    if not args.no_graph:
        try:
            te = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(3)]
            side = torch.cuda.Stream(dev)
            torch.cuda.synchronize()
            tgraph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(tgraph, stream=side):
                te[0].record()
                rope_call(dv)
                te[1].record()
                attn_call(dv, out)
                te[2].record()
            for k in range(args.warmup + K):
                flush.zero_()
                tgraph.replay()
                torch.cuda.synchronize()
                if k >= args.warmup:
                    rope_g_ms.append(te[0].elapsed_time(te[1]))
                    attn_g_ms.append(te[1].elapsed_time(te[2]))
            del tgraph
        except RuntimeError as e:          # timing events inside graphs unavailable: eager figures only
            print(f"bench: in-graph kernel timing unavailable ({e})", file=sys.stderr)
            rope_g_ms, attn_g_ms = [], []
            torch.cuda.synchronize()
        clocks.sample()
        barrier()
    clock_info = clocks.stop()
    step_ms = [a.elapsed_time(c) for a, _, c in ev]
    rope_ms = [a.elapsed_time(b) for a, b, _ in ev]
    attn_ms = [b.elapsed_time(c) for _, b, c in ev]
    st, bits = pkv.pkv_check_device_error(ctx)
    if st != pkv.PKV_OK:
        raise RuntimeError(f"device error during timing: {pkv.pkv_status_str(st)} bits={bits}")

    med = statistics.median
    eager_max = max_over_ranks(med(step_ms))
    attn_max = max_over_ranks(med(attn_ms))
    step_max = max_over_ranks(med(graph_ms)) if graph_ms is not None else eager_max
    step_mean = max_over_ranks(sum(graph_ms if graph_ms is not None else step_ms) / K)
    # the attention's own time: inside the replayed graph when measured,
    # else the eager events (which include the launch gap)
    attn_graph_max = max_over_ranks(med(attn_g_ms)) if attn_g_ms else None
    rope_graph_max = max_over_ranks(med(rope_g_ms)) if rope_g_ms else None
    attn_for_roofline = attn_graph_max if attn_graph_max is not None else attn_max
    by = workload_bytes(w)
    total_bytes = sum_over_ranks(float(by))
    total_reqs = sum_over_ranks(float(B))

    # unflushed ("hot L2") median, labelled as such
    hot = []
    for _ in range(min(K, 50)):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        step()
        b.record()
        hot.append((a, b))
    torch.cuda.synchronize()
    hot_ms = statistics.median(x.elapsed_time(y) for x, y in hot)

    # end to end through the public API: every step copies its inputs (q, k_new,
    # v_new, block_tables, seq_lens, packed in one pinned host buffer) to the
    # device, runs the step through the C ABI and reads `out` back to pinned
    # host memory.  Copy-in, compute and copy-out run on three streams with
    # double-buffered device staging, so step k+1's upload and step k-1's
    # download overlap step k's kernels, as a serving loop would pipeline them.
    # The KV pools stay resident (the cache lives on the GPU); they are 4-20x
    # the L2, so this leg relies on "inputs larger than L2" instead of a flush.
    e2e = None
    if not args.no_e2e:
        keys = ("q", "k_new", "v_new", "block_tables", "seq_lens")
        sizes = [dv[k].numel() * dv[k].element_size() for k in keys]
        offs, off = [], 0
        for sz in sizes:
            offs.append(off)
            off += (sz + 255) // 256 * 256
        host_buf = torch.empty(off, dtype=torch.uint8).pin_memory()
        for k, o, sz in zip(keys, offs, sizes):
            host_buf[o:o + sz].copy_(dv[k].contiguous().view(torch.uint8).reshape(-1).cpu())
        dev_bufs = [torch.empty(off, dtype=torch.uint8, device=dev) for _ in range(2)]
        views = [{k: buf[o:o + sz].view(dv[k].dtype).view(dv[k].shape) for k, o, sz in zip(keys, offs, sizes)}
                 for buf in dev_bufs]
        outs = [torch.empty_like(out) for _ in range(2)]
        outs_h = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
        h2d = sum(sizes)
        d2h = outs_h[0].numel() * outs_h[0].element_size()
        s_in, s_comp, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_comp = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]

        def e2e_run(n):
            for i in range(n):
                sl = i % 2
                v = views[sl]
                if i >= 2:
                    s_in.wait_event(ev_comp[sl])          # staging slot free again
                with torch.cuda.stream(s_in):
                    dev_bufs[sl].copy_(host_buf, non_blocking=True)
                    ev_in[sl].record(s_in)
                s_comp.wait_event(ev_in[sl])
                if i >= 2:
                    s_comp.wait_event(ev_out[sl])         # output slot read back
                step(v, outs[sl], stream=s_comp)
                ev_comp[sl].record(s_comp)
                s_out.wait_event(ev_comp[sl])
                with torch.cuda.stream(s_out):
                    outs_h[sl].copy_(outs[sl], non_blocking=True)
                    ev_out[sl].record(s_out)

        e2e_run(args.warmup)
        torch.cuda.synchronize()
        barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(s_in)
        e2e_run(K)
        s_in.wait_event(ev_out[(K - 1) % 2])
        s_in.wait_event(ev_out[K % 2])
        b.record(s_in)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(a.elapsed_time(b) / K)
        e2e = {"value": total_bytes / (e2e_ms * 1e-3) / 1e9, "unit": "GB/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "ms_per_step": e2e_ms,
               "note": "every step: q, k_new, v_new, block_tables, seq_lens copied in from one pinned host buffer, "
                       "the step run through the C ABI, out read back to pinned memory; copy-in, compute and "
                       "copy-out pipelined on three streams (double-buffered); KV pools resident and larger "
                       "than L2 (no flush in this leg)"}
    pkv.pkv_destroy(ctx)

    peak, peak_src = measured_peak()
    value = total_bytes / (step_max * 1e-3) / 1e9
    attn_gbs = by / (attn_for_roofline * 1e-3) / 1e9
    traffic = recorded_traffic(name)
    kernel = (f"decode_attn_tokens_kernel<{w.d},bf16>" if tok
              else f"decode_attn_kernel<{w.d},{'e4m3' if w.kv_fp8 else 'bf16'}>")
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": step_max, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "e4m3-kv/bf16" if w.kv_fp8 else "bf16",
        "data": "synthetic: seeded lengths, page permutation, block tables and N(0,1) q/k/v "
                "(per-workload recipe in paged_kv_flight_b200/workloads.py)",
        "config": workload_config(w, name, world),
        "timing": ("median over the timed steps; each step replayed from one CUDA-graph capture of "
                   + ("pkv_rope_append + pkv_decode_attn" if args.two_calls else "pkv_decode_step")
                   + " (3 kernels); per-kernel times (rope_append_us, attn_us, step_us_eager) from the same "
                   "steps launched eagerly as two calls with events between them" if graph_ms is not None
                   else "median over the timed steps; eager launches through the C ABI"),
        "request_tokens_per_s": total_reqs / (step_max * 1e-3),
        "step_us": step_max * 1e3, "step_us_eager_one_call": max_over_ranks(med(step_call_ms)) * 1e3,
        "step_us_eager": eager_max * 1e3, "attn_us": attn_max * 1e3,
        "attn_us_in_graph": None if attn_graph_max is None else attn_graph_max * 1e3,
        "rope_append_us_in_graph": None if rope_graph_max is None else rope_graph_max * 1e3,
        "rope_append_us": max_over_ranks(med(rope_ms)) * 1e3,
        "ms_per_step_mean": step_mean,
        "step_us_hot_l2": hot_ms * 1e3,
        "pct_of_8TBs": 100.0 * value / world / NOMINAL_HBM_GBS,
        "pct_of_measured_peak": 100.0 * value / world / peak,
        "roofline": {"bound": "hbm", "achieved": attn_gbs, "peak": peak, "unit": "GB/s",
                     "frac": attn_gbs / peak, "traffic": traffic, "kernel": kernel,
                     "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)" if peak_src == "measured"
                     else "fallback 6650 GB/s",
                     "bytes_per_launch": by,
                     "duration": ("attention + combine inside a replayed CUDA graph (timing events as graph "
                                  "nodes), median" if attn_graph_max is not None
                                  else "attention + combine, eager events (launch gap included), median")},
        "e2e": e2e,
        "gpu_launches": 3 * K,
        "clocks": clock_info,
        "when": datetime.datetime.now(datetime.timezone.utc).isoformat(),
    }
    if cpu is not None:
        line["cpu_baseline"] = cpu
    return line


def run_reference(args, name, world=1, time_budget_s=45.0):
    """The CPU oracle as the reference arm, on a bounded sample per step: a
    prefix of the batch sized so that the warm-up and timed steps together
    take about `time_budget_s` of CPU time (at least one request; at most
    --ref-budget attended token-heads).  The oracle's rate is calibrated on
    the first request.  Under a multi-rank launch only rank 0 runs it; n_gpus
    mirrors the launch."""
    import torch
    from paged_kv_flight_b200 import workloads
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    w = workloads.make(name, device=dev)
    src = _device_inputs(w, dev)
    first = _request_pages(w, 0, src)
    t0 = time.perf_counter()
    oracle_step_requests(w, [first])
    rate = (int(w.seq_lens[0]) + w.q_len) * w.Hkv / max(time.perf_counter() - t0, 1e-6)   # token-heads / s
    budget = int(min(args.ref_budget, rate * time_budget_s / (args.steps + args.warmup)))
    picks = sample_requests(w, budget)
    lens = w.seq_lens[picks].astype(np.int64)
    if (int(lens[0]) + w.q_len) * w.Hkv > budget:
        # even the first request is over the step's budget (long contexts):
        # the sample is that request cut to the cached tokens that fit (at
        # least one page), so that the warm-up and timed steps stay bounded
        lens = np.array([max(w.P, min(int(lens[0]), budget // w.Hkv - w.q_len))], np.int64)
    views = [_request_pages(w, b, src, int(L)) for b, L in zip(picks, lens)]
    by = metric_bytes(lens, w.Hq, w.Hkv, w.d, w.P, w.kv_fp8, w.q_len)
    for _ in range(args.warmup):
        oracle_step_requests(w, views)
    ts = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        oracle_step_requests(w, views)
        ts.append(time.perf_counter() - t0)
    sec = statistics.median(ts)
    value = by / sec / 1e9
    toks = int((lens + w.q_len).sum())
    cut = "" if int(lens[0]) == int(w.seq_lens[picks[0]]) else f", cut to its first {int(lens[0])} cached tokens"
    sample = (f"requests 0..{len(picks) - 1} of {w.batch}{cut} ({toks} attended tokens, "
              f"{100.0 * by / workload_bytes(w):.1f}% of the step's bytes) per step; plain fp64 C oracle, "
              f"single thread, append + attention")
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic: same seeded workload as the GPU arm",
        "config": workload_config(w, name, world),
        "timing": "median over the timed steps of the oracle on the sampled requests (host wall clock)",
        "metric_bytes_per_step_sampled": by,
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": 1, "kind": "oracle", "sample": sample,
                         **host_cpu()},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def run_qkv(args, rank, world, local_rank):
    """The attention step from the layer input on the llama8b batch: the QKV
    projection on tcgen05 fused with RoPE and the append
    (pkv_qkv_rope_append: x [64, 4096] bf16, W [6144, 4096] bf16, N(0,1) and
    N(0, 1/4096)), then pkv_decode_attn.  L2 flushed before every step; the
    projection timed alone with events, the whole step replayed from a CUDA
    graph."""
    import torch
    from paged_kv_flight_b200 import pkv, workloads
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w = workloads.make("llama8b", device=dev, offset=rank)
    dv = _device_inputs(w, dev)
    hidden = 4096
    N = (w.Hq + 2 * w.Hkv) * w.d
    gen = torch.Generator(device=dev)
    gen.manual_seed(workloads.config_seed("llama8b", rank) + 17)
    x = torch.randn(w.batch, hidden, generator=gen, device=dev).to(torch.bfloat16)
    W = (torch.randn(N, hidden, generator=gen, device=dev) / hidden ** 0.5).to(torch.bfloat16)
    q = torch.empty(w.batch, w.Hq, w.d, dtype=torch.bfloat16, device=dev)
    out = torch.empty_like(q)
    cfg = pkv.make_config(w.Hq, w.Hkv, w.d, w.P, "bf16", w.rope_base, w.batch, w.bt_stride, w.num_pages)
    ctx = pkv.pkv_create(cfg)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush_w = torch.empty(2 * l2, dtype=torch.uint8, device=dev)
    flush_r = torch.ones(2 * l2 // 8, dtype=torch.int64, device=dev)
    sink = torch.empty((), dtype=torch.int64, device=dev)

    def flush():
        flush_w.zero_()
        torch.sum(flush_r, dim=0, out=sink)

    if args.qkv_split is not None:
        pkv.pkv_set_qkv_split(ctx, args.qkv_split)
    # the weight is static: packed once into the tiled layout at load time
    Wt = torch.empty_like(W)
    pkv.pkv_qkv_pack_weight(ctx, W, Wt)
    shape = pkv.pkv_qkv_launch_shape(ctx, w.batch, hidden)

    def proj(layout=pkv.PKV_W_TILED):
        pkv.pkv_qkv_rope_append(ctx, x, Wt if layout == pkv.PKV_W_TILED else W, q, dv["k_pool"], dv["v_pool"],
                                None, None, dv["block_tables"], dv["seq_lens"], w_layout=layout)

    def step():
        proj()
        pkv.pkv_decode_attn(ctx, q, dv["k_pool"], dv["v_pool"], None, None, dv["block_tables"], dv["seq_lens"], out)

    for _ in range(args.warmup):
        flush()
        step()
    torch.cuda.synchronize()
    K = args.steps
    side = torch.cuda.Stream(dev)
    with torch.cuda.stream(side):
        step()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=side):
        step()
    for _ in range(args.warmup):
        flush()
        graph.replay()
    torch.cuda.synchronize()
    clocks = ClockSampler(local_rank)
    barrier()
    torch.cuda.synchronize()
    clocks.start()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    for k in range(K):
        flush()
        ev[k][0].record()
        proj()
        ev[k][1].record()
    clocks.sample()
    rev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    for k in range(K):
        flush()
        rev[k][0].record()
        proj(pkv.PKV_W_ROWS)
        rev[k][1].record()
    gev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    for k in range(K):
        flush()
        gev[k][0].record()
        graph.replay()
        gev[k][1].record()
    clocks.sample()
    torch.cuda.synchronize()
    barrier()
    # the projection's own time inside a replayed step: timing events
    # recorded as graph nodes around it, each replay read back before the next
    proj_g = []
    try:
        te = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(2)]
        tgraph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(tgraph, stream=side):
            te[0].record()
            proj()
            te[1].record()
            pkv.pkv_decode_attn(ctx, q, dv["k_pool"], dv["v_pool"], None, None, dv["block_tables"], dv["seq_lens"],
                                out)
        for k in range(args.warmup + K):
            flush()
            tgraph.replay()
            torch.cuda.synchronize()
            if k >= args.warmup:
                proj_g.append(te[0].elapsed_time(te[1]))
        del tgraph
    except RuntimeError as e:
        print(f"bench: in-graph kernel timing unavailable ({e})", file=sys.stderr)
        proj_g = []
        torch.cuda.synchronize()
    clock_info = clocks.stop()
    st, bits = pkv.pkv_check_device_error(ctx)
    if st != pkv.PKV_OK:
        raise RuntimeError(f"device error: {pkv.pkv_status_str(st)} bits={bits}")
    del graph
    pkv.pkv_destroy(ctx)
    proj_graph_ms = max_over_ranks(statistics.median(proj_g)) if proj_g else None
    proj_ms = max_over_ranks(statistics.median(a.elapsed_time(b) for a, b in ev))
    rows_ms = max_over_ranks(statistics.median(a.elapsed_time(b) for a, b in rev))
    step_ms = max_over_ranks(statistics.median(a.elapsed_time(b) for a, b in gev))
    # the projection's algorithmic bytes: weights and x read once, q written,
    # k and v rows written; its flops: 2 x tokens x features x hidden
    proj_bytes = N * hidden * 2 + w.batch * hidden * 2 + w.batch * N * 2
    proj_flop = 2.0 * w.batch * N * hidden
    attn_bytes = workload_bytes(w)
    by = sum_over_ranks(float(proj_bytes + attn_bytes))
    peak, peak_src = measured_peak()
    proj_roof_ms = proj_graph_ms if proj_graph_ms is not None else proj_ms
    gbs = proj_bytes / (proj_roof_ms * 1e-3) / 1e9
    tflops_peak = None
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            tflops_peak = float(json.load(f)["bf16_tflops"])
    except Exception:
        tflops_peak = 1590.0
    return {"metric": METRIC, "value": by / (step_ms * 1e-3) / 1e9, "unit": "GB/s", "n_gpus": world,
            "steps": K, "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": "qkv8b", "description": "llama8b batch (64 tokens) from the layer input: "
                       "QKV projection 4096 -> 6144 on tcgen05 fused with RoPE + append, then decode attention",
                       "l2": "flushed before every step, outside the event window",
                       "timing": "projection: eager events and inside a replayed graph; step: CUDA-graph replay "
                                 "of projection + attention",
                       "weights": "packed once into the tiled layout (pkv_qkv_pack_weight) before timing"},
            "step_us": step_ms * 1e3, "projection_us": proj_ms * 1e3,
            "projection_us_in_graph": None if proj_graph_ms is None else proj_graph_ms * 1e3,
            "projection_rows_layout_us": rows_ms * 1e3,
            "projection_launch": dict(shape, clusters=w.Hq + 2 * w.Hkv),
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peak, "unit": "GB/s", "frac": gbs / peak,
                         "traffic": recorded_traffic("qkv8b"), "kernel": "qkv_rope_append_kernel<128>",
                         "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)", "bytes_per_launch": proj_bytes,
                         "duration": ("the projection inside a replayed CUDA graph (timing events as graph nodes), "
                                      "median" if proj_graph_ms is not None else "the projection, eager events, median")},
            "projection_tflops": proj_flop / (proj_roof_ms * 1e-3) / 1e12,
            "projection_tflops_frac_of_bf16_peak": proj_flop / (proj_roof_ms * 1e-3) / 1e12 / tflops_peak,
            "gpu_launches": 5 * K, "clocks": clock_info}


def run_mixed(args, rank, world, local_rank):
    """Chunked prefill mixed with decode (pkv_rope_append_varlen +
    pkv_decode_attn_varlen) on the llama8b batch: 8 seeded requests take a
    64-token chunk, the other 56 one new token.  L2 flushed before every step;
    the step replayed from a CUDA graph, attention alone timed eagerly."""
    import torch
    from paged_kv_flight_b200 import pkv, workloads
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w, q_lens = workloads.make_mixed(device=dev, offset=rank)
    B = w.batch
    cu = np.zeros(B + 1, np.int32)
    cu[1:] = np.cumsum(q_lens)
    n_tok = int(cu[-1])
    keep = torch.from_numpy(np.concatenate([b * w.q_len + np.arange(q) for b, q in enumerate(q_lens)])).to(dev)
    pack = lambda t: t.reshape(B * w.q_len, *t.shape[2:]).index_select(0, keep).contiguous()   # noqa: E731
    q0, k_new, v_new = pack(w.q), pack(w.k_new), pack(w.v_new)
    q = q0.clone()
    out = torch.empty_like(q)
    k_pool, v_pool = w.k_pool.to(dev).contiguous(), w.v_pool.to(dev).contiguous()
    bt = torch.from_numpy(w.block_tables).to(dev)
    sl = torch.from_numpy(w.seq_lens).to(dev)
    cu_d = torch.from_numpy(cu).to(dev)
    cfg = pkv.make_config(w.Hq, w.Hkv, w.d, w.P, "bf16", w.rope_base, B, w.bt_stride, w.num_pages)
    ctx = pkv.pkv_create(cfg)
    G = w.Hq // w.Hkv
    prefill_rows = 64 if args.prefill_rows is None else args.prefill_rows
    pkv.pkv_set_prefill_rows(ctx, prefill_rows)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush_w = torch.empty(2 * l2, dtype=torch.uint8, device=dev)
    flush_r = torch.ones(2 * l2 // 8, dtype=torch.int64, device=dev)
    sink = torch.empty((), dtype=torch.int64, device=dev)

    def flush():
        flush_w.zero_()
        torch.sum(flush_r, dim=0, out=sink)

    def attn():
        pkv.pkv_decode_attn_varlen(ctx, q, k_pool, v_pool, None, None, bt, sl, cu_d, out)

    def step():
        q.copy_(q0)    # the step rotates q in place: every step starts from the same q
        pkv.pkv_rope_append_varlen(ctx, q, k_new, v_new, k_pool, v_pool, None, None, bt, sl, cu_d)
        attn()

    for _ in range(args.warmup):
        flush()
        step()
    torch.cuda.synchronize()
    side = torch.cuda.Stream(dev)
    with torch.cuda.stream(side):
        step()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=side):
        step()
    for _ in range(args.warmup):
        flush()
        graph.replay()
    torch.cuda.synchronize()
    K = args.steps
    clocks = ClockSampler(local_rank)
    barrier()
    torch.cuda.synchronize()
    clocks.start()
    gev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    for k in range(K):
        flush()
        gev[k][0].record()
        graph.replay()
        gev[k][1].record()
    clocks.sample()
    aev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    for k in range(K):
        flush()
        aev[k][0].record()
        attn()
        aev[k][1].record()
    clocks.sample()
    torch.cuda.synchronize()
    barrier()
    clock_info = clocks.stop()
    st, bits = pkv.pkv_check_device_error(ctx)
    if st != pkv.PKV_OK:
        raise RuntimeError(f"device error: {pkv.pkv_status_str(st)} bits={bits}")
    del graph
    pkv.pkv_destroy(ctx)
    step_ms = max_over_ranks(statistics.median(a.elapsed_time(b) for a, b in gev))
    attn_ms = max_over_ranks(statistics.median(a.elapsed_time(b) for a, b in aev))
    L = w.seq_lens.astype(np.int64)
    row = 2 * w.Hkv * w.d * 2                      # K + V bytes of one token
    # metric bytes: each request's cache (its new tokens included) once, q and out of every new token
    by = int((row * (L + q_lens)).sum()) + 2 * n_tok * w.Hq * w.d * 2
    # streamed: every block reads its own prefix — blocks of 128 / G new tokens
    # for requests with G x new tokens >= prefill_rows (the tensor-core
    # prefill blocks), of 16 / G for the others
    cmin = -(-prefill_rows // G) if prefill_rows > 0 else None
    chunked = [cmin is not None and int(qb) >= cmin for qb in q_lens]
    n_chunked = sum(chunked)
    streamed = sum(row * (int(Lb) + min(j + blk, int(qb)))
                   for Lb, qb, ch in zip(L, q_lens, chunked)
                   for blk in [128 // G if ch else 16 // G]
                   for j in range(0, int(qb), blk)) + 2 * n_tok * w.Hq * w.d * 2
    peak, peak_src = measured_peak()
    gbs = by / (attn_ms * 1e-3) / 1e9
    return {"metric": METRIC, "value": sum_over_ranks(float(by)) / (step_ms * 1e-3) / 1e9, "unit": "GB/s",
            "n_gpus": world, "steps": K, "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": "mixed",
                       "description": "llama8b batch, 56 requests decode one token, 8 prefill a 64-token "
                                      "chunk (568 new tokens): varlen RoPE + append, then varlen attention",
                       "l2": "flushed before every step, outside the event window",
                       "timing": "step: CUDA-graph replay; attention alone: eager events",
                       "prefill_rows": prefill_rows, "prefill_requests": n_chunked},
            "step_us": step_ms * 1e3, "attn_us": attn_ms * 1e3, "new_tokens": n_tok,
            "new_tokens_per_s": sum_over_ranks(float(n_tok)) / (step_ms * 1e-3),
            "streamed_bytes_per_launch": streamed,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peak, "unit": "GB/s", "frac": gbs / peak,
                         "traffic": recorded_traffic("mixed"),
                         "kernel": ("chunk_attn_kernel<128> + " if n_chunked else "") + "decode_attn_tokens_kernel<128> (varlen)",
                         "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)", "bytes_per_launch": by,
                         "note": "bytes = each request's cache once (the metric); a prefill chunk's blocks "
                                 "re-read their prefix, see streamed_bytes_per_launch"},
            # step: rope, plan, (prefill blocks,) attention, combine; alone: the same without rope
            "gpu_launches": (9 if n_chunked else 7) * K, "clocks": clock_info}


def run_loop(args, rank, world, local_rank):
    """The continuous-batching loop (serve_loop.py) on a 70B-shaped layer:
    256 slots, prompts {64,128,512,2048} (+ a 512-token system prompt shared
    through its pages by 30% of requests), output budgets U[16,500]; the
    host page allocator runs between steps, finished requests are replaced.
    Times `--steps` iterations on the device (host scheduling gaps
    included)."""
    import torch
    from paged_kv_flight_b200 import serve_loop
    torch.cuda.set_device(local_rank)
    cfg = serve_loop.LoopConfig(seed=serve_loop.LoopConfig.seed + 1000 * rank)
    clocks = ClockSampler(local_rank)
    barrier()
    clocks.start()
    r = serve_loop.run(cfg, args.steps, warmup=args.warmup, device=f"cuda:{local_rank}")
    clock_info = clocks.stop()
    sec = max_over_ranks(r["seconds"])
    gbs = sum_over_ranks(r["attended_GB_per_s"] * r["seconds"]) / sec
    toks = sum_over_ranks(r["decode_tokens_per_s"] * r["seconds"]) / sec
    return {"metric": METRIC, "value": gbs, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * sec / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded request stream)",
            "config": {"workload": "loop70b",
                       "description": "continuous batching over 256 slots, Hq 64 / Hkv 8, d 128, page 16: "
                                      "host page allocator between steps, requests finish and are replaced, "
                                      "30% share a 512-token system prompt's pages",
                       "timing": "device events around all iterations; host allocator calls, the one H2D "
                                 "copy per step of the table changes, slots and lengths, the device table "
                                 "sync (pkv_table_sync) and the stand-in prefill of new requests' pages "
                                 "included; L2 not flushed (the pools are far larger)"},
            "decode_tokens_per_s": toks, "us_per_iteration": r["us_per_iteration"],
            "host_allocator_us_per_iteration": r["host_allocator_us_per_iteration"],
            "loop_stats": r["stats"], "gpu_launches": int(r["stats"].get("pkv_launches", 0)), "clocks": clock_info}


def run_each_in_own_process(args, names) -> int:
    """One GPU, several workloads: each runs in a fresh process of this script
    (its own CUDA context and allocator), and its JSON line is passed on.
    Measured on one box: the 70B-shaped workload's step ran 5% slower right
    after the llama8b workload in the same process than alone, with the same
    flags."""
    import subprocess
    flags = ["--steps", str(args.steps), "--warmup", str(args.warmup), "--gpus", "1"]
    for opt in ("no_e2e", "no_cpu_baseline", "no_graph", "two_calls"):
        if getattr(args, opt):
            flags.append("--" + opt.replace("_", "-"))
    if args.tail_chunks is not None:
        flags += ["--tail-chunks", str(args.tail_chunks)]
    if args.prefill_rows is not None:
        flags += ["--prefill-rows", str(args.prefill_rows)]
    if args.requests is not None:
        flags += ["--requests", str(args.requests)]
    for i, name in enumerate(names):
        last = i == len(names) - 1
        # the full CPU-baseline budget on the last line printed, a short one before it
        budget = args.cpu_budget if last else min(5.0, args.cpu_budget)
        cmd = [sys.executable, os.path.abspath(__file__), "--config", name, "--cpu-budget", str(budget), *flags]
        r = subprocess.run(cmd, stdout=subprocess.PIPE, text=True)
        for ln in r.stdout.splitlines():
            if ln.startswith("{"):
                print(ln, flush=True)
        if r.returncode != 0:
            print(f"bench: workload {name} failed (exit {r.returncode})", file=sys.stderr)
            return r.returncode
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--config", default=DEFAULT_CONFIG,
                    help="a workload, 'suite' (the default: " + ", ".join(SUITE) + ", in that order) or 'all'")
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graph", action="store_true", help="skip the CUDA-graph replay timing")
    ap.add_argument("--two-calls", action="store_true",
                    help="time the step as pkv_rope_append + pkv_decode_attn instead of pkv_decode_step")
    ap.add_argument("--tail-chunks", type=int, default=None,
                    help="cap on dynamic tail chunks per warp range (library default if omitted; 0: static split)")
    ap.add_argument("--prefill-rows", type=int, default=None,
                    help="mixed: G x new tokens from which a request takes the tensor-core prefill blocks "
                         "(library default 64 if omitted; 0: none)")
    ap.add_argument("--cpu-budget", type=float, default=20.0, help="seconds of oracle work for cpu_baseline")
    ap.add_argument("--requests", type=int, default=None,
                    help="keep only the first N requests of the workload (a smaller case for profiler captures)")
    ap.add_argument("--ref-budget", type=int, default=1_200_000,
                    help="attended token-heads per reference step")
    ap.add_argument("--qkv-split", type=int, default=None,
                    help="qkv8b: CTAs per head for the projection (1..4; library choice if omitted)")
    ap.add_argument("--in-process", action="store_true",
                    help="on one GPU, run several workloads in this process instead of one process each")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    from paged_kv_flight_b200 import workloads
    if args.config == "all":
        names = list(workloads.CONFIG_NAMES) + list(workloads.TOKEN_CONFIG_NAMES)
    elif args.config == "suite":
        names = list(SUITE)
    else:
        names = [args.config]
    rank, world, local_rank = dist_info()

    if args.impl == "reference":
        if rank != 0:
            return 0
        for i, name in enumerate(names):
            last = i == len(names) - 1
            print(json.dumps(run_reference(args, name, world, time_budget_s=45.0 if last else 12.0)), flush=True)
        return 0

    if world == 1 and len(names) > 1 and not args.in_process:
        return run_each_in_own_process(args, names)

    import torch
    if world > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    try:
        for i, name in enumerate(names):
            last = i == len(names) - 1
            if name == "loop70b":
                line = run_loop(args, rank, world, local_rank)
            elif name == "qkv8b":
                line = run_qkv(args, rank, world, local_rank)
            elif name == "mixed":
                line = run_mixed(args, rank, world, local_rank)
            else:
                # the full CPU-baseline budget on the last line printed, a short one before it
                line = run_ours(args, name, rank, world, local_rank,
                                cpu_budget=args.cpu_budget if last else min(5.0, args.cpu_budget))
            if rank == 0:
                print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
