"""A continuous-batching decode loop over one layer's paged KV pools: the
host page allocator (include/pkv_pages.h) between steps, the decode step
through libpkv on the GPU.

Each iteration, after the pages ("TensorRT-LLM Guide: High-Throughput GPU
Inference Engine", section "1. In-Flight Batching: Continuous Iteration
Scheduling"; "Scaling TensorRT-LLM: Kernel Fusion and Inflight Batching in
Production", section "What the Scheduler Actually Does"):

  1. reserve a page for every active request whose new token crosses into a
     new page (pages are allocated on demand as tokens are generated); if the
     pool is short, preempt the most recently admitted request (its pages go
     back, it is re-queued to be recomputed later) and retry;
  2. bring the device copy of the block table up to date by applying the
     allocator's change log (a few entries per step instead of the whole
     table), and gather the active slots' rows and lengths into a contiguous
     batch on the device: one pinned upload (changes, slots, lengths) and one
     pkv_table_sync call, two small kernels;
  3. run the step: pkv_rope_append + pkv_decode_attn over that batch;
  4. advance every active request by one token; requests that reached their
     output budget finish, their pages return to the pool at once, and
     waiting requests take the freed slots (their prompt's KV is written into
     their own pages: a stand-in for the prefill pass, which is not this
     loop's work).

A share of the requests reuses the full pages of a common system prompt held
by slot 0 ("TensorRT-LLM: NVIDIA's Optimized Inference Engine", section "The
paged KV cache, in-flight batching and CUDA graphs": blocks reused across
requests that share a prefix).  Prompt lengths, output budgets and the
sharing choice are seeded draws; K/V, q, k_new, v_new are N(0, 1) bf16.
"""
from __future__ import annotations

import collections
import time
from dataclasses import dataclass

import numpy as np
import torch

from . import pkv


@dataclass
class LoopConfig:
    Hq: int = 64
    Hkv: int = 8
    d: int = 128
    P: int = 16
    rope_base: float = 5e5
    max_batch: int = 256            # batch slots; slot 0 holds the system prompt
    num_pages: int = 16384
    max_blocks: int = 512           # pages per request at most
    prompts: tuple = (64, 128, 512, 2048)
    budget: tuple = (16, 500)       # output tokens per request, uniform
    system_prompt: int = 512        # tokens of the shared prefix
    share_frac: float = 0.3         # requests that start with the system prompt
    seed: int = 20260100


class _Staging:
    """Pinned host buffers for one iteration's uploads, reused in a ring: a
    buffer is rewritten only after the event recorded behind its last copy
    has completed, so the host never overwrites data a queued copy reads."""

    def __init__(self, max_changes, max_batch, max_blocks):
        pin = lambda n: torch.empty(n, dtype=torch.int32).pin_memory()
        self.upload = pin(3 * max_changes + 2 * max_batch)    # changes, then slots, then lengths
        self.pages = torch.empty(max_blocks, dtype=torch.int64).pin_memory()
        self.done = None

    def wait(self):
        if self.done is not None:
            self.done.synchronize()


class DecodeLoop:
    def __init__(self, cfg: LoopConfig, device="cuda"):
        self.cfg = c = cfg
        self.dev = torch.device(device)
        self.rng = np.random.default_rng(c.seed)
        self.gen = torch.Generator(device=self.dev)
        self.gen.manual_seed(c.seed)
        shape = (c.num_pages, c.Hkv, c.P, c.d)
        nan = torch.tensor(0x7FC0, dtype=torch.int16).view(torch.bfloat16).item()
        self.k_pool = torch.full(shape, nan, dtype=torch.bfloat16, device=self.dev)
        self.v_pool = torch.full(shape, nan, dtype=torch.bfloat16, device=self.dev)
        self.pages = pkv.Pages(c.num_pages, c.P, c.max_batch, c.max_blocks)
        self.ctx = pkv.pkv_create(pkv.make_config(c.Hq, c.Hkv, c.d, c.P, "bf16", c.rope_base, c.max_batch,
                                                  c.max_blocks, c.num_pages))
        self.budget = np.zeros(c.max_batch, np.int64)     # output tokens left per slot
        self.admitted_at = np.zeros(c.max_batch, np.int64)
        self.queue = collections.deque()
        self.iteration = 0
        self.stats = collections.Counter()
        # uploads go through a ring of pinned buffers; the device keeps its
        # own copy of the whole block table, updated from the change log
        self.max_changes = c.num_pages + 1024
        self.ring = [_Staging(self.max_changes, c.max_batch, c.max_blocks) for _ in range(16)]
        self.ring_i = 0
        self.table_dev = torch.full((c.max_batch, c.max_blocks), -1, dtype=torch.int32, device=self.dev)
        self.upload_dev = torch.empty(3 * self.max_changes + 2 * c.max_batch, dtype=torch.int32, device=self.dev)
        self.bt_dev = torch.full((c.max_batch, c.max_blocks), -1, dtype=torch.int32, device=self.dev)
        self.len_dev = torch.empty(c.max_batch, dtype=torch.int32, device=self.dev)
        self.slots = np.zeros(0, np.int64)
        # slot 0: the system prompt, decoding for the whole run
        self._admit(0, (c.system_prompt, 1 << 40, False))
        for s in range(1, c.max_batch):
            self._admit(s, self._draw())

    # ---- requests -------------------------------------------------------------
    def _draw(self):
        c = self.cfg
        shared = bool(self.rng.random() < c.share_frac)
        prompt = int(self.rng.choice(np.array(c.prompts)))
        if shared:
            prompt += c.system_prompt
        return prompt, int(self.rng.integers(c.budget[0], c.budget[1], endpoint=True)), shared

    def _admit(self, slot, req) -> bool:
        length, budget, shared = req
        c = self.cfg
        share_tokens = min(c.system_prompt, int(self.pages.seq_lens[0])) if shared and slot != 0 else 0
        st = self.pages.admit(slot, length, 0 if share_tokens else -1, share_tokens, check=False)
        if st != pkv.PKV_OK:
            return False
        self.budget[slot] = budget
        self.admitted_at[slot] = self.iteration
        # the prompt's KV in the request's own pages (stand-in for its prefill)
        own = share_tokens // c.P
        npg = -(-length // c.P)
        if npg > own:
            st_buf = self._staging()
            host = st_buf.pages[:npg - own]
            host.numpy()[:] = self.pages.block_table[slot, own:npg]
            pages = host.to(self.dev, non_blocking=True)
            st_buf.done = torch.cuda.Event()
            st_buf.done.record()
            kv = torch.randn((2, len(pages), c.Hkv, c.P, c.d), generator=self.gen, device=self.dev,
                             dtype=torch.bfloat16)
            self.k_pool.index_copy_(0, pages, kv[0])
            self.v_pool.index_copy_(0, pages, kv[1])
        self.stats["admitted"] += 1
        self.stats["shared"] += int(share_tokens > 0)
        return True

    def _preempt_one(self) -> bool:
        active = np.flatnonzero(self.pages.active[1:]) + 1
        if len(active) == 0:
            return False
        victim = int(active[np.argmax(self.admitted_at[active])])
        self.queue.appendleft((int(self.pages.seq_lens[victim]), int(self.budget[victim]), False))
        self.pages.release(victim)
        self.stats["preempted"] += 1
        return True

    def _staging(self) -> _Staging:
        self.ring_i = (self.ring_i + 1) % len(self.ring)
        st = self.ring[self.ring_i]
        st.wait()
        return st

    # ---- one iteration ---------------------------------------------------------------
    def schedule(self):
        """Host part before the step: pages for the new tokens; the device
        table brought up to date from the change log; the batch's slots and
        lengths uploaded (all copies asynchronous, on the current stream)."""
        while self.pages.reserve(1, check=False) == pkv.PKV_ERR_OOM:
            if not self._preempt_one():
                raise RuntimeError("page pool too small for one request")
        st = self._staging()
        up = st.upload.numpy()
        # the last write of each table entry, once (the allocator merges repeats)
        n = self.pages.take_changes(up[:3 * self.max_changes])
        if n < 0:      # too many writes for the log: copy the whole table
            self.table_dev.copy_(torch.from_numpy(self.pages.block_table.copy()))
            n = 0
        slots = np.flatnonzero(self.pages.active)
        B = len(slots)
        up[3 * n:3 * n + B] = slots
        up[3 * n + B:3 * n + 2 * B] = self.pages.seq_lens[slots]
        k = 3 * n + 2 * B
        self.upload_dev[:k].copy_(st.upload[:k], non_blocking=True)
        st.done = torch.cuda.Event()
        st.done.record()
        pkv.pkv_table_sync(self.upload_dev, n, B, self.table_dev, self.bt_dev, self.len_dev, self.cfg.P)
        self.stats["pkv_launches"] += (n > 0) + (B > 0)          # apply changes, gather rows
        self.slots = slots
        return slots

    def inputs(self, B):
        """q, k_new, v_new of the step: N(0, 1) bf16, one draw cut in three."""
        c = self.cfg
        nq, nk = B * c.Hq * c.d, B * c.Hkv * c.d
        flat = torch.randn(nq + 2 * nk, generator=self.gen, device=self.dev, dtype=torch.bfloat16)
        return (flat[:nq].view(B, c.Hq, c.d), flat[nq:nq + nk].view(B, c.Hkv, c.d),
                flat[nq + nk:].view(B, c.Hkv, c.d))

    def batch_tables(self, B):
        """The batch's block-table rows (gathered on the device by
        pkv_table_sync in schedule) and lengths."""
        return self.bt_dev[:B], self.len_dev[:B]

    def device_step(self, slots, q, k_new, v_new, out):
        bt, ln = self.batch_tables(len(slots))
        pkv.pkv_rope_append(self.ctx, q, k_new, v_new, self.k_pool, self.v_pool, None, None, bt, ln)
        pkv.pkv_decode_attn(self.ctx, q, self.k_pool, self.v_pool, None, None, bt, ln, out)
        self.stats["pkv_launches"] += 3                          # rope + append, attention, combine
        return bt, ln

    def finish(self, slots):
        """Host part after the step: one token more, finished requests out,
        waiting ones in."""
        self.pages.advance(1)
        self.budget[slots] -= 1
        done = slots[(slots != 0) & (self.budget[slots] <= 0)]
        for s in done:
            self.pages.release(int(s))
        self.stats["finished"] += len(done)
        self.iteration += 1
        for s in np.flatnonzero(self.pages.active == 0):
            if s == 0:
                continue
            req = self.queue.popleft() if self.queue else self._draw()
            if not self._admit(int(s), req):
                self.queue.appendleft(req)
                break
        self.stats["tokens"] += len(slots)

    def step(self):
        slots = self.schedule()
        q, k_new, v_new = self.inputs(len(slots))
        out = torch.empty_like(q)
        self.device_step(slots, q, k_new, v_new, out)
        self.finish(slots)
        return out

    def close(self):
        pkv.pkv_destroy(self.ctx)
        self.pages.close()


def run(cfg: LoopConfig, iterations: int, warmup: int = 5, device="cuda") -> dict:
    """Runs the loop and times it: device events around the whole timed
    stretch (host scheduling gaps included), host time per iteration of the
    allocator calls, and the attended bytes of every step."""
    loop = DecodeLoop(cfg, device)
    try:
        for _ in range(warmup):
            loop.step()
        torch.cuda.synchronize()
        st, bits = pkv.pkv_check_device_error(loop.ctx)
        if st != pkv.PKV_OK:
            raise RuntimeError(f"device error in the loop: {pkv.pkv_status_str(st)} bits={bits}")
        c = cfg
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        host_s, tokens, by = 0.0, 0, 0
        pages0 = dict(loop.stats)
        a.record()
        for _ in range(iterations):
            t0 = time.perf_counter()
            slots = loop.schedule()
            host_s += time.perf_counter() - t0
            lens = loop.pages.seq_lens[slots].astype(np.int64)
            by += int((2 * c.Hkv * (lens + 1) * c.d * 2).sum()) + 2 * len(slots) * c.Hq * c.d * 2
            q, k_new, v_new = loop.inputs(len(slots))
            out = torch.empty_like(q)
            loop.device_step(slots, q, k_new, v_new, out)
            t0 = time.perf_counter()
            loop.finish(slots)
            host_s += time.perf_counter() - t0
            tokens += len(slots)
        b.record()
        torch.cuda.synchronize()
        st, bits = pkv.pkv_check_device_error(loop.ctx)
        if st != pkv.PKV_OK:
            raise RuntimeError(f"device error in the loop: {pkv.pkv_status_str(st)} bits={bits}")
        sec = a.elapsed_time(b) * 1e-3
        stats = {k: v - pages0.get(k, 0) for k, v in loop.stats.items()}
        return {"iterations": iterations, "seconds": sec, "us_per_iteration": 1e6 * sec / iterations,
                "decode_tokens_per_s": tokens / sec, "attended_GB_per_s": by / sec / 1e9,
                "host_allocator_us_per_iteration": 1e6 * host_s / iterations, "stats": stats,
                "pages_free_at_end": loop.pages.free_count}
    finally:
        loop.close()
