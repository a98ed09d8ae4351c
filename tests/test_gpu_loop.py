"""The continuous-batching loop (paged_kv_flight_b200/serve_loop.py) on the
GPU: block tables come from the host page allocator, requests finish and are
replaced, a share of them reuses the system prompt's pages.  At sampled
iterations the step's inputs (pools, q, k_new, v_new, the batch's block
table and lengths) are copied to the host before the step and the oracle
recomputes the whole step from them; the GPU step must match it, and the
system prompt's shared pages must never change."""
import numpy as np
import pytest
import torch

import oracle
from paged_kv_flight_b200 import serve_loop
from tests import _gpu
from tests._util import bits16

pytestmark = pytest.mark.gpu


def _cfg():
    return serve_loop.LoopConfig(Hq=8, Hkv=2, d=64, P=16, rope_base=1e4, max_batch=12, num_pages=160,
                                 max_blocks=48, prompts=(5, 40, 100), budget=(2, 12), system_prompt=48,
                                 share_frac=0.5, seed=7)


def test_loop_steps_match_oracle_and_shared_pages_stay_put():
    loop = serve_loop.DecodeLoop(_cfg())
    try:
        c = loop.cfg
        shared_pages = loop.pages.block_table[0, :c.system_prompt // c.P].astype(np.int64).copy()
        idx = torch.from_numpy(shared_pages).cuda()
        k_shared0 = bits16(loop.k_pool.index_select(0, idx))
        v_shared0 = bits16(loop.v_pool.index_select(0, idx))
        checked = 0
        for it in range(80):
            slots = loop.schedule()
            q, k_new, v_new = loop.inputs(len(slots))
            snap = None
            if it in (3, 20, 47, 79):
                bt, ln = loop.batch_tables(len(slots))
                snap = dict(q=bits16(q), k_new=bits16(k_new), v_new=bits16(v_new),
                            k_pool=bits16(loop.k_pool), v_pool=bits16(loop.v_pool),
                            block_tables=bt.cpu().numpy().copy(), seq_lens=ln.cpu().numpy().copy())
                # the device table the step reads is the allocator's table
                assert np.array_equal(snap["block_tables"], loop.pages.block_table[slots])
                assert np.array_equal(snap["seq_lens"], loop.pages.seq_lens[slots])
            out = torch.empty_like(q)
            loop.device_step(slots, q, k_new, v_new, out)
            if snap is not None:
                torch.cuda.synchronize()
                cfg = oracle.OracleConfig(c.Hq, c.Hkv, c.d, c.P, False, c.num_pages, c.rope_base)
                assert oracle.rope_append(cfg, snap["q"], snap["k_new"], snap["v_new"], snap["k_pool"],
                                          snap["v_pool"], None, None, snap["block_tables"], snap["seq_lens"]) == 0
                ref, st = oracle.decode_attn(cfg, snap["q"], snap["k_pool"], snap["v_pool"], None, None,
                                             snap["block_tables"], snap["seq_lens"])
                assert st == 0
                mx, mean, finite = _gpu.errors(out, ref)
                assert finite and mx <= _gpu.TOL_BF16["max"] and mean <= _gpu.TOL_BF16["mean"], (it, mx, mean)
                # the step appended exactly what the oracle appended (V bit for bit)
                assert np.array_equal(bits16(loop.v_pool), snap["v_pool"])
                checked += 1
            loop.finish(slots)
        torch.cuda.synchronize()
        assert pkv_ok(loop)
        assert checked == 4
        assert loop.stats["finished"] > 20 and loop.stats["shared"] > 5
        assert np.array_equal(bits16(loop.k_pool.index_select(0, idx)), k_shared0)
        assert np.array_equal(bits16(loop.v_pool.index_select(0, idx)), v_shared0)
    finally:
        loop.close()


def pkv_ok(loop):
    from paged_kv_flight_b200 import pkv
    return pkv.pkv_check_device_error(loop.ctx)[0] == pkv.PKV_OK


def test_loop_survives_a_tight_pool_by_preempting():
    c = _cfg()
    c.num_pages = 60                       # too few pages for every slot to keep growing
    c.budget = (30, 60)
    loop = serve_loop.DecodeLoop(c)
    try:
        for _ in range(60):
            loop.step()
        torch.cuda.synchronize()
        assert pkv_ok(loop)
        assert loop.stats["preempted"] > 0
        # every page is free or referenced by the slots that name it
        names = np.zeros(c.num_pages, np.int64)
        for s in range(c.max_batch):
            if loop.pages.active[s]:
                r = loop.pages.block_table[s]
                np.add.at(names, r[r >= 0], 1)
        assert (names == np.asarray(loop.pages.refcount)).all()
    finally:
        loop.close()


def test_table_sync_applies_changes_and_gathers_rows():
    """pkv_table_sync against numpy: every in-range triple applied, triples
    outside the table skipped, each batch row = the updated table's row of its
    slot (a slot outside the table gives -1), lengths passed through."""
    from paged_kv_flight_b200 import pkv
    rng = np.random.default_rng(3)
    max_batch, max_blocks = 12, 20
    table = rng.integers(-1, 100, size=(max_batch, max_blocks)).astype(np.int32)
    keys = rng.choice(max_batch * max_blocks, size=40, replace=False)
    chg = np.stack([keys // max_blocks, keys % max_blocks, rng.integers(0, 100, 40)], 1).astype(np.int32)
    chg = np.concatenate([chg, np.array([[max_batch + 3, 0, 7], [0, max_blocks, 7], [-1, 2, 7]], np.int32)])
    slots = np.array([5, 0, 11, 3, 40], np.int32)
    lens = np.array([10, 0, 300, 17, 5], np.int32)
    up = torch.from_numpy(np.concatenate([chg.ravel(), slots, lens]).astype(np.int32)).cuda()
    t_dev = torch.from_numpy(table.copy()).cuda()
    bt = torch.zeros(len(slots), max_blocks, dtype=torch.int32, device="cuda")
    ln = torch.zeros(len(slots), dtype=torch.int32, device="cuda")
    pkv.pkv_table_sync(up, len(chg), len(slots), t_dev, bt, ln, 16)
    ref = table.copy()
    for s, i, v in chg[:40]:
        ref[s, i] = v
    assert np.array_equal(t_dev.cpu().numpy(), ref)
    want = np.stack([ref[s] if 0 <= s < max_batch else np.full(max_blocks, -1, np.int32) for s in slots])
    assert np.array_equal(bt.cpu().numpy(), want)
    assert np.array_equal(ln.cpu().numpy(), lens)
    assert pkv.pkv_table_sync(up, -1, 1, t_dev, bt, ln, 16, check=False) == pkv.PKV_ERR_INVALID_ARG
    assert pkv.pkv_table_sync(up, 0, 13, t_dev, bt, ln, 16, check=False) == pkv.PKV_ERR_INVALID_ARG
