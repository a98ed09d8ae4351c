"""Seeded input generator: shapes, length recipes, page assignment, NaN
sentinels and determinism (CPU only)."""
import numpy as np
import pytest
import torch

from paged_kv_flight_b200 import workloads


def test_tiny_matches_its_recipe():
    w = workloads.make("tiny")
    assert list(w.seq_lens) == [17, 64, 100, 255]
    assert w.num_pages == 64
    pages = (w.seq_lens + 1 + w.P - 1) // w.P
    assert list(pages) == [2, 5, 7, 16]
    used = w.block_tables[w.block_tables >= 0]
    assert len(used) == 30 and len(set(used.tolist())) == 30
    assert tuple(w.q.shape) == (4, 8, 64) and tuple(w.k_pool.shape) == (64, 2, 16, 64)


@pytest.mark.parametrize("name", ["llama8b", "hetero70b", "longctx", "fp8"])
def test_length_recipes(name):
    seed = workloads.config_seed(name)
    L = workloads.draw_lengths(name, np.random.default_rng(seed))
    if name == "llama8b":
        assert len(L) == 64 and L.min() >= 128 and L.max() <= 4096
    if name == "hetero70b":
        assert len(L) == 256 and (L == 64).sum() >= 51
        prompts = {64, 128, 512, 2048}
        assert all(any(0 <= x - p <= 500 for p in prompts) for x in L)
    if name == "longctx":
        assert len(L) == 8 and L.min() >= 32768 and L.max() <= 131072
    if name == "fp8":
        assert len(L) == 128 and L.min() >= 16 and L.max() <= 16384
        assert 600 < np.median(L) < 1700


def test_sentinels_and_resident_slots_bf16():
    w = workloads.build("t", 4, 2, 16, 8, False, 1e4, [0, 7, 8, 19], seed=3)
    bits = w.k_pool.view(torch.int16).numpy().view(np.uint16)
    for b, L in enumerate(w.seq_lens):
        for t in range(int(L) + 1 + 8):
            lp = t // w.P
            if lp >= w.block_tables.shape[1] or w.block_tables[b, lp] < 0:
                continue
            row = bits[w.block_tables[b, lp], :, t % w.P, :]
            if t < L:
                assert not np.any(row == workloads.BF16_NAN_BITS)
            else:
                assert np.all(row == workloads.BF16_NAN_BITS)   # landing slot and beyond
    used = set(w.block_tables[w.block_tables >= 0].tolist())
    free = [p for p in range(w.num_pages) if p not in used]
    assert free and np.all(bits[free] == workloads.BF16_NAN_BITS)


def test_fp8_scales_and_codes():
    w = workloads.build("t", 4, 2, 32, 16, True, 1e4, [3, 16, 40], seed=5)
    assert w.k_pool.dtype == torch.uint8 and w.k_scale.dtype == torch.float32
    codes = w.k_pool.numpy()
    used = sorted(set(w.block_tables[w.block_tables >= 0].tolist()))
    for p in used:
        for kvh in range(w.Hkv):
            vals = codes[p, kvh]
            finite = vals[vals != workloads.E4M3_NAN_CODE]
            assert np.all((finite & 0x7F) <= 0x7E)
    assert np.all(w.k_scale.numpy() > 0)


def test_deterministic():
    a = workloads.make("tiny")
    b = workloads.make("tiny")
    assert torch.equal(a.k_pool.view(torch.int16), b.k_pool.view(torch.int16))
    assert np.array_equal(a.block_tables, b.block_tables)
    c = workloads.make("tiny", offset=1)
    assert not torch.equal(a.q.view(torch.int16), c.q.view(torch.int16))
