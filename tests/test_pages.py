"""The host page allocator (include/pkv_pages.h) against a plain Python model
of the same bookkeeping, on random sequences of admissions (some sharing a
prefix), step reservations, advances and releases, valid and invalid.

The model is the definition written out: a slot holds ceil(L / P) pages (or
more, after a reservation), a shared prefix of S tokens shares floor(S / P)
full pages, a page's reference count is the number of slots whose table
names it, and a page returns to the free stack when its count drops to 0.
Runs on the CPU (host code only)."""
import random

import numpy as np
import pytest

from paged_kv_flight_b200 import pkv

OK, INVALID, OOM = pkv.PKV_OK, pkv.PKV_ERR_INVALID_ARG, pkv.PKV_ERR_OOM


class Model:
    def __init__(self, num_pages, P, max_batch, max_blocks):
        self.N, self.P, self.B, self.M = num_pages, P, max_batch, max_blocks
        self.rows = {}                       # slot -> list of pages
        self.lens = {}
        self.ref = [0] * num_pages
        self.free = list(range(num_pages - 1, -1, -1))   # top = last element

    def _pop(self):
        p = self.free.pop()
        self.ref[p] = 1
        return p

    def admit(self, slot, length, share_slot=-1, share_tokens=0):
        if not (0 <= slot < self.B) or slot in self.rows or length < 0:
            return INVALID
        need = -(-length // self.P)
        if need > self.M:
            return INVALID
        shared = 0
        if share_slot >= 0:
            if not (0 <= share_slot < self.B) or share_slot == slot or share_slot not in self.rows:
                return INVALID
            if share_tokens < 0 or share_tokens > length or share_tokens > self.lens[share_slot]:
                return INVALID
            shared = share_tokens // self.P
        if need - shared > len(self.free):
            return OOM
        row = list(self.rows[share_slot][:shared]) if shared else []
        for p in row:
            self.ref[p] += 1
        row += [self._pop() for _ in range(need - shared)]
        self.rows[slot], self.lens[slot] = row, length
        return OK

    def reserve(self, q_len):
        if q_len < 1:
            return INVALID
        want = 0
        for s, row in self.rows.items():
            need = -(-(self.lens[s] + q_len) // self.P)
            if need > self.M:
                return INVALID
            want += max(0, need - len(row))
        if want > len(self.free):
            return OOM
        for s in sorted(self.rows):
            need = -(-(self.lens[s] + q_len) // self.P)
            while len(self.rows[s]) < need:
                self.rows[s].append(self._pop())
        return OK

    def advance(self, q_len):
        if q_len < 1:
            return INVALID
        for s, row in self.rows.items():
            if -(-(self.lens[s] + q_len) // self.P) > len(row):
                return INVALID
        for s in self.rows:
            self.lens[s] += q_len
        return OK

    def release(self, slot):
        if slot not in self.rows:
            return INVALID
        for p in self.rows.pop(slot):
            self.ref[p] -= 1
            if self.ref[p] == 0:
                self.free.append(p)
        del self.lens[slot]
        return OK


def _agree(pp, m):
    assert pp.free_count == len(m.free)
    assert list(pp.refcount) == m.ref
    for s in range(m.B):
        row = pp.block_table[s]
        if s in m.rows:
            assert pp.active[s] == 1 and pp.seq_lens[s] == m.lens[s]
            n = len(m.rows[s])
            assert list(row[:n]) == m.rows[s] and (row[n:] == -1).all()
        else:
            assert pp.active[s] == 0 and pp.seq_lens[s] == 0 and (row == -1).all()
    # invariants, independent of the model's own bookkeeping
    names = np.zeros(m.N, np.int64)
    for s in range(m.B):
        if pp.active[s]:
            r = pp.block_table[s]
            pages = r[r >= 0]
            assert len(pages) >= -(-int(pp.seq_lens[s]) // m.P)
            np.add.at(names, pages, 1)
    assert (names == np.asarray(pp.refcount)).all()
    assert int((names == 0).sum()) == pp.free_count


@pytest.mark.parametrize("seed", range(12))
def test_random_operations_match_the_model(seed):
    rnd = random.Random(seed)
    N, P, B, M = rnd.choice([(40, 16, 6, 10), (200, 16, 12, 40), (64, 32, 8, 8)])
    pp, m = pkv.Pages(N, P, B, M), Model(N, P, B, M)
    replica = np.full((B, M), -1, np.int32)      # a copy kept up to date from the change log only
    buf = np.zeros(3 * (N + 1024), np.int32)
    try:
        for _ in range(400):
            op = rnd.random()
            if op < 0.35:
                slot = rnd.randrange(-1, B + 1)
                length = rnd.choice([0, 1, P - 1, P, P + 1, rnd.randrange(0, M * P + 5)])
                share = rnd.choice([-1, -1, rnd.randrange(-1, B + 1)])
                st_tok = rnd.randrange(-1, length + 2) if share >= 0 else 0
                got = pp.admit(slot, length, share, st_tok, check=False)
                want = m.admit(slot, length, share, st_tok)
            elif op < 0.6:
                q = rnd.choice([0, 1, 1, 1, 4])
                got, want = pp.reserve(q, check=False), m.reserve(q)
            elif op < 0.8:
                q = rnd.choice([0, 1, 1, 1, 4])
                got, want = pp.advance(q, check=False), m.advance(q)
            else:
                slot = rnd.randrange(-1, B + 1)
                got, want = pp.release(slot, check=False), m.release(slot)
            assert got == want
            _agree(pp, m)
            n = pp.take_changes(buf)
            assert n >= 0
            keys = {(int(slot), int(i)) for slot, i, _ in buf[:3 * n].reshape(n, 3)}
            assert len(keys) == n                      # each entry at most once: order-free
            for slot, i, v in buf[:3 * n].reshape(n, 3):
                replica[slot, i] = v
            assert np.array_equal(replica, pp.block_table)
    finally:
        pp.close()


def test_change_log_overflow_asks_for_a_full_copy():
    pp = pkv.Pages(8, 16, 4, 4)
    try:
        pp.admit(0, 48)                        # 3 writes
        small = np.zeros(3 * 2, np.int32)
        assert pp.take_changes(small) == -1    # more than 2 triples: copy the whole table
        assert pp.take_changes(small) == 0     # the log starts empty again
    finally:
        pp.close()


def test_shared_prefix_pages_are_never_a_landing_page():
    P = 16
    pp = pkv.Pages(200, P, 4, 64)
    try:
        pp.admit(0, 100)                       # holds a 100-token prefix: 6 full pages + 1
        pp.admit(1, 130, 0, 100)               # shares the 6 full pages
        pp.admit(2, 97, 0, 97)                 # shares 6 full pages, its 97th token is its own
        shared = set(pp.block_table[0, :6])
        assert set(pp.block_table[1, :6]) == shared and set(pp.block_table[2, :6]) == shared
        assert all(pp.refcount[p] == 3 for p in shared)
        for _ in range(300):
            pp.reserve(1)
            for s in range(3):
                L = int(pp.seq_lens[s])
                assert int(pp.block_table[s, L // P]) not in shared   # where the new token lands
            pp.advance(1)
        pp.release(0)
        assert all(pp.refcount[p] == 2 for p in shared)
        pp.release(1)
        pp.release(2)
        assert pp.free_count == 200 and (np.asarray(pp.refcount) == 0).all()
    finally:
        pp.close()


def test_reserve_is_all_or_nothing():
    pp = pkv.Pages(5, 16, 3, 8)
    try:
        assert pp.admit(0, 16) == OK and pp.admit(1, 32) == OK and pp.admit(2, 16) == OK   # 4 pages used
        before = pp.block_table.copy()
        assert pp.reserve(1, check=False) == OOM            # three slots cross a page, one page free
        assert (pp.block_table == before).all() and pp.free_count == 1
        pp.release(2)
        assert pp.reserve(1) == OK and pp.free_count == 0
    finally:
        pp.close()


def test_freed_pages_are_reused_last_in_first_out():
    pp = pkv.Pages(10, 16, 2, 4)
    try:
        pp.admit(0, 48)                        # pages 0, 1, 2
        assert list(pp.block_table[0, :3]) == [0, 1, 2]
        pp.release(0)                          # pushed 0, 1, 2: page 2 on top
        pp.admit(1, 16)
        assert int(pp.block_table[1, 0]) == 2
    finally:
        pp.close()
