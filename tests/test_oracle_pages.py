"""Brute-force invariants of the oracle's paged-KV bookkeeping."""
import numpy as np
import pytest

import synth
from oracle import pages as op


def _setup(B, N, P, seed, spare=40, max_pages=32):
    lens = synth.integers(0, 300, (B,), seed, 1)
    R = 2 * N - 1
    need = [op.pages_covering(L + R, P) for L in lens]
    num_pages = int(sum(need)) + spare
    table, free = synth.page_layout(need, num_pages, max_pages, seed)
    return lens, table, free


@pytest.mark.parametrize("seed", range(5))
def test_bookkeep_covers_and_never_shares(seed):
    B, N, P = 9, 4, 16
    lens, table, free = _setup(B, N, P, seed, spare=200, max_pages=64)
    head = 0
    R = 2 * N - 1
    for step in range(6):
        A = synth.integers(0, N, (B,), seed, 10 + step)
        new_len, table2, head2, ok = op.bookkeep(lens, A, table, free, head, N, P)
        assert ok
        assert np.array_equal(new_len, lens + 1 + A)
        # every position a request may touch next step maps to one of its pages
        seen = {}
        for b in range(B):
            for t in range(int(new_len[b]) + R):
                page, slot = op.slot_of(table2, b, t, P)
                assert page >= 0
                assert (page, slot) not in seen, "two (request, position) share a slot"
                seen[(page, slot)] = (b, t)
        # pages handed out are exactly the next free-list entries, in request order
        handed = [int(table2[b, j]) for b in range(B) for j in range(table.shape[1])
                  if table[b, j] < 0 <= table2[b, j]]
        assert handed == list(free[head:head2])
        # pages already held never move
        held = table >= 0
        assert np.array_equal(table2[held], table[held])
        lens, table, head = new_len, table2, head2


def test_bookkeep_exhausted_pool_assigns_nothing():
    N, P = 4, 16
    R = 2 * N - 1
    lens = np.array([P - R, 2 * P - R, 5 * P - R])      # blocks end exactly on a page edge
    need = [op.pages_covering(L + R, P) for L in lens]
    table, _ = synth.page_layout(need, int(sum(need)), 16, 7)
    free = np.array([99, 98], np.int32)                 # three requests need a page each
    A = np.full(3, N - 1)
    new_len, table2, head2, ok = op.bookkeep(lens, A, table, free, 0, N, P)
    assert not ok and head2 == 0 and np.array_equal(table2, table)
    assert np.array_equal(new_len, lens + N)
    free = np.array([99, 98, 97], np.int32)
    _, table3, head3, ok = op.bookkeep(lens, A, table, free, 0, N, P)
    assert ok and head3 == 3
    assert [table3[b, need[b]] for b in range(3)] == [99, 98, 97]


def test_bookkeep_table_row_too_short_assigns_nothing():
    """A request whose next block would need more pages than its page-table
    row holds: no page is handed out to anyone, the free-list head stays,
    lengths still advance and the step reports failure."""
    N, P = 4, 16
    R = 2 * N - 1
    lens = np.array([3 * P - R, P - R])                 # request 0 fills its 3-page row exactly
    need = [op.pages_covering(L + R, P) for L in lens]
    table, _ = synth.page_layout(need, int(sum(need)), 3, 5)
    free = np.arange(40, 50, dtype=np.int32)            # plenty of free pages
    A = np.array([N - 1, 0])
    new_len, table2, head2, ok = op.bookkeep(lens, A, table, free, 0, N, P)
    assert not ok and head2 == 0 and np.array_equal(table2, table)
    assert np.array_equal(new_len, lens + 1 + A)
    # the same step with a 4-page row goes through: request 0 takes its
    # fourth page and request 1 (length 9 + 1, block of 7) its second, in
    # request order
    table4 = np.full((2, 4), -1, np.int64)
    table4[:, :3] = table
    _, table5, head5, ok = op.bookkeep(lens, A, table4, free, 0, N, P)
    assert ok and head5 == 2 and table5[0, 3] == 40 and table5[1, 1] == 41


def test_page_layout_is_a_permutation():
    need = [3, 1, 4, 1, 5]
    table, free = synth.page_layout(need, 30, 8, 3)
    used = table[table >= 0]
    assert sorted(np.concatenate([used, free]).tolist()) == list(range(30))
