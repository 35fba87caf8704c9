"""Paged-KV bookkeeping after an ISD step (oracle; test infrastructure only).

The pages' engine keeps SGLang's paged KV cache and continuous batching
unchanged, because attention stays strictly causal ([wiki] TL;DR, Key claims
(i); [blog] "Why Dropping into SGLang Matters"). The pages do not spell out
the bookkeeping; this is the plainest one consistent with them:

* position t of request b lives in physical page page_table[b][t // P], slot
  t % P;
* at the start of a step, request b holds the pages covering positions
  [0, L_b + 2N - 1) (its committed prefix plus the whole block);
* after the step L_b grows by 1 + A_b, and the request receives new pages so
  that it again covers [0, L_b' + 2N - 1);
* new pages come off a free list in ascending request order, request b
  taking the slice that starts at free_head + (exclusive prefix sum of the
  earlier requests' counts); when the list cannot cover all requests no page
  is handed out and an error is reported.
"""
from __future__ import annotations

import numpy as np


def pages_covering(length: int, page_size: int) -> int:
    """Pages that cover positions [0, length)."""
    return -(-int(length) // int(page_size))


def slot_of(page_table: np.ndarray, b: int, t: int, page_size: int):
    """(physical page, slot) holding position t of request b."""
    return int(page_table[b, t // page_size]), t % page_size


def bookkeep(seq_len, accepted, page_table, free_list, free_head: int, stride_n: int,
             page_size: int):
    """Advance lengths and hand out pages after one step.

    Returns (new_seq_len, new_page_table, new_free_head, ok). On failure
    (free list exhausted, or a request outgrowing its page-table row) the
    lengths still advance but no page is assigned and ok is False.
    """
    seq_len = np.asarray(seq_len, dtype=np.int64)
    accepted = np.asarray(accepted, dtype=np.int64)
    table = np.array(page_table, dtype=np.int64, copy=True)
    R = 2 * stride_n - 1
    new_len = seq_len + 1 + accepted
    have = np.array([pages_covering(L + R, page_size) for L in seq_len])
    want = np.array([pages_covering(L + R, page_size) for L in new_len])
    count = want - have
    offsets = np.concatenate([[0], np.cumsum(count)[:-1]]) if len(count) else count
    total = int(count.sum())
    ok = free_head + total <= len(free_list) and bool(np.all(want <= table.shape[1]))
    if not ok:
        return new_len, table, free_head, False
    for b in range(len(seq_len)):
        for j in range(int(count[b])):
            table[b, have[b] + j] = free_list[free_head + offsets[b] + j]
    return new_len, table, free_head + total, True
