"""Work split of the tcgen05 attention kernel, checked on the CPU through the C ABI.

isd_attention_split runs the same split functions the kernel runs on the
device. These are the properties the kernel and its combine rely on:
- every 128-key tile of every (request, KV head) pair is covered exactly once;
- each CTA's segments are contiguous in the (request, head, tile) order;
- a pair cut between CTAs is spread over consecutive CTAs, and part p of it
  lands in slot (request * n_kv + head) * max_parts + p with p < max_parts;
- the ranges are balanced with every segment counted as 2 tiles.
"""
import numpy as np
import pytest

import synth
from strided_verify_propose_b200 import binding as B

TILE_KEYS = 128


def seg_cost(R, nq, nkv):
    """Tiles one segment counts for in the split: 3 for tiles of 32 query
    rows per KV head, 5 for 64."""
    return 5 if R * (nq // nkv) > 32 else 3


def _check(batch, R, nq, nkv, maxp, page, kend, sms):
    r = B.attention_split(batch, R, nq, nkv, 128, maxp, page, kend, sms)
    assert r is not None
    seg, max_parts = r
    ke = np.minimum(np.maximum(np.asarray(kend), 0), maxp * page)
    nt = (ke + TILE_KEYS - 1) // TILE_KEYS
    covered = {}
    order = []
    for c, b, g, t0, ln, slot in seg.tolist():
        assert 0 <= c < sms and 0 <= b < batch and 0 <= g < nkv
        assert ln >= 1 and 0 <= t0 and t0 + ln <= nt[b], (b, g, t0, ln, nt[b])
        for t in range(t0, t0 + ln):
            assert (b, g, t) not in covered, ("tile covered twice", b, g, t)
            covered[(b, g, t)] = (c, slot)
        order.append((c, b, g, t0, ln))
    assert len(covered) == nkv * int(nt.sum()), "a tile is not covered"
    # in CTA order, and contiguous inside one CTA
    last = {}
    for c, b, g, t0, ln in order:
        if c in last:
            pb, pt_end = last[c]
            if pb == b * nkv + g:
                assert t0 == pt_end
            else:
                assert (b * nkv + g) > pb and t0 == 0
                assert pt_end == nt[pb // nkv]   # the previous pair ended inside this CTA
        last[c] = (b * nkv + g, t0 + ln)
    assert [o[0] for o in order] == sorted(o[0] for o in order)
    # parts of a pair: consecutive CTAs, slots in part order
    for b in range(batch):
        for g in range(nkv):
            if nt[b] == 0:
                continue
            ctas = [covered[(b, g, t)][0] for t in range(nt[b])]
            slots = [covered[(b, g, t)][1] for t in range(nt[b])]
            c0 = ctas[0]
            assert ctas == sorted(ctas) and ctas[-1] - c0 + 1 == len(set(ctas))
            for c, s in zip(ctas, slots):
                assert 0 <= c - c0 < max_parts
                assert s == (b * nkv + g) * max_parts + (c - c0)
    # balance: a CTA's tiles plus the overhead of the segments it starts fit
    # in its share of the units
    sc = seg_cost(R, nq, nkv)
    units = nkv * (int(nt.sum()) + sc * batch)
    used = sorted(set(int(c) for c in seg[:, 0]))
    share = -(-units // len(used))
    per_cta = {}
    for c, b, g, t0, ln, _ in seg.tolist():
        tiles, segs = per_cta.get(c, (0, 0))
        per_cta[c] = (tiles + ln, segs + 1)
    for c, (tiles, segs) in per_cta.items():
        assert tiles + sc * (segs - 1) <= share, (c, tiles, segs, share)
    return seg, max_parts


def test_benchmark_shape():
    """Qwen3-8B widths, batch 64, 7 rows per request, prompts U[512, 4096]."""
    lens = synth.prompt_lengths(64, 512, 4096, 7)
    seg, max_parts = _check(64, 7, 32, 8, 66, 64, lens + 7, 148)
    # at this size every SM gets work and most pairs run whole in one CTA
    assert len(set(seg[:, 0].tolist())) == 148
    whole = sum(1 for b in range(64) for g in range(8)
                if ((seg[:, 1] == b) & (seg[:, 2] == g)).sum() == 1)
    assert whole > 300


@pytest.mark.parametrize("seed", range(40))
def test_random_shapes(seed):
    rng = np.random.default_rng(seed)
    batch = int(rng.integers(1, 200))
    nkv = int(rng.choice([1, 2, 4, 8, 16]))
    G = int(rng.choice([1, 2, 4, 8]))
    R = int(rng.integers(1, 32 // G + 1))
    page = 64
    maxp = int(rng.integers(1, 80))
    kend = rng.integers(0, maxp * page + 200, batch)    # some past the table, some empty
    if seed % 5 == 0:
        kend[:] = rng.integers(0, 3, batch)             # almost no keys
    if kend.max() <= 0:
        kend[0] = 1
    sms = int(rng.choice([1, 7, 148]))
    _check(batch, R, nkv * G, nkv, maxp, page, kend, sms)


def test_benchmark_shape_qwen3_32b():
    """Qwen3-32B widths, batch 64, 7 rows per request (56 query rows per KV
    head: tiles of 64 rows, 5 tiles per segment), prompts U[1024, 8192]."""
    lens = synth.prompt_lengths(64, 1024, 8192, 7)
    seg, _ = _check(64, 7, 64, 8, 130, 64, lens + 7, 148)
    assert len(set(seg[:, 0].tolist())) == 148


@pytest.mark.parametrize("seed", range(20))
def test_random_shapes_64_rows(seed):
    """33..64 query rows per KV head (the 64-row tile and its segment cost)."""
    rng = np.random.default_rng(1000 + seed)
    batch = int(rng.integers(1, 120))
    nkv = int(rng.choice([1, 2, 4, 8]))
    G = int(rng.choice([1, 2, 4, 8]))
    R = int(rng.integers(32 // G + 1, 64 // G + 1))
    page = 64
    maxp = int(rng.integers(1, 80))
    kend = rng.integers(0, maxp * page + 200, batch)
    if seed % 5 == 0:
        kend[:] = rng.integers(0, 3, batch)
    if kend.max() <= 0:
        kend[0] = 1
    sms = int(rng.choice([1, 7, 148]))
    assert R * G > 32
    _check(batch, R, nkv * G, nkv, maxp, page, kend, sms)


def test_shapes_not_on_tensor_cores():
    # head_dim 64, 32-key pages and more than 64 query rows per KV head go to
    # the other kernel; 33..64 rows (Qwen3-32B's 8 heads x 7 rows) stay
    assert B.attention_split(4, 7, 32, 8, 64, 10, 64, [100] * 4) is None
    assert B.attention_split(4, 7, 32, 8, 128, 10, 32, [100] * 4) is None
    assert B.attention_split(4, 17, 32, 8, 128, 10, 64, [100] * 4) is None
    assert B.attention_split(4, 7, 64, 8, 128, 10, 64, [100] * 4) is not None
    assert B.attention_split(4, 16, 32, 8, 128, 10, 64, [100] * 4) is not None


def test_bad_arguments():
    with pytest.raises(ValueError):
        B.attention_split(4, 7, 32, 8, 128, 10, 64, [100] * 3)
    with pytest.raises(RuntimeError):
        B.attention_split(4, 7, 30, 8, 128, 10, 64, [100] * 4)   # heads not a multiple
