"""Tile plans of the tcgen05 GEMM, checked on the CPU through the C ABI.

isd_gemm_plan is the host computation the library runs before every
projection launch; these invariants are what the kernel relies on (shared
memory and tensor memory fit, whole swizzle atoms per TMA box, valid UMMA
shapes, no empty K-split, stream-K ranges of at least one tile).
"""
import itertools

import pytest

from strided_verify_propose_b200 import binding as B

K_TILE = 64
MAX_SMEM = 231424 + 1280   # dynamic shared memory the kernel is given, plus alignment slack


def _shapes():
    # Qwen3-8B and Qwen3-32B widths (hidden 4096 / 5120, QKV 6144 / 10240,
    # gate/up 24576 / 51200, down K 12288 / 25600), the adapter's rank 128
    ms = [1, 7, 28, 96, 224, 300, 448, 449, 512, 960, 1024, 4096]
    ns = [128, 256, 384, 1024, 4096, 5120, 6144, 10240, 19072, 24576, 51200, 151936]
    ks = [64, 128, 256, 4096, 5120, 8192, 12288, 25600]
    return list(itertools.product(ms, ns, ks))


@pytest.mark.parametrize("single", [False, True])
def test_plans_satisfy_the_kernel_invariants(single):
    checked = 0
    for m, n, k in _shapes():
        p = B.gemm_plan(m, n, k, single=single, max_splits=8, num_sms=148)
        assert p is not None, (m, n, k)
        kb = k // K_TILE
        tiles = n // 128
        # token columns: every row of the chunk, padded for the UMMA N rules
        assert p["n_pad"] * p["n_chunks"] >= m and p["n_pad"] <= 512
        assert p["n_pad"] % 16 == 0
        assert p["n_mma"] * p["mma_n"] == p["n_pad"] and 16 <= p["mma_n"] <= 256
        assert p["mma_n"] % 16 == 0
        assert p["tmem_cols"] >= p["n_pad"] and p["tmem_cols"] in (32, 64, 128, 256, 512)
        # TMA boxes: whole 8-row swizzle atoms, covering this CTA's token rows
        assert p["box_rows"] % 8 == 0 and p["box_rows"] <= 256
        if p["pair"]:
            assert tiles % 2 == 0 and p["box_rows"] * 2 == p["mma_n"]
            assert p["n_boxes"] == p["n_mma"]
            assert p["n_pad"] > 32          # few tokens: single CTAs
        else:
            assert p["box_rows"] * p["n_boxes"] == p["n_pad"]
        # shared memory: stages of 16 KB weights + this CTA's token rows
        stage = 16384 + p["n_boxes"] * p["box_rows"] * 128
        assert p["stages"] >= 2 and p["stages"] * stage <= p["smem_bytes"] <= MAX_SMEM
        # K-splits: none empty, all K-blocks covered
        s, kbs = p["splits"], p["kb_per_split"]
        assert s * kbs >= kb and (s - 1) * kbs < kb
        if single:
            assert s == 1
        # stream-K: more tiles than one wave, ranges of at least one tile
        if p["streamk"]:
            assert single and p["n_chunks"] == 1 and s == 1
            unit_tiles = tiles // (2 if p["pair"] else 1)
            assert unit_tiles > p["units"] and unit_tiles * kb // p["units"] >= kb
        checked += 1
    assert checked == len(_shapes())


def test_the_step_shapes_plan_as_measured():
    """Qwen3-8B at batch 64, stride 4 (448 rows): the plans the step runs."""
    qkv = B.gemm_plan(448, 6144, 4096)
    assert (qkv["pair"], qkv["splits"], qkv["streamk"]) == (1, 3, 0)
    gate_up = B.gemm_plan(448, 24576, 4096, single=True)
    assert (gate_up["pair"], gate_up["streamk"], gate_up["units"]) == (1, 1, 74)
    lm_head = B.gemm_plan(448, 151936, 4096, single=True)
    assert (lm_head["pair"], lm_head["streamk"], lm_head["units"]) == (0, 1, 148)   # 1187 tiles: odd


def test_the_batch1_shapes_plan_as_measured():
    """Qwen3-8B at batch 1, stride 4 (7 rows): single CTAs (a pair would share
    only a 2 KB token tile per K-block), one wave of K-splits or stream-K."""
    qkv = B.gemm_plan(7, 6144, 4096)
    assert (qkv["pair"], qkv["n_pad"], qkv["splits"]) == (0, 16, 3)
    o = B.gemm_plan(7, 4096, 4096)
    assert (o["pair"], o["splits"]) == (0, 4)
    gate_up = B.gemm_plan(7, 24576, 4096, single=True)
    assert (gate_up["pair"], gate_up["streamk"], gate_up["units"]) == (0, 1, 148)


def test_invalid_shapes_are_refused():
    assert B.gemm_plan(448, 100, 4096) is None      # n not a multiple of 128
    assert B.gemm_plan(448, 128, 100) is None       # k not a multiple of 64
