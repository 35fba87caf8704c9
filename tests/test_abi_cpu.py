"""Host-side checks of the C-ABI library (no GPU needed, no compute calls)."""
import ctypes
import os
import re

import numpy as np
import pytest

import synth
from strided_verify_propose_b200 import binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "isd.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(isd_[a-z0-9_]+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    lib = binding.lib()
    names = _declared_functions()
    assert len(names) >= 12
    for n in names:
        assert hasattr(lib, n), n
    assert set(binding.EXPORTS) == set(names)


def test_struct_layouts_match_header():
    """The ctypes mirrors have the sizes the C compiler gives the structs."""
    # isd_model_cfg: 14 x 4-byte fields
    assert ctypes.sizeof(binding.ModelCfg) == 14 * 4
    # isd_weights: 3 pointers + 8 pointer-to-pointer
    assert ctypes.sizeof(binding.Weights) == 11 * 8
    # isd_batch: 3 ints, pad, 3 pointers
    assert ctypes.sizeof(binding.Batch) == 16 + 3 * 8
    # isd_kv: 5 pointers + 3 ints (+ pad)
    assert ctypes.sizeof(binding.KV) == 5 * 8 + 16
    assert ctypes.sizeof(binding.Lora) == 8 + 14 * 8


def test_last_error_is_callable_without_gpu():
    assert binding.lib().isd_last_error() is not None


def test_gate_up_packing_interleaves_blocks_of_16():
    torch = pytest.importorskip("torch")
    shape = synth.ModelShape(n_layers=1, hidden=128, n_q_heads=2, n_kv_heads=1, head_dim=64,
                             intermediate=192, vocab=256, page_size=16)
    w = synth.decoder_weights(shape, seed=1)
    packed = binding.pack_weights(shape, w, device="cpu")
    gu = packed["layers"][0]["w_gate_up"].float().numpy()
    g, u = w["layers"][0]["w_gate"], w["layers"][0]["w_up"]
    for t in range(shape.intermediate // 16):
        assert np.array_equal(gu[32 * t:32 * t + 16], g[16 * t:16 * t + 16])
        assert np.array_equal(gu[32 * t + 16:32 * t + 32], u[16 * t:16 * t + 16])
    qkv = packed["layers"][0]["w_qkv"].float().numpy()
    assert np.array_equal(qkv[:shape.q_dim], w["layers"][0]["wq"])
    assert np.array_equal(qkv[shape.q_dim + shape.kv_dim:], w["layers"][0]["wv"])
