"""The bench's roofline arithmetic, on the CPU with made-up timings.

bench.py turns per-class device times into the JSON line's `roofline`
object; these tests fix what that object must say for known inputs: the
algorithmic bytes of one attention launch (one layer's K + V at the profiled
lengths, plus the QKV reduction's bytes that the timed class also covers),
the achieved rate and its fraction of the copy peak, the traffic scaled from
the ncu capture, and the tensor-bound GEMM case.
"""
import os
import sys

import numpy as np
import pytest

import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402

PEAKS = dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, source="fallback")


def test_attention_roofline_from_known_times():
    shape = synth.QWEN3_8B
    B, N = 64, 4
    R = 2 * N - 1
    lens = np.full((3, B), 2000)                       # three profiled steps, L = 2000
    per_launch_ms = 0.125
    launches = 36 * 3
    prof = {"attention": (per_launch_ms * launches, launches),
            "gemm_qkv": (0.01 * launches, launches)}
    roof = bench.roofline_entry(prof, shape, B, N, lens, 3, PEAKS)
    kv = B * (2000 + R) * shape.kv_dim * 2 * 2         # one layer's K and V, bf16
    qkv = B * R * shape.qkv_dim * 4 + B * R * (shape.q_dim + 2 * shape.kv_dim) * 2
    assert roof["kernel"] == "attention" and roof["bound"] == "hbm"
    assert roof["kv_bytes"] == pytest.approx(kv)
    assert roof["algorithmic_bytes"] == pytest.approx(kv + qkv)
    achieved = (kv + qkv) / (per_launch_ms * 1e-3) / 1e9
    assert roof["achieved"] == pytest.approx(achieved)
    assert roof["frac"] == pytest.approx(achieved / PEAKS["hbm"])
    assert roof["frac_of_nominal"] == pytest.approx(achieved / 8000.0)
    assert roof["traffic"] == pytest.approx(bench.ATTN_DRAM_PER_KV_BYTE * kv)
    assert roof["launches"] == launches and roof["avg_launch_ms"] == pytest.approx(per_launch_ms)


def test_tensor_bound_gemm_roofline():
    shape = synth.QWEN3_8B
    B, N = 64, 4
    M = B * (2 * N - 1)
    prof = {"gemm_gate_up_silu": (3.5, 36)}
    roof = bench.roofline_entry(prof, shape, B, N, np.full((1, B), 1000), 1, PEAKS)
    flops = 2 * M * shape.hidden * 2 * shape.intermediate
    assert roof["bound"] == "tensor" and roof["unit"] == "TFLOP/s"
    assert roof["achieved"] == pytest.approx(flops / (3.5 / 36 * 1e-3) / 1e12)
    assert roof["frac"] == pytest.approx(roof["achieved"] / PEAKS["bf16_sus"])


def test_weight_streaming_gemm_is_hbm_bound():
    """At batch 1 (7 rows, far below the ~210 flop/byte ridge) a projection
    streams its weights: the roofline is bytes, not flops."""
    shape = synth.QWEN3_8B
    prof = {"gemm_down": (0.97, 36)}
    roof = bench.roofline_entry(prof, shape, 1, 4, np.full((1, 1), 2048), 1, PEAKS)
    wbytes = 2 * shape.intermediate * shape.hidden
    assert roof["bound"] == "hbm"
    assert roof["achieved"] == pytest.approx(wbytes / (0.97 / 36 * 1e-3) / 1e9)


def test_step_bytes_count_weights_kv_and_logits_once():
    shape = synth.QWEN3_8B
    B, N = 2, 4
    R = 2 * N - 1
    w, kv, logits, flops = bench.step_bytes_flops(shape, [100, 300], B, N)
    params = shape.n_layers * shape.params_per_layer() + shape.vocab * shape.hidden
    assert w == 2 * params
    assert kv == (100 + R + 300 + R) * shape.kv_bytes_per_token()
    assert logits == B * R * shape.vocab * 4
    assert flops == pytest.approx(2.0 * B * R * params)


def test_peaks_file_figures_and_fallbacks(tmp_path):
    """The measured peaks are used when the driver's file holds them as plain
    numbers; anything else falls back figure by figure, and `source` says so."""
    f = tmp_path / "peaks.json"
    assert bench.load_peaks(str(tmp_path / "absent.json"))["source"] == "fallback"
    f.write_text('{"hbm_gbs": 6531.3, "bf16_tflops": 1636.3, "bf16_tflops_sustained": 1396.6}')
    p = bench.load_peaks(str(f))
    assert (p["hbm"], p["bf16"], p["bf16_sus"], p["source"]) == (6531.3, 1636.3, 1396.6, "measured")
    f.write_text('{"hbm_gbs": {"burst": 6531.3}, "bf16_tflops": 1636.3, "notes": "x"}')
    p = bench.load_peaks(str(f))
    assert p["hbm"] == bench.FALLBACK_PEAKS["hbm"] and p["bf16"] == 1636.3
    assert p["bf16_sus"] == bench.FALLBACK_PEAKS["bf16_sus"] and "fallback" in p["source"]
    for bad in ("not json", "[1, 2]", '{"hbm_gbs": true}', '{"hbm_gbs": -1}'):
        f.write_text(bad)
        p = bench.load_peaks(str(f))
        assert p["hbm"] == bench.FALLBACK_PEAKS["hbm"] and p["source"].endswith("fallback")
