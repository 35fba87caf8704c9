"""The seeded input generators shared by the oracle tests, the GPU tests and
the bench: what they produce is the input recipe the tests and the
benchmark rely on.

* bf16 rounding (every weight both sides use passes through it) equals
  PyTorch's float32 -> bfloat16 conversion, round to nearest even, on random
  values over many magnitudes and on exact ties;
* uniforms lie in [0, 1) on the 2^-24 grid (exact in float32), are fixed by
  (seed, step) and differ between steps;
* acceptance-controlled uniforms put 0 or 1 - 2^-24 in the accept slots,
  0 at the requested rate, and leave the other slots as plain uniforms;
* prompt lengths lie in their range, prompt tokens never use the MASK id.
"""
import numpy as np
import pytest

import synth


def test_bf16_round_matches_the_library_conversion():
    torch = pytest.importorskip("torch")
    g = np.random.default_rng(0)
    x = (g.standard_normal(200_000) * np.exp(g.uniform(-30, 30, 200_000))).astype(np.float32)
    # exact ties: a bf16 value plus half an ulp of bf16, both parities
    base = synth.bf16_round(g.standard_normal(2000).astype(np.float32))
    half = (base.view(np.uint32) & np.uint32(0x7F800000)).view(np.float32) * np.float32(2.0**-8)
    ties = (base + half).astype(np.float32)
    x = np.concatenate([x, ties, np.float32([0.0, -0.0, 1.0, -1.0, 3.0e38, 1e-40])])
    ours = synth.bf16_round(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy()
    assert np.array_equal(ours.view(np.uint32), ref.view(np.uint32))
    assert np.array_equal(synth.bf16_bits(ours), (ref.view(np.uint32) >> 16).astype(np.uint16))


def test_uniforms_are_exact_seeded_and_step_keyed():
    u = synth.uniforms(64, 7, seed=5, step=3)
    assert u.dtype == np.float32 and u.shape == (64, 7)
    assert (u >= 0).all() and (u < 1).all()
    assert np.array_equal(u.astype(np.float64) * 2**24, np.floor(u.astype(np.float64) * 2**24))
    assert np.array_equal(u, synth.uniforms(64, 7, seed=5, step=3))
    assert not np.array_equal(u, synth.uniforms(64, 7, seed=5, step=4))
    assert abs(float(u.mean()) - 0.5) < 0.05


def test_controlled_uniforms_accept_at_the_requested_rate():
    B, N, a = 512, 4, 0.9
    hits = total = 0
    for step in range(8):
        u = synth.controlled_uniforms(B, N, a, seed=1, step=step)
        acc = u[:, :N - 1]
        assert set(np.unique(acc)) <= {np.float32(0.0), np.float32(1.0 - 2.0**-24)}
        hits += int((acc == 0).sum())
        total += acc.size
        assert np.array_equal(u[:, N - 1:], synth.uniforms(B, 2 * N - 1, 1, step)[:, N - 1:])
    sd = np.sqrt(a * (1 - a) / total)
    assert abs(hits / total - a) < 4 * sd


def test_prompts_stay_in_range_and_avoid_the_mask_id():
    lens = synth.prompt_lengths(200, 512, 4096, seed=2)
    assert lens.min() >= 512 and lens.max() <= 4096 and len(set(lens.tolist())) > 100
    ps = synth.prompts(synth.TINY, lens[:20], seed=2)
    assert [len(p) for p in ps] == lens[:20].tolist()
    allp = np.concatenate(ps)
    assert allp.min() >= 0 and allp.max() < synth.TINY.vocab - 1
    assert synth.TINY.mask_token_id == synth.TINY.vocab - 1
