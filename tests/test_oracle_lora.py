"""Pins of the oracle's gated LoRA (R-ISD).

The pages: R-ISD adds a rank-128 LoRA gated on at MASK positions only;
verify positions run on the base weights, so the committed output is the
base AR model's bit for bit (Bud's Wiki, "Introspective Diffusion Language
Models", Key claims and Method; GeekNews (hi), "Lossless R-ISD").

Each pin checks the oracle against something other than its own LoRA code:

(a) verify rows bitwise base-only: the block logits of rows 0..n (x* and
    the n pending drafts) with the adapter on are bit-identical to the same
    step without it, in a restart step (n = 0) and in full steps (n = N-1);
    every MASK row changes.
(b) MASK rows equal a model with merged weights: W' = W + s (A B)^T on all
    seven targets, evaluated on the MASK rows against the prefix plus the
    verify rows' base-weight K/V (what a MASK row sees under the gate). The
    merged matrix is a different computation of the same linear map, so a
    wrong orientation, a double scale or a delta on the wrong input shows.
(c) planted mistakes in the oracle (gate including the last verify row or
    x*, A and B swapped, the scale applied twice, a target left without the
    adapter) each fail (a) or (b).
"""
import numpy as np
import pytest

import synth
from oracle import isd as oi
from oracle import model as om

# every projection square (hidden = q width = kv width = intermediate), so a
# swapped A/B is still computable and must be caught by value, not by shape
SQUARE = synth.ModelShape(n_layers=2, hidden=16, n_q_heads=2, n_kv_heads=2, head_dim=8,
                          intermediate=16, vocab=24, page_size=16)
RANK = 4
SCALE = 0.5          # not 1, so a scale applied twice shows


def _models(shape, seed=3):
    w = synth.decoder_weights(shape, seed=seed, std=0.3)
    lw = synth.lora_weights(shape, rank=RANK, seed=seed, std=0.3)
    gated = om.Decoder(shape, w, lora=lw, lora_scale=SCALE)
    base = om.Decoder(shape, w)
    # W' = W + s (A B)^T, nn.Linear layout [out, in]
    names = {"q": "wq", "k": "wk", "v": "wv", "o": "wo", "gate": "w_gate", "up": "w_up",
             "down": "w_down"}
    mw = {k: v for k, v in w.items() if k != "layers"}
    mw["layers"] = []
    for l, layer in enumerate(w["layers"]):
        ml = {k: np.asarray(v, np.float64) for k, v in layer.items()}
        for t, wn in names.items():
            a, b = (np.asarray(x, np.float64) for x in lw[l][t])
            ml[wn] = ml[wn] + SCALE * (a @ b).T
        mw["layers"].append(ml)
    merged = om.Decoder(shape, mw)
    return gated, base, merged


def _states(gated, N, steps=3, seed=5):
    """The states a run passes through: a restart step first, then full steps
    (accept-test uniforms of 0 keep every draft, so each later step is full)."""
    st = oi.start_state(gated, [1, 7, 3, 9, 2, 11])
    out = []
    for s in range(steps):
        out.append(st.copy())
        u = synth.uniforms(1, 2 * N - 1, seed, s)[0].copy()
        u[:N - 1] = 0.0
        oi.isd_step(gated, st, N, u, lora=True)
    return out


def pin_verify_rows_bitwise(gated, states, N):
    for st in states:
        n = len(st.drafts)
        on, _, _ = oi.step_logits(gated, st, N, lora=True)
        off, _, _ = oi.step_logits(gated, st, N, lora=False)
        assert np.array_equal(on[:n + 1], off[:n + 1]), f"verify rows changed (n={n})"
        for r in range(n + 1, 2 * N - 1):
            assert np.abs(on[r] - off[r]).max() > 1e-6, f"MASK row {r} untouched (n={n})"


def pin_mask_rows_merged(gated, base, merged, states, N):
    for st in states:
        n = len(st.drafts)
        on, _, _ = oi.step_logits(gated, st, N, lora=True)
        tokens, pos = oi.block_tokens(st, N, gated.shape.mask_token_id)
        kv = st.kv.copy()
        _, bk, bv = om.block_forward(base, kv, tokens[:n + 1], pos[:n + 1], return_kv=True)
        om.commit_kv(kv, bk, bv, n + 1)
        want = om.block_forward(merged, kv, tokens[n + 1:], pos[n + 1:])
        err = np.abs(on[n + 1:] - want).max()
        assert err <= 1e-12 * max(1.0, np.abs(want).max()), f"MASK rows differ by {err} (n={n})"


@pytest.mark.parametrize("N", [2, 3, 4])
def test_verify_rows_bitwise_base_only(N):
    gated, _, _ = _models(SQUARE)
    states = _states(gated, N)
    assert [len(s.drafts) for s in states] == [0] + [N - 1] * (len(states) - 1)
    pin_verify_rows_bitwise(gated, states, N)


@pytest.mark.parametrize("N", [2, 3, 4])
def test_mask_rows_equal_merged_weight_model(N):
    gated, base, merged = _models(SQUARE)
    pin_mask_rows_merged(gated, base, merged, _states(gated, N), N)


def test_mask_rows_merged_at_uneven_widths():
    """The same identity on a GQA model whose projections are not square
    (orientation of A and B fixed by the shapes alone)."""
    shape = synth.ModelShape(n_layers=2, hidden=24, n_q_heads=4, n_kv_heads=2, head_dim=8,
                             intermediate=40, vocab=30, page_size=16)
    gated, base, merged = _models(shape, seed=8)
    states = _states(gated, 3)
    pin_verify_rows_bitwise(gated, states, 3)
    pin_mask_rows_merged(gated, base, merged, states, 3)


# ------------------------------------------------------ planted mistakes --

def _proj_swapped(m, l, name, wname, x, lora_rows):
    y = x @ m.layers[l][wname].T
    if m.lora is not None and lora_rows is not None and lora_rows.any():
        a, b = m.lora[l][name]
        y = y.copy()
        y[lora_rows] = y[lora_rows] + m.lora_scale * ((x[lora_rows] @ b.T) @ a.T)
    return y


def _proj_scale_twice(m, l, name, wname, x, lora_rows):
    y = x @ m.layers[l][wname].T
    if m.lora is not None and lora_rows is not None and lora_rows.any():
        a, b = m.lora[l][name]
        y = y.copy()
        y[lora_rows] = y[lora_rows] + m.lora_scale * (m.lora_scale * ((x[lora_rows] @ a) @ b))
    return y


def _gate_mutant(include):
    def step_logits(m, st, n_stride, lora=False):
        tokens, positions = oi.block_tokens(st, n_stride, m.shape.mask_token_id)
        n = len(st.drafts)
        rows = np.arange(len(tokens))
        lora_rows = include(rows, n) if lora else None
        return om.block_forward(m, st.kv, tokens, positions, lora_rows, return_kv=True)
    return step_logits


def _proj_skip(target):
    real = om._proj

    def proj(m, l, name, wname, x, lora_rows):
        return real(m, l, name, wname, x, None if name == target else lora_rows)
    return proj


MUTANTS = {
    "gate includes the last verify row": ("step", _gate_mutant(lambda r, n: r >= n)),
    "gate includes x*": ("step", _gate_mutant(lambda r, n: (r > n) | (r == 0))),
    "A and B swapped": ("proj", _proj_swapped),
    "scale applied twice": ("proj", _proj_scale_twice),
    "adapter missing on the down projection": ("proj", _proj_skip("down")),
    "adapter missing on v": ("proj", _proj_skip("v")),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistakes_fail_a_pin(name, monkeypatch):
    kind, fn = MUTANTS[name]
    if kind == "step":
        monkeypatch.setattr(oi, "step_logits", fn)
    else:
        monkeypatch.setattr(om, "_proj", fn)
    N = 3
    gated, base, merged = _models(SQUARE)
    failed = []
    try:
        states = _states(gated, N)
    except AssertionError:
        failed.append("run")
        states = []
    for pin in (lambda: pin_verify_rows_bitwise(gated, states, N),
                lambda: pin_mask_rows_merged(gated, base, merged, states, N)):
        try:
            pin()
        except AssertionError:
            failed.append(pin)
    assert failed, f"planted mistake '{name}' passed every pin"
