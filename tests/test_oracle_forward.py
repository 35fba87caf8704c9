"""Pins of the oracle's decoder forward to things other than itself.

* An independent implementation of the same architecture: the Qwen3 decoder
  of HF transformers, run in float64 on the same weights (random norm
  weights, so a dropped or misplaced norm weight shows).
* Closed forms of the rotary embedding: identity at position 0, norm
  preservation, and scores that depend only on the relative offset.
* Causality: a block's row logits equal the logits of the same token
  evaluated alone after committing the earlier rows.
"""
import numpy as np
import pytest

import synth
from oracle import model as om

SMALL = synth.ModelShape(n_layers=2, hidden=32, n_q_heads=4, n_kv_heads=2, head_dim=8,
                         intermediate=48, vocab=64, page_size=16)


def _weights(shape, seed=3):
    w = synth.decoder_weights(shape, seed=seed, std=0.2)
    # random (not unit) norm weights so every norm weight is exercised
    k = 0
    def rnd(n):
        nonlocal k
        k += 1
        return 1.0 + synth.normal((n,), seed, 50 + k, std=0.3)
    w["final_norm"] = rnd(shape.hidden)
    for lw in w["layers"]:
        lw["attn_norm"] = rnd(shape.hidden)
        lw["mlp_norm"] = rnd(shape.hidden)
        lw["q_norm"] = rnd(shape.head_dim)
        lw["k_norm"] = rnd(shape.head_dim)
    return w


def _hf_logits(shape, w, tokens):
    torch = pytest.importorskip("torch")
    tr = pytest.importorskip("transformers")
    cfg = tr.Qwen3Config(vocab_size=shape.vocab, hidden_size=shape.hidden,
                         intermediate_size=shape.intermediate, num_hidden_layers=shape.n_layers,
                         num_attention_heads=shape.n_q_heads, num_key_value_heads=shape.n_kv_heads,
                         head_dim=shape.head_dim, rope_theta=shape.rope_theta,
                         rms_norm_eps=shape.rms_eps, tie_word_embeddings=False,
                         attention_bias=False, max_position_embeddings=4096)
    cfg._attn_implementation = "eager"
    m = tr.Qwen3ForCausalLM(cfg).double().eval()
    t = lambda a: torch.tensor(np.asarray(a, dtype=np.float64))
    sd = {"model.embed_tokens.weight": t(w["embed"]), "lm_head.weight": t(w["lm_head"]),
          "model.norm.weight": t(w["final_norm"])}
    for l, lw in enumerate(w["layers"]):
        p = f"model.layers.{l}."
        sd.update({p + "self_attn.q_proj.weight": t(lw["wq"]), p + "self_attn.k_proj.weight": t(lw["wk"]),
                   p + "self_attn.v_proj.weight": t(lw["wv"]), p + "self_attn.o_proj.weight": t(lw["wo"]),
                   p + "self_attn.q_norm.weight": t(lw["q_norm"]), p + "self_attn.k_norm.weight": t(lw["k_norm"]),
                   p + "mlp.gate_proj.weight": t(lw["w_gate"]), p + "mlp.up_proj.weight": t(lw["w_up"]),
                   p + "mlp.down_proj.weight": t(lw["w_down"]),
                   p + "input_layernorm.weight": t(lw["attn_norm"]),
                   p + "post_attention_layernorm.weight": t(lw["mlp_norm"])})
    missing, unexpected = m.load_state_dict(sd, strict=False)
    assert not unexpected and all("rotary" in k for k in missing), (missing, unexpected)
    with torch.no_grad():
        out = m(torch.tensor([list(tokens)])).logits[0].numpy()
    return out


def test_forward_matches_independent_qwen3():
    shape = SMALL
    w = _weights(shape)
    dec = om.Decoder(shape, w)
    tokens = synth.integers(0, shape.vocab, (23,), seed=1, stream=1).tolist()
    ref = _hf_logits(shape, w, tokens)
    # oracle: prefix as a dense cache, then a block of the last 7 rows
    kv = om.prefill(dec, tokens[:16])
    ours = om.block_forward(dec, kv, tokens[16:], np.arange(16, 23))
    full = om.block_forward(dec, om.DenseKV(shape), tokens, np.arange(23))
    # the library normalises in float32 internally, hence the 1e-5 scale
    scale = np.abs(ref).max()
    assert np.abs(full - ref).max() <= 2e-5 * scale
    assert np.abs(ours - ref[16:]).max() <= 2e-5 * scale


def test_rope_closed_forms():
    g = synth.normal((5, 3, 16), 0, 1)
    x = np.asarray(g, dtype=np.float64)
    # identity at position 0
    assert np.array_equal(om.rope_neox(x, np.zeros(5, np.int64), 1e6), x)
    # rotation preserves the norm of each head vector
    pos = np.array([1, 7, 100, 4095, 131071])
    y = om.rope_neox(x, pos, 1e6)
    assert np.allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-13)
    # scores depend only on the offset m - n
    q = x[0:1, 0]
    k = x[1:2, 0]
    s = []
    for m_, n_ in [(10, 3), (107, 100), (5007, 5000)]:
        qm = om.rope_neox(q[:, None, :], np.array([m_]), 1e6)[0, 0]
        kn = om.rope_neox(k[:, None, :], np.array([n_]), 1e6)[0, 0]
        s.append(qm @ kn)
    assert np.allclose(s, s[0], rtol=1e-9)
    # pair (i, i + d/2) at i = 0 rotates by exactly pos radians
    e = np.zeros((1, 1, 16))
    e[0, 0, 0] = 1.0
    r = om.rope_neox(e, np.array([3]), 1e6)[0, 0]
    assert np.isclose(r[0], np.cos(3.0)) and np.isclose(r[8], np.sin(3.0))


def test_rms_norm_closed_form():
    x = np.array([[3.0, 4.0]])
    y = om.rms_norm(x, np.array([1.0, 2.0]), 0.0)
    rms = np.sqrt((9 + 16) / 2)
    assert np.allclose(y, [[3 / rms, 8 / rms]], rtol=1e-15)


def test_rms_norm_matches_the_library_norm_at_large_eps():
    """eps sits inside the root: against the Qwen3 RMSNorm of HF transformers
    (an independent implementation) at an eps large enough to show where it
    is added."""
    torch = pytest.importorskip("torch")
    tr = pytest.importorskip("transformers.models.qwen3.modeling_qwen3")
    x = np.asarray(synth.normal((6, 10), 4, 1), dtype=np.float64) * 0.3
    g = 1.0 + np.asarray(synth.normal((10,), 4, 2), dtype=np.float64) * 0.3
    for eps in (0.0, 0.05, 0.5):
        norm = tr.Qwen3RMSNorm(10, eps=eps).double()
        with torch.no_grad():
            norm.weight.copy_(torch.tensor(g))
            ref = norm(torch.tensor(x)).numpy()
        # the library normalises in float32
        assert np.allclose(om.rms_norm(x, g, eps), ref, rtol=2e-6, atol=0)


def test_block_rows_are_causal():
    shape = SMALL
    dec = om.Decoder(shape, _weights(shape, seed=5))
    tokens = synth.integers(0, shape.vocab, (12,), seed=2, stream=2).tolist()
    kv = om.prefill(dec, tokens[:8])
    blk = om.block_forward(dec, kv, tokens[8:], np.arange(8, 12))
    # same row evaluated alone after committing its predecessors
    kv2 = om.prefill(dec, tokens[:10])
    alone = om.block_forward(dec, kv2, tokens[10:11], [10])
    assert np.allclose(blk[2], alone[0], rtol=0, atol=1e-11)
    # changing a later row leaves earlier rows untouched (bitwise)
    blk2 = om.block_forward(dec, kv, tokens[8:11] + [(tokens[11] + 1) % shape.vocab], np.arange(8, 12))
    assert np.array_equal(blk[:3], blk2[:3])


def test_single_key_attention_returns_value():
    """With one visible key, attention returns that key's V, so a one-token
    model's first row is a deterministic function we can write out."""
    shape = synth.ModelShape(n_layers=1, hidden=16, n_q_heads=2, n_kv_heads=1, head_dim=8,
                             intermediate=8, vocab=8, page_size=16)
    w = _weights(shape, seed=9)
    dec = om.Decoder(shape, w)
    lw = dec.layers[0]
    tok = 5
    x = dec.embed[tok]
    h = om.rms_norm(x, lw["attn_norm"], shape.rms_eps)
    v = h @ lw["wv"].T
    att = np.concatenate([v, v])              # both q-heads share the single kv head
    x2 = x + att @ lw["wo"].T
    h2 = om.rms_norm(x2, lw["mlp_norm"], shape.rms_eps)
    x3 = x2 + (om.silu(h2 @ lw["w_gate"].T) * (h2 @ lw["w_up"].T)) @ lw["w_down"].T
    want = om.rms_norm(x3, dec.final_norm, shape.rms_eps) @ dec.lm_head.T
    got = om.block_forward(dec, om.DenseKV(shape), [tok], [0])[0]
    assert np.allclose(got, want, rtol=0, atol=1e-12)
