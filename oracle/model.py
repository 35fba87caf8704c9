"""Qwen3-style decoder forward in float64 (oracle; test infrastructure only).

The pages convert pretrained Qwen3-8B / Qwen3-32B checkpoints ([wiki] TL;DR,
Model Zoo in [gn-hi]); the decoder is therefore the Qwen3 architecture:
pre-norm blocks with RMSNorm, per-head RMSNorm on q and k (QK-norm), NeoX
rotary embedding (rotate-half pairs (i, i + d/2), theta = 1e6), grouped-query
causal softmax attention with scale 1/sqrt(head_dim), SwiGLU MLP, final
RMSNorm and an untied LM head. Strict causal attention over the joint
sequence is what lets the ISD block share the AR KV cache ([wiki] TL;DR,
Method; [blog] "Introspective Consistency").

Each request keeps a dense cache of K and V per layer for its committed
positions; a block of rows is evaluated against that cache plus the earlier
rows of the same block. Rows never interact except through causal attention.
"""
from __future__ import annotations

from typing import Dict, List, Optional, Sequence

import numpy as np


def rms_norm(x: np.ndarray, g: np.ndarray, eps: float) -> np.ndarray:
    """y = x / sqrt(mean(x^2) + eps) * g over the last axis."""
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * g


def silu(x: np.ndarray) -> np.ndarray:
    return x / (1.0 + np.exp(-x))


def rope_neox(x: np.ndarray, pos: np.ndarray, theta: float) -> np.ndarray:
    """Rotate-half rotary embedding at absolute positions.

    x: [rows, heads, d]; pos: [rows]. Pair (i, i + d/2) is rotated by angle
    pos * theta^(-2i/d).
    """
    d = x.shape[-1]
    half = d // 2
    inv_freq = theta ** (-(2.0 * np.arange(half, dtype=np.float64)) / d)
    ang = pos.astype(np.float64)[:, None] * inv_freq[None, :]          # [rows, half]
    c = np.cos(ang)[:, None, :]
    s = np.sin(ang)[:, None, :]
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


class Decoder:
    """fp64 copy of the decoder weights (bf16-exact values from ``synth``)."""

    def __init__(self, shape, weights: Dict[str, object], lora: Optional[List[dict]] = None,
                 lora_scale: float = 1.0):
        f = lambda a: np.asarray(a, dtype=np.float64)
        self.shape = shape
        self.embed = f(weights["embed"])
        self.lm_head = f(weights["lm_head"])
        self.final_norm = f(weights["final_norm"])
        self.layers = [{k: f(v) for k, v in lw.items()} for lw in weights["layers"]]
        self.lora = None
        if lora is not None:
            self.lora = [{t: (f(a), f(b)) for t, (a, b) in ll.items()} for ll in lora]
        self.lora_scale = lora_scale


class DenseKV:
    """Per-request K/V history: per layer arrays [T, n_kv, d] (float64)."""

    def __init__(self, shape):
        self.k = [np.zeros((0, shape.n_kv_heads, shape.head_dim)) for _ in range(shape.n_layers)]
        self.v = [np.zeros((0, shape.n_kv_heads, shape.head_dim)) for _ in range(shape.n_layers)]
        self.n = 0           # committed positions (kept separately so 0 layers works)

    @property
    def length(self) -> int:
        return self.n

    def copy(self) -> "DenseKV":
        c = DenseKV.__new__(DenseKV)
        c.k = [a.copy() for a in self.k]
        c.v = [a.copy() for a in self.v]
        c.n = self.n
        return c


def causal_gqa_attention(q: np.ndarray, K: np.ndarray, V: np.ndarray, q_pos: np.ndarray,
                         k_pos: np.ndarray) -> np.ndarray:
    """Grouped-query causal softmax attention.

    q [R, n_q, d] at positions q_pos; K, V [T, n_kv, d] at positions k_pos.
    Query head h reads KV head h // (n_q / n_kv); row r sees keys with
    k_pos <= q_pos[r]; scores are scaled by 1/sqrt(d). Returns [R, n_q, d]
    (a row with no visible key returns zeros).
    """
    R, n_q, d = q.shape
    G = n_q // K.shape[1]
    att = np.zeros((R, n_q, d))
    scale = 1.0 / np.sqrt(d)
    for r in range(R):
        visible = k_pos <= q_pos[r]
        if not visible.any():
            continue
        for hq in range(n_q):
            g = hq // G
            sc = (K[visible, g, :] @ q[r, hq]) * scale
            w = np.exp(sc - sc.max())
            w /= w.sum()
            att[r, hq] = w @ V[visible, g, :]
    return att


def _proj(m: Decoder, l: int, name: str, wname: str, x: np.ndarray,
          lora_rows: Optional[np.ndarray]) -> np.ndarray:
    """x @ W^T, plus the gated-LoRA delta (x A) B on the rows flagged in
    lora_rows only ([wiki] Method: the rank-128 LoRA is active only at MASK
    positions; verify positions stay on base weights)."""
    y = x @ m.layers[l][wname].T
    if m.lora is not None and lora_rows is not None and lora_rows.any():
        a, b = m.lora[l][name]
        y = y.copy()
        y[lora_rows] = y[lora_rows] + m.lora_scale * ((x[lora_rows] @ a) @ b)
    return y


def block_forward(m: Decoder, kv: DenseKV, tokens: Sequence[int], positions: Sequence[int],
                  lora_rows: Optional[np.ndarray] = None, return_kv: bool = False):
    """Strictly causal forward of a block of rows against a dense KV history.

    Row r (token tokens[r] at absolute position positions[r]) attends to every
    cached position plus block rows r' with positions[r'] <= positions[r].
    Returns logits [rows, vocab]; with return_kv, also the block's own
    per-layer K and V ([rows, n_kv, d]) so the caller can commit a prefix.
    """
    s = m.shape
    tokens = np.asarray(tokens, dtype=np.int64)
    pos = np.asarray(positions, dtype=np.int64)
    R = len(tokens)
    T = kv.length
    key_pos_prefix = np.arange(T, dtype=np.int64)
    x = m.embed[tokens].copy()
    block_k, block_v = [], []
    for l, lw in enumerate(m.layers):
        h = rms_norm(x, lw["attn_norm"], s.rms_eps)
        q = _proj(m, l, "q", "wq", h, lora_rows).reshape(R, s.n_q_heads, s.head_dim)
        k = _proj(m, l, "k", "wk", h, lora_rows).reshape(R, s.n_kv_heads, s.head_dim)
        v = _proj(m, l, "v", "wv", h, lora_rows).reshape(R, s.n_kv_heads, s.head_dim)
        q = rope_neox(rms_norm(q, lw["q_norm"], s.rms_eps), pos, s.rope_theta)
        k = rope_neox(rms_norm(k, lw["k_norm"], s.rms_eps), pos, s.rope_theta)
        block_k.append(k)
        block_v.append(v)
        K = np.concatenate([kv.k[l], k], axis=0)            # [T+R, n_kv, d]
        V = np.concatenate([kv.v[l], v], axis=0)
        kpos = np.concatenate([key_pos_prefix, pos])
        att = causal_gqa_attention(q, K, V, pos, kpos)
        x = x + _proj(m, l, "o", "wo", att.reshape(R, s.q_dim), lora_rows)
        h = rms_norm(x, lw["mlp_norm"], s.rms_eps)
        a = silu(_proj(m, l, "gate", "w_gate", h, lora_rows)) * _proj(m, l, "up", "w_up", h, lora_rows)
        x = x + _proj(m, l, "down", "w_down", a, lora_rows)
    logits = rms_norm(x, m.final_norm, s.rms_eps) @ m.lm_head.T
    if return_kv:
        return logits, block_k, block_v
    return logits


def commit_kv(kv: DenseKV, block_k, block_v, n_rows: int) -> None:
    """Append the first n_rows block rows' K/V to the history."""
    for l in range(len(kv.k)):
        kv.k[l] = np.concatenate([kv.k[l], block_k[l][:n_rows]], axis=0)
        kv.v[l] = np.concatenate([kv.v[l], block_v[l][:n_rows]], axis=0)
    kv.n += n_rows


def prefill(m: Decoder, tokens: Sequence[int]) -> DenseKV:
    """KV history of a token prefix (one causal block over positions 0..T-1)."""
    kv = DenseKV(m.shape)
    if len(tokens) == 0:
        return kv
    _, bk, bv = block_forward(m, kv, tokens, np.arange(len(tokens)), return_kv=True)
    commit_kv(kv, bk, bv, len(tokens))
    return kv
