"""Seeded synthetic inputs for the ISD step.

This module is shared by the CPU oracle, the tests and the benchmark. It
creates inputs only: model shapes, random-init weights, prompts, page
permutations, uniforms and synthetic logits. It holds none of the decoding
arithmetic (no softmax, no acceptance test, no attention, no sampling rule).

All host-side randomness comes from numpy's Philox4x32-10 counter-based bit
generator, keyed by ``(seed, stream id)`` so every tensor has its own
independent stream and the result does not depend on generation order.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional, Sequence

import numpy as np


# ---------------------------------------------------------------- shapes ---

@dataclasses.dataclass(frozen=True)
class ModelShape:
    """Shape of a Qwen3-style decoder (pre-norm, QK-norm, GQA, SwiGLU)."""
    n_layers: int
    hidden: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    intermediate: int
    vocab: int
    rope_theta: float = 1.0e6
    rms_eps: float = 1.0e-6
    page_size: int = 64

    @property
    def mask_token_id(self) -> int:
        # The MASK token is the last vocabulary entry.
        return self.vocab - 1

    @property
    def q_dim(self) -> int:
        return self.n_q_heads * self.head_dim

    @property
    def kv_dim(self) -> int:
        return self.n_kv_heads * self.head_dim

    @property
    def qkv_dim(self) -> int:
        return self.q_dim + 2 * self.kv_dim

    def params_per_layer(self) -> int:
        h, i = self.hidden, self.intermediate
        return h * self.qkv_dim + self.q_dim * h + 3 * h * i

    def kv_bytes_per_token(self) -> int:
        # K and V, all layers, bf16.
        return self.n_layers * 2 * self.kv_dim * 2


# Tiny decoder the CPU oracle runs in seconds.
TINY = ModelShape(n_layers=2, hidden=256, n_q_heads=4, n_kv_heads=2, head_dim=64,
                  intermediate=704, vocab=1024, page_size=16)
# Qwen3-8B widths.
QWEN3_8B = ModelShape(n_layers=36, hidden=4096, n_q_heads=32, n_kv_heads=8, head_dim=128,
                      intermediate=12288, vocab=151936, page_size=64)
# Qwen3-8B widths, two layers: full-width kernels at a depth the oracle can follow.
QWEN3_8B_2L = dataclasses.replace(QWEN3_8B, n_layers=2)
# Qwen3-32B widths.
QWEN3_32B = ModelShape(n_layers=64, hidden=5120, n_q_heads=64, n_kv_heads=8, head_dim=128,
                       intermediate=25600, vocab=151936, page_size=64)
# Qwen3-32B widths, two layers.
QWEN3_32B_2L = dataclasses.replace(QWEN3_32B, n_layers=2)


# --------------------------------------------------------------- streams ---

def rng(seed: int, *stream: int) -> np.random.Generator:
    """Independent Philox4x32-10 stream for (seed, *stream)."""
    ss = np.random.SeedSequence([int(seed) & 0xFFFFFFFF, *[int(s) & 0xFFFFFFFF for s in stream]])
    return np.random.Generator(np.random.Philox(ss))


# Stream ids (arbitrary distinct constants).
_S_EMBED, _S_LMHEAD, _S_LAYER, _S_PROMPT, _S_LEN, _S_PAGES, _S_UNIF, _S_LOGITS, _S_LORA, _S_MISC = \
    101, 102, 1000, 201, 202, 203, 204, 205, 206, 207


# ------------------------------------------------------------- bf16 cast ---

def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even); float32 out."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    b = x.view(np.uint32)
    r = ((b >> 16) & 1) + np.uint32(0x7FFF)
    out = ((b + r) & np.uint32(0xFFFF0000)).astype(np.uint32)
    return out.view(np.float32)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """bfloat16 bit patterns (uint16) of values that are already bf16-exact."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    return (x.view(np.uint32) >> 16).astype(np.uint16)


# ---------------------------------------------------------------- weights ---

def _normal(g: np.random.Generator, shape: Sequence[int], std: float) -> np.ndarray:
    return (g.standard_normal(size=tuple(shape), dtype=np.float32) * np.float32(std))


def decoder_weights(shape: ModelShape, seed: int = 0, std: float = 0.02,
                    layers: Optional[Sequence[int]] = None) -> Dict[str, object]:
    """Random-init decoder weights, N(0, std), rounded once to bf16 values.

    Returned as float32 arrays holding bf16-exact values, in nn.Linear layout
    ([out_features, in_features]). All norm weights are 1.0. ``layers``
    restricts generation to a subset of layer indices (others are omitted).
    """
    h, i, v = shape.hidden, shape.intermediate, shape.vocab
    w: Dict[str, object] = {
        "embed": bf16_round(_normal(rng(seed, _S_EMBED), (v, h), std)),
        "lm_head": bf16_round(_normal(rng(seed, _S_LMHEAD), (v, h), std)),
        "final_norm": np.ones(h, np.float32),
        "layers": [],
    }
    idx = range(shape.n_layers) if layers is None else layers
    for l in idx:
        g = rng(seed, _S_LAYER + l)
        w["layers"].append({
            "attn_norm": np.ones(h, np.float32),
            "wq": bf16_round(_normal(g, (shape.q_dim, h), std)),
            "wk": bf16_round(_normal(g, (shape.kv_dim, h), std)),
            "wv": bf16_round(_normal(g, (shape.kv_dim, h), std)),
            "q_norm": np.ones(shape.head_dim, np.float32),
            "k_norm": np.ones(shape.head_dim, np.float32),
            "wo": bf16_round(_normal(g, (h, shape.q_dim), std)),
            "mlp_norm": np.ones(h, np.float32),
            "w_gate": bf16_round(_normal(g, (i, h), std)),
            "w_up": bf16_round(_normal(g, (i, h), std)),
            "w_down": bf16_round(_normal(g, (h, i), std)),
        })
    return w


LORA_TARGETS = ("q", "k", "v", "o", "gate", "up", "down")


def lora_dims(shape: ModelShape) -> Dict[str, tuple]:
    """(in_features, out_features) of each gated-LoRA target projection."""
    h, i = shape.hidden, shape.intermediate
    return {"q": (h, shape.q_dim), "k": (h, shape.kv_dim), "v": (h, shape.kv_dim),
            "o": (shape.q_dim, h), "gate": (h, i), "up": (h, i), "down": (i, h)}


def lora_weights(shape: ModelShape, rank: int = 128, seed: int = 0, std: float = 0.01
                 ) -> List[Dict[str, tuple]]:
    """Per layer, per target: (A [in, rank], B [rank, out]) bf16-exact float32."""
    out = []
    dims = lora_dims(shape)
    for l in range(shape.n_layers):
        g = rng(seed, _S_LORA, l)
        out.append({t: (bf16_round(_normal(g, (dims[t][0], rank), std)),
                        bf16_round(_normal(g, (rank, dims[t][1]), std))) for t in LORA_TARGETS})
    return out


# ---------------------------------------------------------------- prompts ---

def prompt_lengths(batch: int, lo: int, hi: int, seed: int) -> np.ndarray:
    """Per-request prompt lengths, uniform integers in [lo, hi]."""
    return rng(seed, _S_LEN).integers(lo, hi + 1, size=batch).astype(np.int64)


def prompts(shape: ModelShape, lengths: Sequence[int], seed: int) -> List[np.ndarray]:
    """Uniform random prompt tokens over [0, vocab-1) (the MASK id is excluded)."""
    g = rng(seed, _S_PROMPT)
    return [g.integers(0, shape.vocab - 1, size=int(n)).astype(np.int32) for n in lengths]


# ------------------------------------------------------------------ pages ---

def page_layout(need: Sequence[int], num_pages: int, max_pages_per_req: int, seed: int):
    """Randomly permuted physical pages.

    Request b receives ``need[b]`` pages taken in order from a seeded random
    permutation of [0, num_pages); the rest of the permutation is the free
    list. Returns (page_table [B, max_pages_per_req] int32 padded with -1,
    free_list int32).
    """
    perm = rng(seed, _S_PAGES).permutation(num_pages).astype(np.int32)
    B = len(need)
    table = np.full((B, max_pages_per_req), -1, np.int32)
    off = 0
    for b in range(B):
        k = int(need[b])
        if k > max_pages_per_req:
            raise ValueError("request needs more pages than max_pages_per_req")
        table[b, :k] = perm[off:off + k]
        off += k
    if off > num_pages:
        raise ValueError("page pool too small")
    return table, perm[off:].copy()


# --------------------------------------------------------------- uniforms ---

def uniforms(batch: int, slots: int, seed: int, step: int) -> np.ndarray:
    """Uniforms in [0, 1): the top 24 bits of a Philox word times 2^-24.

    Exactly representable in float32, so both implementations see the same
    values. Shape [batch, slots]; keyed by (seed, step).
    """
    words = rng(seed, _S_UNIF, step).integers(0, 2**32, size=(batch, slots), dtype=np.uint64)
    return ((words >> np.uint64(8)).astype(np.float64) * 2.0**-24).astype(np.float32)


def controlled_uniforms(batch: int, stride_n: int, accept_rate: float, seed: int, step: int
                        ) -> np.ndarray:
    """Uniforms whose accept-test slots force i.i.d. acceptance at a given rate.

    Slots [0, N-1) (the per-draft accept tests) are 0 with probability
    ``accept_rate`` and 1 - 2^-24 otherwise; the remaining slots are ordinary
    uniforms. A zero slot accepts any draft with nonzero probability; the
    other value rejects all but near-certain drafts.
    """
    slots = 2 * stride_n - 1
    u = uniforms(batch, slots, seed, step)
    g = rng(seed, _S_UNIF + 1, step)
    hit = g.random(size=(batch, stride_n - 1)) < accept_rate
    u[:, : stride_n - 1] = np.where(hit, 0.0, 1.0 - 2.0**-24).astype(np.float32)
    return u


# ----------------------------------------------------- synthetic logits ---

def synthetic_logits(rows: int, vocab: int, seed: int, scale: float = 1.0,
                     boost: float = 0.0) -> np.ndarray:
    """float32 logits [rows, vocab], N(0, scale^2), one random token per row
    raised by ``boost`` (so one token carries most of the mass when large)."""
    g = rng(seed, _S_LOGITS)
    z = g.standard_normal(size=(rows, vocab), dtype=np.float32) * np.float32(scale)
    if boost:
        top = g.integers(0, vocab, size=rows)
        z[np.arange(rows), top] += np.float32(boost)
    return z


def perturbed_logits(z: np.ndarray, sigma: float, seed: int) -> np.ndarray:
    """z plus independent N(0, sigma^2) noise (float32)."""
    g = rng(seed, _S_MISC)
    return (z + g.standard_normal(size=z.shape, dtype=np.float32) * np.float32(sigma)).astype(np.float32)


def normal(shape: Sequence[int], seed: int, stream: int, std: float = 1.0) -> np.ndarray:
    """Generic N(0, std^2) float32 tensor on its own stream."""
    return _normal(rng(seed, _S_MISC + 1000 + stream), shape, std)


def integers(lo: int, hi: int, shape: Sequence[int], seed: int, stream: int) -> np.ndarray:
    """Generic uniform integers in [lo, hi) on their own stream."""
    return rng(seed, _S_MISC + 2000 + stream).integers(lo, hi, size=tuple(shape))
