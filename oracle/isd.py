"""One Introspective Strided Decoding step, per request, in float64.

Oracle (test infrastructure only). The method, as the pages give it:

* one strictly causal forward over a block verifies the previous step's
  drafts and proposes new ones at MASK positions ([wiki] TL;DR, Key claims,
  Method; [blog] "How Introspective Strided Decoding Works");
* the anchor p comes from the current forward, the proposal q from the
  previous one; a draft x is kept when u < min(1, p(x)/q(x)), u ~ U(0,1),
  tested left to right; at the first rejection the block restarts from that
  position ([wiki] Key claims, Method);
* the rule is the speculative-sampling rule, so the rejected slot is refilled
  from the normalised residual max(0, p - q) ([blog] "How ISD Works": it
  keeps the output distribution equal to the AR model's; [wiki] "Why it's
  interesting": the same rule as target-model verification);
* the logit shift: the row at position t scores the token at t + 1 ([wiki]
  TL;DR, Method; [blog] "Introspective Consistency", "Dream shift");
* MASK proposals by argmax are the serving default ([wiki] Key claims (iv)).

Readings fixed here where the pages are silent (each applied below):

R1 block layout: rows [x*, d_1..d_n, MASK x (2N-2-n)] at positions
   L..L+2N-2, where L is the committed length, x* the newest final token
   (KV not yet written) and n in {0, N-1} the number of pending drafts. A
   full step (n = N-1) scores N-1 pending positions and N MASK positions:
   2N-1 queries per forward.
R2 verify: draft d_j is scored by row j-1; accepted iff u_j * q_j(d_j) <
   p_j(d_j) (the multiplication form of u < min(1, p/q), u in [0, 1)).
R3 the one new final token comes from row A (A = number of accepted drafts):
   from max(0, p - q_{A+1}) normalised after a rejection (from p itself when
   that residual sums to 0), from p (the bonus) when all n drafts pass. It
   lands at position L+A+1 and becomes the next x*.
R4 proposals: rows n+1..n+N-1 (the MASK rows after the bonus slot) give the
   next drafts, valid only when no draft was rejected; after a rejection the
   next step is a restart step (n = 0) whose padding rows are ignored.
   The acceptance rule keeps the AR distribution for any proposal, so no
   distribution-level pin can see which MASK row proposes which position;
   it is pinned instead by a predictor that is perfect for a token sequence:
   every proposal must then be the sequence's next token and be accepted,
   giving N tokens per forward, the pages' formula at acceptance 1.
R5 commit: seq_len += 1 + A (x* and the accepted drafts); committed tokens
   this step = accepted drafts + the new token.
R6 sampling: inverse CDF in ascending token order: the smallest i whose
   running sum exceeds u * sum(w); if rounding leaves none, the largest i with
   w_i > 0. Argmax takes the lowest index among equal maxima.
R7 uniform slots per request (2N-1): [0, N-1) accept tests, [N-1] the new
   token, [N, 2N-1) sampled proposals.
R8 greedy verify (temperature 0): accept iff d_j == argmax p_j; the new
   token is argmax of row A.
R9 R-ISD: the gated LoRA delta is applied to MASK rows only (restart padding
   rows included); x* and the pending drafts run on the base weights.
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional, Sequence

import numpy as np

from .model import Decoder, DenseKV, block_forward, commit_kv, prefill


ARGMAX, SAMPLE = "argmax", "sample"      # proposal modes
STOCHASTIC, GREEDY = "sample", "greedy"  # verify modes


def softmax(z: np.ndarray) -> np.ndarray:
    z = np.asarray(z, dtype=np.float64)
    e = np.exp(z - z.max())
    return e / e.sum()


def argmax_lowest(z: np.ndarray) -> int:
    """Index of the maximum; the lowest index among equal maxima (R6)."""
    z = np.asarray(z)
    return int(np.flatnonzero(z == z.max())[0])


def inverse_cdf(w: np.ndarray, u: float):
    """Sample index for weights w with uniform u (R6).

    Returns (index, margin) where margin is the distance of u * sum(w) to the
    nearest CDF boundary of the chosen index, relative to sum(w).
    """
    w = np.asarray(w, dtype=np.float64)
    c = np.cumsum(w)
    total = c[-1]
    t = u * total
    hits = np.flatnonzero(c > t)
    if len(hits):
        i = int(hits[0])
    else:
        i = int(np.flatnonzero(w > 0)[-1])
    lo = c[i - 1] if i > 0 else 0.0
    margin = min(abs(t - lo), abs(c[i] - t)) / total if total > 0 else 0.0
    return i, margin


def residual(p: np.ndarray, q: np.ndarray) -> np.ndarray:
    """max(0, p - q), or p itself when that is identically zero (R3)."""
    r = np.maximum(0.0, p - q)
    return r if r.sum() > 0 else p


def tpf_formula(a: float, n_stride: int) -> float:
    """Memory-bound tokens per forward at per-draft acceptance a, stride N:
    (2 + a + ... + a^(N-2)) / (2 - a^(N-1)) ([wiki] Method; [gn-hi] Speedup
    Factor Explorer)."""
    num = 2.0 + sum(a ** k for k in range(1, n_stride - 1))
    return num / (2.0 - a ** (n_stride - 1))


@dataclasses.dataclass
class RequestState:
    """One request between steps."""
    kv: DenseKV                      # K/V of committed positions 0..L-1
    history: List[int]               # tokens at positions 0..L-1
    x_star: int                      # final token at position L (KV not yet written)
    drafts: List[int]                # pending drafts at L+1..L+n
    q_rows: Optional[List[np.ndarray]] = None   # proposal distributions (SAMPLE mode)

    @property
    def seq_len(self) -> int:
        return self.kv.length

    def copy(self) -> "RequestState":
        return RequestState(self.kv.copy(), list(self.history), self.x_star, list(self.drafts),
                            None if self.q_rows is None else [q.copy() for q in self.q_rows])


@dataclasses.dataclass
class StepResult:
    accepted: int                    # A
    new_token: int
    proposals: List[int]             # next drafts (empty after a rejection)
    committed: List[int]             # accepted drafts + the new token
    logits: np.ndarray               # [2N-1, V] block logits
    accept_margins: List[float]      # |u - p/q| of every accept test performed
    sample_margin: Optional[float]   # boundary distance of the new-token draw
    argmax_gaps: List[float]         # top-2 logit gaps behind argmax decisions
    proposal_margins: List[float]    # boundary distances of sampled proposals


def start_state(m: Decoder, prompt: Sequence[int]) -> RequestState:
    """Prefill the prompt's first P-1 tokens; x* = its last token, no drafts."""
    prompt = [int(t) for t in prompt]
    kv = prefill(m, prompt[:-1])
    return RequestState(kv, prompt[:-1], prompt[-1], [], None)


def _top2_gap(z: np.ndarray) -> float:
    s = np.sort(np.asarray(z, dtype=np.float64))
    return float(s[-1] - s[-2]) if len(s) > 1 else np.inf


@dataclasses.dataclass
class Decision:
    """What one step decides from its block logits (no state change)."""
    accepted: int
    new_token: int
    proposals: List[int]
    q_rows: Optional[List[np.ndarray]]
    accept_margins: List[float]
    sample_margin: Optional[float]
    argmax_gaps: List[float]
    proposal_margins: List[float]


def block_tokens(st: RequestState, n_stride: int, mask_token: int):
    """Input tokens and positions of the block (R1)."""
    R = 2 * n_stride - 1
    n = len(st.drafts)
    if n not in (0, n_stride - 1):
        raise ValueError("pending drafts must be 0 or N-1")
    tokens = [st.x_star] + list(st.drafts) + [mask_token] * (R - 1 - n)
    return tokens, st.seq_len + np.arange(R)


def decide(logits: np.ndarray, drafts: Sequence[int], q_rows, n_stride: int,
           u: Sequence[float], propose: str = ARGMAX, verify: str = STOCHASTIC) -> Decision:
    """Verify the drafts, draw the new token and read the proposals (R2-R4,
    R6-R8) from the block logits [2N-1, V]."""
    N = n_stride
    n = len(drafts)
    if len(u) != 2 * N - 1:
        raise ValueError("expected 2N-1 uniforms")
    A = n
    accept_margins: List[float] = []
    argmax_gaps: List[float] = []
    for j in range(1, n + 1):
        z = logits[j - 1]
        d = int(drafts[j - 1])
        if verify == GREEDY:
            ok = d == argmax_lowest(z)
            argmax_gaps.append(_top2_gap(z))
        else:
            p = softmax(z)
            qd = 1.0 if propose == ARGMAX else float(q_rows[j - 1][d])
            ok = float(u[j - 1]) * qd < p[d]
            accept_margins.append(abs(float(u[j - 1]) - p[d] / qd) if qd > 0 else np.inf)
        if not ok:
            A = j - 1
            break

    z = logits[A]
    sample_margin = None
    if verify == GREEDY:
        new = argmax_lowest(z)
        argmax_gaps.append(_top2_gap(z))
    else:
        p = softmax(z)
        if A < n:
            if propose == ARGMAX:
                q = np.zeros_like(p)
                q[int(drafts[A])] = 1.0
            else:
                q = np.asarray(q_rows[A], dtype=np.float64)
            w = residual(p, q)
        else:
            w = p
        new, sample_margin = inverse_cdf(w, float(u[N - 1]))

    proposals: List[int] = []
    new_q: Optional[List[np.ndarray]] = [] if propose == SAMPLE else None
    proposal_margins: List[float] = []
    if A == n:
        for i in range(1, N):
            zi = logits[n + i]
            if propose == ARGMAX:
                proposals.append(argmax_lowest(zi))
                argmax_gaps.append(_top2_gap(zi))
            else:
                qi = softmax(zi)
                di, mg = inverse_cdf(qi, float(u[N + i - 1]))
                proposals.append(di)
                new_q.append(qi)
                proposal_margins.append(mg)
    return Decision(A, int(new), proposals, new_q if A == n else None, accept_margins,
                    sample_margin, argmax_gaps, proposal_margins)


def step_logits(m: Decoder, st: RequestState, n_stride: int, lora: bool = False):
    """Block forward of one step (R1, R9): (logits, block K, block V)."""
    tokens, positions = block_tokens(st, n_stride, m.shape.mask_token_id)
    n = len(st.drafts)
    lora_rows = (np.arange(len(tokens)) > n) if lora else None
    return block_forward(m, st.kv, tokens, positions, lora_rows, return_kv=True)


def isd_step(m: Decoder, st: RequestState, n_stride: int, u: Sequence[float],
             propose: str = ARGMAX, verify: str = STOCHASTIC, lora: bool = False
             ) -> StepResult:
    """Advance one request by one ISD step; mutates ``st`` in place."""
    logits, bk, bv = step_logits(m, st, n_stride, lora)
    dec = decide(logits, st.drafts, st.q_rows, n_stride, u, propose, verify)
    A = dec.accepted
    committed = list(st.drafts[:A]) + [dec.new_token]                   # R5
    commit_kv(st.kv, bk, bv, A + 1)
    st.history.extend([st.x_star] + list(st.drafts[:A]))
    st.x_star = dec.new_token
    st.drafts = list(dec.proposals)
    st.q_rows = dec.q_rows
    return StepResult(A, dec.new_token, list(dec.proposals), committed, logits,
                      dec.accept_margins, dec.sample_margin, dec.argmax_gaps,
                      dec.proposal_margins)


def ar_decode(m: Decoder, prompt: Sequence[int], n_tokens: int,
              u: Optional[Sequence[float]] = None, greedy: bool = False) -> List[int]:
    """Plain autoregressive decoding of the same model: one row per forward,
    token t+1 drawn from p = softmax(row t) with uniform u[t] (R6), or argmax."""
    st = start_state(m, prompt)
    out = []
    for t in range(n_tokens):
        L = st.seq_len
        logits, bk, bv = block_forward(m, st.kv, [st.x_star], [L], return_kv=True)
        z = logits[0]
        nxt = argmax_lowest(z) if greedy else inverse_cdf(softmax(z), float(u[t]))[0]
        commit_kv(st.kv, bk, bv, 1)
        st.history.append(st.x_star)
        st.x_star = nxt
        out.append(nxt)
    return out
