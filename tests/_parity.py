"""Comparison rules shared by the GPU parity tests.

The CUDA path computes in fp32 with bf16 operands, the oracle in fp64, so
their logits differ by rounding. Every decision of a step (accept test,
inverse-CDF draw, argmax) is classified before it is compared:

* the expected value is always the oracle's, from its own trajectory;
* the same decision is recomputed here in fp64 from the CUDA path's logits
  (and its stored q rows) only to see whether the logit difference moves it.
  When both logit sets give the same outcome, clear of fp32 rounding, the
  CUDA path must reproduce the oracle's value exactly;
* otherwise the decision is "near": the CUDA path's value must still be a
  correct decision for its own logits (validity), and the trajectories may
  part there;
* accept tests within 1e-3 of the ratio p/q are always "near" (the
  tolerance the method's accuracy statement sets), except u = 0, which
  accepts any draft of nonzero probability whatever the rounding.

Logits are compared element-wise against LOGIT_TOL scaled by the logit
spread (logit_tolerance below).
"""
from __future__ import annotations

import numpy as np

ACCEPT_BAR = 1e-3      # |u - p/q| below this: the accept decision may differ
FP32_REL = 1e-5        # relative rounding band of the kernel's own fp32 sums
LOGIT_TOL = 2e-2       # max-abs logit tolerance at the tiny decoder's logit scale
TINY_LOGIT_STD = 0.32  # logit standard deviation of the tiny decoder (N(0, 0.02) weights)


def logit_tolerance(oracle_logits: np.ndarray) -> float:
    """2e-2 at the tiny decoder's logit spread, scaled with the spread of
    wider models: the bf16 rounding of every GEMM input grows with the
    activations, which grow with the logit spread (an fp64 emulation of the
    kernels' rounding points gives 5.5e-2 at Qwen3-8B widths after two
    layers, against 8e-2 here)."""
    return LOGIT_TOL * max(1.0, float(np.std(oracle_logits)) / TINY_LOGIT_STD)


def _softmax(z):
    z = np.asarray(z, dtype=np.float64)
    e = np.exp(z - z.max())
    return e / e.sum()


def _cdf_draw(w, u):
    """(index, relative margin) of the inverse-CDF draw of weights w at u.
    u = 0 picks the first token of nonzero weight in any precision: no
    rounding can move that draw (margin inf)."""
    w = np.asarray(w, dtype=np.float64)
    if u == 0.0:
        return int(np.flatnonzero(w > 0)[0]), np.inf
    c = np.cumsum(w)
    total = c[-1]
    t = u * total
    hits = np.flatnonzero(c > t)
    i = int(hits[0]) if len(hits) else int(np.flatnonzero(w > 0)[-1])
    lo = c[i - 1] if i > 0 else 0.0
    return i, (min(t - lo, c[i] - t) / total if total > 0 else 0.0)


def _weights(z, q_row, excluded):
    p = _softmax(z)
    if q_row is not None:
        r = np.maximum(0.0, p - np.asarray(q_row, dtype=np.float64))
        return r if r.sum() > 0 else p
    if excluded >= 0:
        r = p.copy()
        r[excluded] = 0.0
        return r if r.sum() > 0 else p
    return p


def draw_is_valid(w, u, token, eps_rel):
    """token is a legal inverse-CDF draw of weights w at u, up to eps_rel * sum(w)."""
    w = np.asarray(w, dtype=np.float64)
    c = np.cumsum(w)
    t = u * c[-1]
    eps = eps_rel * c[-1]
    lo = c[token - 1] if token > 0 else 0.0
    return w[token] > 0 and lo - eps <= t < c[token] + eps


def _argmax(z):
    z = np.asarray(z)
    return int(np.flatnonzero(z == z.max())[0])


# decision kinds the near cases are counted by
KINDS = ("accept", "argmax", "draw")


class Outcome:
    """What the comparison of one request-step found: per decision kind, the
    decisions examined and how many of them fell inside the error band."""

    def __init__(self):
        self.clear = True          # every decision clear of the error band
        self.accept_clear = True   # the accept tests were (A compared exactly)
        self.notes = []
        self.decisions = {k: 0 for k in KINDS}
        self.near_kinds = {k: 0 for k in KINDS}

    def seen(self, kind):
        self.decisions[kind] += 1

    def near(self, kind, what):
        self.clear = False
        self.near_kinds[kind] += 1
        self.notes.append(what)


class Report:
    """Counts over a whole run: request-steps compared and compared exactly,
    requests that left the comparison after a near decision went the other
    way, and per decision kind the decisions examined and the near ones."""

    def __init__(self, label):
        self.label = label
        self.request_steps = 0
        self.exact = 0
        self.dropped = 0
        self.decisions = {k: 0 for k in KINDS}
        self.near = {k: 0 for k in KINDS}
        self.max_dz = 0.0
        self.tol = 0.0

    def add(self, out):
        self.request_steps += 1
        self.exact += 1 if out.clear else 0
        for k in KINDS:
            self.decisions[k] += out.decisions[k]
            self.near[k] += out.near_kinds[k]

    def near_fraction(self, kind):
        return self.near[kind] / self.decisions[kind] if self.decisions[kind] else 0.0

    def line(self):
        parts = [f"{k} {self.near[k]}/{self.decisions[k]} near" for k in KINDS]
        return (f"parity[{self.label}]: {self.exact}/{self.request_steps} request-steps exact, "
                f"{self.dropped} requests parted; " + ", ".join(parts) +
                f"; max |dz| {self.max_dz:.3g} (bar {self.tol:.3g})")

    def check(self, max_near, min_request_steps=1):
        """Upper bounds on the near fraction of each decision kind."""
        assert self.request_steps >= min_request_steps, self.line()
        for k, bound in max_near.items():
            assert self.near_fraction(k) <= bound, (k, self.line())


def compare_decision(dec, gpu_A, gpu_new, gpu_props, lo, lg, drafts, q_o, q_g, u, N, propose,
                     verify):
    """Check one request's step.

    dec: the oracle's decision (accepted, new_token, proposals); lo / lg: the
    oracle's and the CUDA path's block logits [2N-1, V]; q_o / q_g: each
    side's proposal rows of the pending drafts (SAMPLE mode) or None.
    Returns an Outcome; raises AssertionError on a real mismatch.
    """
    out = Outcome()
    n = len(drafts)
    sample_prop = propose == "sample"
    greedy = verify == "greedy"
    # ---- accept tests, left to right
    A_g_expected = None
    for j in range(n):
        d = drafts[j]
        if greedy:
            out.seen("argmax")
            ok_o = d == _argmax(lo[j])
            ok_g = d == _argmax(lg[j])
            if ok_o != ok_g:
                out.near("argmax", f"greedy test {j}")
                A_g_expected = None
                break
        else:
            p_o, p_g = _softmax(lo[j])[d], _softmax(lg[j])[d]
            qd_o = 1.0 if not sample_prop else float(q_o[j][d])
            qd_g = 1.0 if not sample_prop else float(q_g[j][d])
            r_o = p_o / qd_o if qd_o > 0 else np.inf
            r_g = p_g / qd_g if qd_g > 0 else np.inf
            ok_o, ok_g = u[j] < r_o, u[j] < r_g
            out.seen("accept")
            # u = 0 accepts any draft of nonzero probability in any precision
            # (u q < p is 0 < p): no rounding can move that decision
            certain = u[j] == 0.0 and p_o > 0 and p_g > 0
            if not certain and (abs(u[j] - r_o) < ACCEPT_BAR or ok_o != ok_g
                                or abs(u[j] - r_g) < FP32_REL * max(r_g, 1e-30)):
                out.near("accept", f"accept test {j}")
                break
        if not ok_o:
            break
    if not out.clear:
        out.accept_clear = False
        return out
    assert gpu_A == dec.accepted, f"accepted {gpu_A} vs oracle {dec.accepted}"
    A = dec.accepted
    # ---- the new token from row A
    if greedy:
        out.seen("argmax")
        t_o, t_g = _argmax(lo[A]), _argmax(lg[A])
        assert gpu_new == t_g, "greedy new token is not the argmax of the kernel's logits"
        if t_o == t_g:
            assert gpu_new == dec.new_token
        else:
            out.near("argmax", "greedy new token")
    else:
        exc = drafts[A] if (A < n and not sample_prop) else -1
        w_o = _weights(lo[A], q_o[A] if (A < n and sample_prop) else None, exc)
        w_g = _weights(lg[A], q_g[A] if (A < n and sample_prop) else None, exc)
        out.seen("draw")
        t_o, m_o = _cdf_draw(w_o, u[N - 1])
        t_g, m_g = _cdf_draw(w_g, u[N - 1])
        assert t_o == dec.new_token
        if m_g >= FP32_REL:
            assert gpu_new == t_g, f"new token {gpu_new} is not the kernel logits' draw {t_g}"
        else:
            assert draw_is_valid(w_g, u[N - 1], gpu_new, FP32_REL), "new token outside the band"
        if t_o == t_g and m_g >= FP32_REL:
            assert gpu_new == dec.new_token
        else:
            out.near("draw", "new-token draw")
    # ---- proposals (rows n+1..n+N-1), only after no rejection
    if A == n:
        for i in range(1, N):
            r = n + i
            if not sample_prop:
                out.seen("argmax")
                a_o, a_g = _argmax(lo[r]), _argmax(lg[r])
                assert gpu_props[i - 1] == a_g, "argmax proposal is not the kernel logits' argmax"
                if a_o == a_g:
                    assert gpu_props[i - 1] == dec.proposals[i - 1]
                else:
                    out.near("argmax", f"argmax proposal {i}")
            else:
                out.seen("draw")
                t_o, _ = _cdf_draw(_softmax(lo[r]), u[N + i - 1])
                t_g, m_g = _cdf_draw(_softmax(lg[r]), u[N + i - 1])
                if m_g >= FP32_REL:
                    assert gpu_props[i - 1] == t_g
                else:
                    assert draw_is_valid(_softmax(lg[r]), u[N + i - 1], gpu_props[i - 1], FP32_REL)
                if t_o == t_g and m_g >= FP32_REL:
                    assert gpu_props[i - 1] == dec.proposals[i - 1]
                else:
                    out.near("draw", f"sampled proposal {i}")
    return out
