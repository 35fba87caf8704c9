"""The GPU parity tests' comparison rules (tests/_parity.py), on the CPU.

The GPU tests excuse a decision only when rounding can move it; everything
else must match the oracle exactly. Here the oracle's decide() stands in for
both sides on random block logits: a faithful result must pass (and be
counted clear when the two logit sets are equal), any planted mistake in a
clear decision (the accepted count, the new token, a proposal) must raise,
and an accept test placed inside the 1e-3 band of p/q must be counted near
and excused, not failed.
"""
import numpy as np
import pytest

import synth
from oracle import isd as oi
from tests import _parity

V, N = 40, 3
R = 2 * N - 1


def _case(seed, propose, verify):
    rng = np.random.default_rng(seed)
    lo = rng.normal(0.0, 2.0, (R, V))
    q = [oi.softmax(rng.normal(0.0, 2.0, V)) for _ in range(N - 1)] if propose == oi.SAMPLE else None
    # drafts that are often accepted: the argmax of their scoring row, or a
    # random token
    drafts = [int(np.argmax(lo[j])) if rng.random() < 0.7 else int(rng.integers(V))
              for j in range(N - 1)]
    u = synth.uniforms(1, R, seed, 0)[0].astype(np.float64)
    return lo, q, drafts, u


def _compare(dec, gpu, lo, lg, drafts, q, u, propose, verify):
    return _parity.compare_decision(dec, gpu.accepted, gpu.new_token, gpu.proposals, lo, lg, drafts,
                                    q, q, u, N, propose, verify)


MODES = [(oi.ARGMAX, oi.STOCHASTIC), (oi.SAMPLE, oi.STOCHASTIC), (oi.ARGMAX, oi.GREEDY)]


@pytest.mark.parametrize("propose,verify", MODES)
def test_faithful_results_pass_and_planted_mistakes_raise(propose, verify):
    clear = planted = 0
    for seed in range(60):
        lo, q, drafts, u = _case(seed, propose, verify)
        dec = oi.decide(lo, drafts, q, N, u, propose, verify)
        lg = lo.copy()
        out = _compare(dec, dec, lo, lg, drafts, q, u, propose, verify)
        if not out.clear:
            continue
        clear += 1
        A = dec.accepted
        wrong = []
        wrong.append(("A", dict(accepted=(A + 1) % (len(drafts) + 1))))
        wrong.append(("new token", dict(new_token=(dec.new_token + 1) % V)))
        if dec.proposals:
            props = list(dec.proposals)
            props[-1] = (props[-1] + 1) % V
            wrong.append(("proposal", dict(proposals=props)))
        for what, change in wrong:
            bad = oi.Decision(**{**dec.__dict__, **change})
            with pytest.raises(AssertionError):
                _compare(dec, bad, lo, lg, drafts, q, u, propose, verify)
            planted += 1
    assert clear >= 40 and planted >= 2 * clear


def test_rounding_sized_logit_differences_still_compare_exactly():
    """With the CUDA path's logits a few ulp of fp32 away, clear decisions
    are still compared exactly and pass."""
    clear = 0
    for seed in range(60):
        lo, q, drafts, u = _case(seed, oi.ARGMAX, oi.STOCHASTIC)
        lg = lo + np.random.default_rng(seed + 1000).normal(0.0, 1e-6, lo.shape)
        dec = oi.decide(lo, drafts, q, N, u, oi.ARGMAX, oi.STOCHASTIC)
        gpu = oi.decide(lg, drafts, q, N, u, oi.ARGMAX, oi.STOCHASTIC)
        out = _compare(dec, gpu, lo, lg, drafts, q, u, oi.ARGMAX, oi.STOCHASTIC)
        clear += out.clear
    assert clear >= 40


def test_an_accept_test_inside_the_band_is_near_not_failed():
    lo, q, drafts, u = _case(3, oi.ARGMAX, oi.STOCHASTIC)
    p = oi.softmax(lo[0])[drafts[0]]
    u = u.copy()
    u[0] = min(p + 2e-4, 1.0 - 1e-9)          # just above p / q (q = 1): rejected by the oracle
    dec = oi.decide(lo, drafts, q, N, u, oi.ARGMAX, oi.STOCHASTIC)
    assert dec.accepted == 0
    # the other side accepted it (its logits put the ratio just above u)
    gpu = oi.Decision(**{**dec.__dict__, "accepted": 1})
    out = _compare(dec, gpu, lo, lo, drafts, q, u, oi.ARGMAX, oi.STOCHASTIC)
    assert not out.clear and out.near_kinds["accept"] == 1


def test_report_bounds_the_near_fraction():
    rep = _parity.Report("synthetic")
    for k in range(10):
        out = _parity.Outcome()
        out.seen("accept")
        if k < 2:
            out.near("accept", "planted")
        rep.add(out)
    assert rep.near_fraction("accept") == pytest.approx(0.2)
    rep.check({"accept": 0.2})
    with pytest.raises(AssertionError):
        rep.check({"accept": 0.1})
