"""Pins of the oracle's ISD decision logic and block layout.

Each pin checks the oracle's own code against something the pages or the
mathematics fix, never against a retyped copy of the same formula:

* exact enumeration: the probability of every output token, integrated over
  the uniforms by bisection on the oracle's decision function, equals the
  anchor distribution p (the min(1, p/q) rule with residual resampling keeps
  the AR distribution: [blog] "How ISD Works");
* q == p accepts every draft;
* N = 1 is plain AR decoding, and greedy ISD equals greedy AR for every N
  (verify rows are ordinary causal AR rows: [wiki] TL;DR, Method);
* the layout's long-run tokens per forward equals the pages' formula
  (2 + a + ... + a^(N-2)) / (2 - a^(N-1)) ([wiki] Method), exactly via the
  step's renewal structure and by Monte Carlo through whole steps;
* brute force: the exact distribution of the first committed tokens of a
  multi-step ISD run equals the AR model's.
"""
import itertools

import numpy as np
import pytest

import synth
from oracle import isd as oi
from oracle import model as om

MICRO = synth.ModelShape(n_layers=1, hidden=16, n_q_heads=2, n_kv_heads=1, head_dim=8,
                         intermediate=16, vocab=6, page_size=16)


def _decoder(shape, seed=0, std=0.5):
    return om.Decoder(shape, synth.decoder_weights(shape, seed=seed, std=std))


def _threshold(pred, lo=0.0, hi=1.0, iters=64):
    """For a predicate true on [0, t) and false on [t, 1): t, by bisection."""
    if not pred(lo):
        return 0.0
    if pred(np.nextafter(hi, 0)):
        return 1.0
    for _ in range(iters):
        mid = 0.5 * (lo + hi)
        if pred(mid):
            lo = mid
        else:
            hi = mid
    return 0.5 * (lo + hi)


def _sampler_intervals(tok_of_u, vocab):
    """Measure of u in [0,1) mapped to each token by a monotone sampler."""
    cuts = [0.0]
    for x in range(1, vocab):
        cuts.append(_threshold(lambda u: tok_of_u(u) < x))
    cuts.append(1.0)
    cuts = np.maximum.accumulate(np.array(cuts))
    return np.diff(cuts)


# ------------------------------------------------------------ enumeration --

@pytest.mark.parametrize("propose", [oi.ARGMAX, oi.SAMPLE])
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_accept_resample_reproduces_p_exactly(propose, seed):
    """P(first committed token = x) == p(x) for every x, integrating the
    oracle's decide() over the draft and both uniforms (N = 2)."""
    V = 7
    zp = synth.normal((V,), seed, 1, std=1.5).astype(np.float64)
    zq = synth.normal((V,), seed, 2, std=1.5).astype(np.float64)
    p = oi.softmax(zp)
    logits = np.stack([zp, synth.normal((V,), seed, 3), synth.normal((V,), seed, 4)]).astype(np.float64)
    if propose == oi.ARGMAX:
        drafts_q = [(int(np.argmax(zq)), 1.0, None)]
    else:
        q = oi.softmax(zq)
        drafts_q = [(d, q[d], [q]) for d in range(V)]
    total = np.zeros(V)
    for d, qd, qrows in drafts_q:
        def run(u0, u1):
            return oi.decide(logits, [d], qrows, 2, [u0, u1, 0.5], propose=propose)
        t_acc = _threshold(lambda u0: run(u0, 0.5).accepted == 1)
        total[d] += qd * t_acc
        # rejection branch: resampled token as a function of u1
        u_rej = min(1.0 - 1e-12, t_acc + 0.5 * (1.0 - t_acc))
        if t_acc < 1.0:
            probs = _sampler_intervals(lambda u1: run(u_rej, u1).new_token, V)
            total += qd * (1.0 - t_acc) * probs
    assert np.abs(total - p).max() < 1e-12


@pytest.mark.parametrize("propose", [oi.ARGMAX, oi.SAMPLE])
@pytest.mark.parametrize("seed", [0, 1])
def test_second_draft_reproduces_its_row_exactly(propose, seed):
    """N = 3, first draft accepted: P(the token committed after it = x) ==
    p_1(x), row 1's distribution, integrating decide() over the second
    draft's accept test and the resampling uniform. The two drafts differ,
    so the residual must remove the second draft's proposal mass, not the
    first's."""
    V, N = 7, 3
    z = np.stack([synth.normal((V,), seed, 10 + r, std=1.5) for r in range(2 * N - 1)]).astype(np.float64)
    zq = [synth.normal((V,), seed, 20 + r, std=1.5).astype(np.float64) for r in range(2)]
    p1 = oi.softmax(z[1])
    if propose == oi.ARGMAX:
        d2 = int(np.argmax(zq[1]))
        cases = [((d2 + 1) % V, d2, 1.0, None)]
    else:
        q = [oi.softmax(r) for r in zq]
        cases = [(int(np.argmax(zq[0])), d2, q[1][d2], q) for d2 in range(V)]
    total = np.zeros(V)
    for d1, d2, qd, qrows in cases:
        assert d1 != d2 or propose == oi.SAMPLE

        def run(u1, u2):
            return oi.decide(z, [d1, d2], qrows, N, [0.0, u1, u2, 0.5, 0.5], propose=propose)
        assert run(0.0, 0.5).accepted >= 1                  # u = 0 accepts the first draft
        t_acc = _threshold(lambda u1: run(u1, 0.5).accepted == 2)
        total[d2] += qd * t_acc
        if t_acc < 1.0:
            u_rej = min(1.0 - 1e-12, t_acc + 0.5 * (1.0 - t_acc))
            assert run(u_rej, 0.5).accepted == 1
            total += qd * (1.0 - t_acc) * _sampler_intervals(lambda u2: run(u_rej, u2).new_token, V)
    assert np.abs(total - p1).max() < 1e-12


def test_residual_with_identical_p_q_falls_back_to_p():
    p = oi.softmax(np.array([0.3, -1.0, 2.0]))
    assert np.array_equal(oi.residual(p, p), p)
    r = oi.residual(p, np.array([1.0, 0.0, 0.0]))
    assert r[0] == 0.0 and np.array_equal(r[1:], p[1:])


def test_a_draft_of_probability_zero_is_never_accepted():
    """min(1, p/q) = 0 when p(d) = 0: the draft is rejected for every u in
    [0, 1), u = 0 included, whatever its proposal probability."""
    V, N = 5, 2
    rows = np.array([[0.0, 1.0, -1000.0, 0.5, 0.2],     # p(2) underflows to exactly 0
                     [0.3, 0.1, 0.0, -0.2, 0.4],
                     [0.0, 0.0, 0.0, 0.0, 0.0]])
    assert oi.softmax(rows[0])[2] == 0.0
    q = np.full(V, 0.2)
    for u0 in (0.0, 0.5, 1.0 - 2.0**-53):
        u = [u0, 0.3, 0.6]
        assert oi.decide(rows, [2], None, N, u, propose=oi.ARGMAX).accepted == 0
        assert oi.decide(rows, [2], [q], N, u, propose=oi.SAMPLE).accepted == 0


def test_layout_rejects_draft_and_uniform_counts_outside_it():
    """The block holds 0 or N - 1 pending drafts and a step takes 2N - 1
    uniforms; anything else is refused, not silently padded."""
    m = _decoder(MICRO, seed=2)
    st = oi.start_state(m, [1, 2, 3])
    st.drafts = [4]                                   # 1 draft at N = 3
    with pytest.raises(ValueError):
        oi.block_tokens(st, 3, MICRO.mask_token_id)
    z = np.zeros((5, MICRO.vocab))
    with pytest.raises(ValueError):
        oi.decide(z, [], None, 3, [0.5] * 4)          # 4 uniforms at N = 3


def test_inverse_cdf_rules():
    w = np.array([0.0, 0.25, 0.0, 0.5, 0.25])
    assert oi.inverse_cdf(w, 0.0)[0] == 1
    assert oi.inverse_cdf(w, 0.2499)[0] == 1
    assert oi.inverse_cdf(w, 0.25)[0] == 3          # strict ">" moves past the boundary
    assert oi.inverse_cdf(w, 0.9999)[0] == 4
    # rounding leaves no running sum above the target: the last nonzero weight
    assert oi.inverse_cdf(np.array([0.1, 0.2, 0.0]), 1.0)[0] == 1
    assert oi.argmax_lowest(np.array([1.0, 3.0, 3.0, -2.0])) == 1


# ---------------------------------------------------- special cases (model) --

def _advance(m, prompt, N, steps, seed, propose, verify, u_fn=None):
    st = oi.start_state(m, prompt)
    out = []
    for s in range(steps):
        u = synth.uniforms(1, 2 * N - 1, seed, s)[0] if u_fn is None else u_fn(s)
        r = oi.isd_step(m, st, N, u, propose=propose, verify=verify)
        out.extend(r.committed)
    return out, st


def test_q_equal_p_accepts_every_draft():
    m = _decoder(MICRO, seed=4)
    prompt = [1, 2, 3, 4]
    for N in (2, 3, 4):
        st = oi.start_state(m, prompt)
        oi.isd_step(m, st, N, synth.uniforms(1, 2 * N - 1, 7, 0)[0], propose=oi.SAMPLE)
        for s in range(1, 6):
            assert len(st.drafts) == N - 1
            logits, _, _ = oi.step_logits(m, st, N)
            st.q_rows = [oi.softmax(logits[j]) for j in range(N - 1)]     # q := p
            r = oi.isd_step(m, st, N, synth.uniforms(1, 2 * N - 1, 7, s)[0], propose=oi.SAMPLE)
            assert r.accepted == N - 1


def test_stride_one_is_plain_ar():
    m = _decoder(MICRO, seed=6)
    prompt = [0, 5, 2]
    n_tok = 12
    us = [synth.uniforms(1, 1, 11, s)[0] for s in range(n_tok)]
    isd, _ = _advance(m, prompt, 1, n_tok, 0, oi.ARGMAX, oi.STOCHASTIC, u_fn=lambda s: us[s])
    ar = oi.ar_decode(m, prompt, n_tok, u=[u[0] for u in us])
    assert isd == ar


@pytest.mark.parametrize("N", [2, 3, 4])
def test_greedy_isd_equals_greedy_ar(N):
    m = _decoder(synth.ModelShape(n_layers=2, hidden=32, n_q_heads=4, n_kv_heads=2, head_dim=8,
                                  intermediate=32, vocab=12, page_size=16), seed=8, std=0.6)
    prompt = [3, 1, 4, 1, 5]
    toks, _ = _advance(m, prompt, N, 10, 0, oi.ARGMAX, oi.GREEDY)
    ar = oi.ar_decode(m, prompt, len(toks), greedy=True)
    assert toks == ar


def test_kv_history_matches_committed_tokens():
    """After any run, the dense KV equals a fresh prefill of the committed
    tokens: speculative rows never leak into the history."""
    m = _decoder(MICRO, seed=10)
    toks, st = _advance(m, [1, 2, 3], 3, 6, 5, oi.SAMPLE, oi.STOCHASTIC)
    ref = om.prefill(m, st.history)
    assert st.seq_len == len(st.history)
    for l in range(MICRO.n_layers):
        assert np.allclose(st.kv.k[l], ref.k[l], atol=1e-12)
        assert np.allclose(st.kv.v[l], ref.v[l], atol=1e-12)


# ------------------------------------------------------------------ TPF ----

@pytest.mark.parametrize("N", [2, 3, 4, 5])
def test_layout_tpf_equals_pages_formula_exactly(N):
    """Drive one full step per first-rejection index with forced uniforms,
    read what the oracle commits and where it goes next, and solve the
    resulting two-state renewal process exactly."""
    m = _decoder(MICRO, seed=12)
    a = 0.9
    accept_u, reject_u = 0.0, 1.0 - 2.0**-24
    # a full-step state: one restart step first
    st0 = oi.start_state(m, [1, 2, 3])
    oi.isd_step(m, st0, N, synth.uniforms(1, 2 * N - 1, 3, 0)[0])
    outcomes = []        # (prob, committed, next_is_full) for full steps
    for k in range(N):   # k accepted drafts
        st = st0.copy()
        u = synth.uniforms(1, 2 * N - 1, 3, 1)[0].copy()
        u[: N - 1] = reject_u
        u[:k] = accept_u
        r = oi.isd_step(m, st, N, u)
        assert r.accepted == k
        prob = a ** k * (1 - a) if k < N - 1 else a ** (N - 1)
        outcomes.append((prob, len(r.committed), len(st.drafts) == N - 1))
    # restart step: always commits one token and returns to a full step
    st = oi.start_state(m, [1, 2, 3])
    r = oi.isd_step(m, st, N, synth.uniforms(1, 2 * N - 1, 3, 2)[0])
    assert len(r.committed) == 1 and len(st.drafts) == N - 1
    p_full_to_restart = sum(p for p, _, full in outcomes if not full)
    # stationary chain over {full, restart}
    pi_full = 1.0 / (1.0 + p_full_to_restart)
    pi_restart = 1.0 - pi_full
    tpf = pi_full * sum(p * c for p, c, _ in outcomes) + pi_restart * 1.0
    assert abs(tpf - oi.tpf_formula(a, N)) < 1e-12
    if N == 4:
        assert abs(oi.tpf_formula(0.9, 4) - 2.919) < 1e-3       # pages: ~2.9 / 2.96
        assert abs(oi.tpf_formula(0.9, 4) ** 2 / 7 - 1.22) < 5e-3  # efficiency 1.22


def test_tpf_monte_carlo_through_whole_steps():
    m = _decoder(MICRO, seed=14)
    N, a, steps = 4, 0.9, 1500
    st = oi.start_state(m, [2, 3])
    committed = 0
    for s in range(steps):
        u = synth.controlled_uniforms(1, N, a, 21, s)[0]
        committed += len(oi.isd_step(m, st, N, u).committed)
    tpf = committed / steps
    # std of the per-step commit count is < 1.5; 3 sigma of the mean
    assert abs(tpf - oi.tpf_formula(a, N)) < 3 * 1.5 / np.sqrt(steps)


# ------------------------------------------------------------ brute force --

def _exact_isd_distribution(m, prompt, N, K, propose):
    """Exact distribution of the first K committed tokens: recurse over every
    region of uniform space where the step's outcome is constant."""
    V = m.shape.vocab
    R = 2 * N - 1
    dist = {}

    def explore(st, prob, got):
        if len(got) >= K:
            key = tuple(got[:K])
            dist[key] = dist.get(key, 0.0) + prob
            return
        logits, _, _ = oi.step_logits(m, st, N)
        n = len(st.drafts)
        base = np.full(R, 0.5)

        def dec(u):
            return oi.decide(logits, st.drafts, st.q_rows, N, u, propose=propose)
        # accept thresholds of each draft, given the earlier ones accepted
        thr = []
        for j in range(n):
            def acc(x, j=j):
                u = base.copy()
                u[:j] = [t * 0.5 for t in thr]
                u[j] = x
                return dec(u).accepted > j
            thr.append(_threshold(acc))
        for A in range(n + 1):
            pa = np.prod(thr[:A]) * (1.0 - thr[A] if A < n else 1.0)
            if pa <= 0:
                continue
            u = base.copy()
            u[:A] = [t * 0.5 for t in thr[:A]]
            if A < n:
                u[A] = thr[A] + 0.5 * (1.0 - thr[A])
            def new_of(x, u=u):
                uu = u.copy(); uu[N - 1] = x
                return dec(uu).new_token
            pn = _sampler_intervals(new_of, V)
            for tok in range(V):
                if pn[tok] <= 0:
                    continue
                u2 = u.copy()
                u2[N - 1] = _threshold(lambda x: new_of(x) < tok) + 0.5 * pn[tok]
                if A < n or propose == oi.ARGMAX:
                    branches = [(1.0, u2)]
                else:
                    branches = []
                    per_slot = []
                    for i in range(1, N):
                        def prop_of(x, i=i, u2=u2):
                            uu = u2.copy(); uu[N + i - 1] = x
                            return dec(uu).proposals[i - 1]
                        per_slot.append((_sampler_intervals(prop_of, V), prop_of))
                    for combo in itertools.product(range(V), repeat=N - 1):
                        pc = 1.0
                        u3 = u2.copy()
                        for i, x in enumerate(combo):
                            pi, prop_of = per_slot[i]
                            pc *= pi[x]
                            u3[N + i] = _threshold(lambda y: prop_of(y) < x) + 0.5 * pi[x]
                        if pc > 0:
                            branches.append((pc, u3))
                for pb, ub in branches:
                    st2 = st.copy()
                    r = oi.isd_step(m, st2, N, ub, propose=propose)
                    assert r.accepted == A and r.new_token == tok
                    explore(st2, prob * pa * pn[tok] * pb, got + r.committed)

    explore(oi.start_state(m, prompt), 1.0, [])
    return dist


def _exact_ar_distribution(m, prompt, K):
    V = m.shape.vocab
    dist = {}
    for seq in itertools.product(range(V), repeat=K):
        kv = om.prefill(m, prompt[:-1])
        toks = list(prompt)
        pr = 1.0
        for x in seq:
            z = om.block_forward(m, om.prefill(m, toks[:-1]), [toks[-1]], [len(toks) - 1])[0]
            pr *= oi.softmax(z)[x]
            toks.append(x)
        dist[seq] = pr
    return dist


@pytest.mark.parametrize("N,propose,K", [(2, oi.SAMPLE, 3), (3, oi.SAMPLE, 3), (2, oi.ARGMAX, 3),
                                         (3, oi.ARGMAX, 3)])
def test_isd_trajectory_distribution_equals_ar(N, propose, K):
    shape = synth.ModelShape(n_layers=1, hidden=8, n_q_heads=2, n_kv_heads=1, head_dim=4,
                             intermediate=8, vocab=3, page_size=16)
    m = _decoder(shape, seed=21, std=0.8)
    prompt = [0, 2]
    isd = _exact_isd_distribution(m, prompt, N, K, propose)
    ar = _exact_ar_distribution(m, prompt, K)
    assert abs(sum(isd.values()) - 1.0) < 1e-12
    keys = set(isd) | set(ar)
    err = max(abs(isd.get(k, 0.0) - ar.get(k, 0.0)) for k in keys)
    assert err < 1e-12


def _perfect_predictor_run(monkeypatch, N, shift=0, steps=12, seed=3):
    """Whole oracle steps (greedy verification, argmax proposals) with the
    block logits replaced by those of a predictor that is perfect for a fixed
    token sequence: the row at position t scores seq[t + 1] (the logit shift).
    shift != 0 plants a mistake: the proposals are read from the MASK rows
    `shift` places off. Returns the accepted counts and the committed tokens."""
    shape = synth.TINY
    dec = om.Decoder(shape, synth.decoder_weights(shape, seed=seed))
    rng = np.random.default_rng(seed)
    seq = rng.integers(0, shape.mask_token_id, 64 + steps * (2 * N + 2))
    real_logits, real_decide = oi.step_logits, oi.decide

    def logits_fn(m, st, n_stride, lora=False):
        logits, bk, bv = real_logits(m, st, n_stride, lora)
        R = 2 * n_stride - 1
        z = np.zeros_like(logits)
        z[np.arange(R), seq[st.seq_len + 1 + np.arange(R)]] = 10.0
        return z, bk, bv

    def decide_fn(logits, drafts, q_rows, n_stride, u, propose=oi.ARGMAX, verify=oi.STOCHASTIC):
        d = real_decide(logits, drafts, q_rows, n_stride, u, propose, verify)
        if shift and d.proposals:
            n = len(drafts)
            d.proposals = [oi.argmax_lowest(logits[n + i + shift]) for i in range(1, n_stride)]
        return d

    monkeypatch.setattr(oi, "step_logits", logits_fn)
    monkeypatch.setattr(oi, "decide", decide_fn)
    prompt = seq[:20]
    st = oi.start_state(dec, prompt)  # x* = seq[19] at position L = 19 (KV not yet written)
    assert st.seq_len == 19 and st.x_star == int(seq[19])
    accepted, committed = [], []
    for s in range(steps):
        res = oi.isd_step(dec, st, N, np.zeros(2 * N - 1), oi.ARGMAX, oi.GREEDY)
        accepted.append(res.accepted)
        committed.extend(res.committed)
    return accepted, committed, seq


@pytest.mark.parametrize("N", [2, 3, 4])
def test_a_perfect_predictor_accepts_every_draft(monkeypatch, N):
    """Pins R4 (which MASK row proposes which draft position): with a
    predictor that is perfect for a token sequence, every draft it proposed
    is the sequence's next token, so after the first (restart) step every
    full step accepts all N - 1 drafts and commits N tokens: tokens per
    forward N, the pages' formula at acceptance 1 (tpf_formula(1, N) = N,
    [wiki] Method). The committed stream is the sequence itself."""
    accepted, committed, seq = _perfect_predictor_run(monkeypatch, N)
    assert oi.tpf_formula(1.0, N) == pytest.approx(N)
    assert accepted[0] == 0                          # restart step: nothing pending
    assert all(a == N - 1 for a in accepted[1:])
    assert list(committed) == [int(t) for t in seq[20:20 + len(committed)]]


@pytest.mark.parametrize("shift", [-1, 1])
def test_proposals_read_from_the_wrong_mask_row_are_rejected(monkeypatch, shift):
    """The planted mistake the pin above must catch: proposals read one MASK
    row early or late are not the sequence's next tokens, so full steps
    reject drafts (the committed stream stays the sequence: greedy ISD is
    lossless whatever the proposals)."""
    N = 4
    accepted, committed, seq = _perfect_predictor_run(monkeypatch, N, shift=shift)
    assert any(a < N - 1 for a in accepted[1:])
    assert list(committed) == [int(t) for t in seq[20:20 + len(committed)]]
