"""End-to-end GPU parity of whole ISD steps against the oracle.

Both sides start from the same seeded weights, prompts, page layout and
uniforms and run their own trajectories; nothing computed by the CUDA path
is fed to the oracle. Per step and per request the test compares the block
logits (max-abs <= 2e-2), the accept decisions, the new token, the next
drafts, the committed tokens and the lengths; page tables are compared
bit-exactly while every request is still in step. A request whose
trajectory reaches a decision inside the numerical error bound (see
tests/_parity.py) is checked for validity and then left out of the
comparison from the next step on. Near decisions are counted per kind
(accept test, argmax, inverse-CDF draw), printed as one "parity[...]" line
per run, and bounded from above per test.
"""
import numpy as np
import pytest

import synth
from oracle import isd as oi
from oracle import model as om
from oracle import pages as op
from tests import _parity

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")



# Oracle models and start states are reused across tests of one session:
# generating Qwen3-8B-width weights and prefilling 64 prompts in fp64 takes
# minutes, and both are fixed by (shape, seed, prompt).
_ORACLE = {}


def _oracle_decoder(shape, seed, lora_std=None):
    key = ("dec", shape, seed)
    if key not in _ORACLE:
        w = synth.decoder_weights(shape, seed=seed)
        _ORACLE[key] = (w, om.Decoder(shape, w))
    w, dec = _ORACLE[key]
    if lora_std is None:
        return w, dec, None
    lkey = ("lora", shape, seed, lora_std)
    if lkey not in _ORACLE:
        lw = synth.lora_weights(shape, rank=128, seed=seed, std=lora_std)
        # the same fp64 base arrays (no copy) plus the adapter
        base = {"embed": dec.embed, "lm_head": dec.lm_head, "final_norm": dec.final_norm,
                "layers": dec.layers}
        _ORACLE[lkey] = (lw, om.Decoder(shape, base, lora=lw))
    lw, ldec = _ORACLE[lkey]
    return w, ldec, lw


def _start_state(dec, shape, seed, prompt):
    key = ("start", shape, seed, prompt.tobytes())
    if key not in _ORACLE:
        _ORACLE[key] = oi.start_state(dec, prompt)
    return _ORACLE[key].copy()


def run_pair(shape, Bn, N, steps, propose, verify, seed, len_lo, len_hi, max_near=None,
             useed=None, lora=False, prefill_rows=None, lora_std=0.05, label=None,
             min_request_steps=1, controlled=None, draw_u=None):
    """Run the CUDA path and the oracle side by side from the same inputs and
    compare every step; returns the parity Report (also printed). max_near:
    upper bounds on the near fraction of each decision kind (accept, argmax,
    draw). controlled: an acceptance rate for acceptance-controlled uniforms
    (accept slots 0 or 1 - 2^-24), else plain uniforms. draw_u: a fixed value
    for the new-token slot (0 draws the first token of nonzero weight, a
    decision no rounding can move, which keeps trajectories over flat
    152k-token distributions in step)."""
    from strided_verify_propose_b200 import binding as B
    R = 2 * N - 1
    P = shape.page_size
    V = shape.vocab
    w, dec, lw = _oracle_decoder(shape, seed, lora_std if lora else None)
    lens = synth.prompt_lengths(Bn, len_lo, len_hi, seed)
    prompts = synth.prompts(shape, lens, seed)
    maxp = op.pages_covering(int(lens.max()) + steps * N + R + 1, P) + 1
    need = [op.pages_covering(int(L) - 1 + R, P) for L in lens]
    num_pages = int(sum(need)) + Bn * (op.pages_covering(steps * N, P) + 2)
    table, free = synth.page_layout(need, num_pages, maxp, seed)
    G = shape.n_q_heads // shape.n_kv_heads
    model = B.Model(shape, B.pack_weights(shape, w), max_batch=Bn,
                    max_rows=max(Bn * R, Bn * (prefill_rows or 64 // G)), max_position=maxp * P)
    if lora:
        model.load_lora(lw, rank=128)
    kv = B.KVCache(shape, num_pages, table, free)
    st = B.StepState(Bn, N, V, sample=propose == oi.SAMPLE)
    B.prefill(model, kv, st, prompts)
    torch.cuda.synchronize()
    assert int(st.status.item()) == 0
    states = [_start_state(dec, shape, seed, p) for p in prompts]
    assert np.array_equal(st.seq_len.cpu().numpy(), [s.seq_len for s in states])
    assert np.array_equal(st.pending[:, 0].cpu().numpy(), [s.x_star for s in states])
    flags = (B.PROPOSE_SAMPLE if propose == oi.SAMPLE else 0) | \
            (B.VERIFY_GREEDY if verify == oi.GREEDY else 0) | (B.USE_LORA if lora else 0)
    rep = _parity.Report(label or f"{shape.hidden}w B{Bn} N{N} {propose}/{verify}")
    in_sync = [True] * Bn
    all_sync = True
    o_table, o_head = table.copy(), 0
    logits_buf = torch.empty(Bn * R, V, device="cuda", dtype=torch.float32)
    for s in range(steps):
        us = seed if useed is None else useed
        u = (synth.uniforms(Bn, R, us, s) if controlled is None
             else synth.controlled_uniforms(Bn, N, controlled, us, s))
        if draw_u is not None:
            u[:, N - 1] = draw_u
        q_before = None if st.q_cache is None else st.q_cache.double().cpu().numpy()
        B.step(model, kv, st, torch.from_numpy(u).cuda(), flags, logits_out=logits_buf)
        torch.cuda.synchronize()
        assert int(st.status.item()) == 0
        g_logits = logits_buf.double().cpu().numpy()
        gA = st.accepted.cpu().numpy()
        gp = st.pending.cpu().numpy()
        gc = st.committed.cpu().numpy()
        gl = st.seq_len.cpu().numpy()
        o_acc = []
        o_len_before = np.array([x.seq_len for x in states])
        for b in range(Bn):
            if not in_sync[b]:
                o_acc.append(None)
                continue
            ost = states[b]
            drafts = list(ost.drafts)
            q_o = None if ost.q_rows is None else [q.copy() for q in ost.q_rows]
            q_g = None if q_before is None else [q_before[b, j] for j in range(len(drafts))]
            res = oi.isd_step(dec, ost, N, u[b], propose, verify, lora=lora)
            logits = res.logits
            rows = g_logits[b * R:(b + 1) * R]
            n = len(drafts)
            # the rows whose outputs the method reads (restart padding is ignored)
            used = list(range(R)) if n == N - 1 else list(range(N))
            tol = _parity.logit_tolerance(logits[used])
            rep.tol = max(rep.tol, tol)
            dz = np.abs(rows - logits).max(axis=1)
            for r in used:
                assert dz[r] <= tol, (s, b, r, dz[r], tol)
            rep.max_dz = max(rep.max_dz, float(max(dz[r] for r in used)))
            out = _parity.compare_decision(res, int(gA[b]), int(gp[b, 0]),
                                           [int(t) for t in gp[b, 1:]], logits, rows, drafts,
                                           q_o, q_g, u[b], N, propose, verify)
            rep.add(out)
            same = (int(gA[b]) == res.accepted and list(gc[b, :res.accepted + 1]) == res.committed
                    and int(gp[b, 0]) == res.new_token
                    and [int(t) for t in gp[b, 1:1 + len(res.proposals)]] == res.proposals
                    and int(gl[b]) == ost.seq_len)
            if out.clear:
                assert same
            if not same:
                # a decision inside the error band went the other way: the
                # trajectories part here, so this request is not compared further
                in_sync[b] = False
                all_sync = False
                rep.dropped += 1
                o_acc.append(None)
                continue
            o_acc.append(res.accepted)
        if all_sync:
            new_len, o_table, o_head, ok = op.bookkeep(
                o_len_before, np.array(o_acc), o_table, free, o_head, N, P)
            assert ok
            assert np.array_equal(kv.page_table.cpu().numpy(), o_table)
            assert int(kv.free_head.item()) == o_head
        else:
            # once a request has parted the oracle's page hand-out no longer
            # follows the GPU's; what must still hold at any size: every
            # request covers [0, L + 2N - 1) with valid pages, none shared
            gtab = kv.page_table.cpu().numpy()
            used_pages = []
            for b in range(Bn):
                n_have = op.pages_covering(int(gl[b]) + R, P)
                row = gtab[b, :n_have]
                assert np.all((row >= 0) & (row < num_pages)), (s, b)
                used_pages.extend(row.tolist())
            assert len(used_pages) == len(set(used_pages)), s
    print(rep.line())
    if max_near is not None:
        rep.check(max_near, min_request_steps)
    model.close()
    return rep


def test_tiny_config_sample_mode():
    """The tiny decoder (2 layers, hidden 256, 4/2 heads x 64, vocab 1024,
    page 16) at stride 2, batch 1, a 32-token prompt, 8 steps, sampled
    proposals so every step after the first is a real p/q test."""
    total = _parity.Report("tiny N2 sample, 4 uniform streams")
    for useed in range(4):
        rep = run_pair(synth.TINY, 1, 2, 8, oi.SAMPLE, oi.STOCHASTIC, seed=0, len_lo=32,
                       len_hi=32, useed=100 + useed)
        total.request_steps += rep.request_steps
        total.exact += rep.exact
        for k in _parity.KINDS:
            total.decisions[k] += rep.decisions[k]
            total.near[k] += rep.near[k]
    print(total.line())
    total.check(TINY_NEAR, min_request_steps=8)


# Upper bounds on the near fraction per decision kind. Tiny decoder: logits
# within 5e-3 of the oracle's, vocabulary 1024.
TINY_NEAR = {"accept": 0.02, "argmax": 0.08, "draw": 0.12}


@pytest.mark.parametrize("N,propose,verify", [
    (2, oi.ARGMAX, oi.STOCHASTIC),
    (4, oi.ARGMAX, oi.STOCHASTIC),
    (3, oi.SAMPLE, oi.STOCHASTIC),
    (4, oi.ARGMAX, oi.GREEDY),
    (1, oi.ARGMAX, oi.STOCHASTIC),
])
def test_tiny_batch(N, propose, verify):
    run_pair(synth.TINY, 6, N, 8, propose, verify, seed=N + 10, len_lo=1, len_hi=70,
             max_near=TINY_NEAR, min_request_steps=24)


# Qwen3-8B widths: argmax decisions flip only where the oracle's top-2 logit
# gap is below the kernels' logit error (a few hundredths).
WIDE_NEAR = {"accept": 0.01, "argmax": 0.05}


def test_qwen3_8b_widths_two_layers():
    """Full Qwen3-8B widths (hidden 4096, 32/8 heads x 128, intermediate
    12288, vocab 151936, page 64) with two layers, batch 3, stride 4, greedy
    verification and argmax proposals: every decision is an argmax, so the
    comparison is exact wherever the top-2 gap exceeds the logit error
    (draws over 152k-token flat distributions would always sit inside the
    fp32 rounding band of a CDF boundary)."""
    run_pair(synth.QWEN3_8B_2L, 3, 4, 4, oi.ARGMAX, oi.GREEDY, seed=1, len_lo=20, len_hi=90,
             max_near=WIDE_NEAR, min_request_steps=6)


def test_qwen3_8b_widths_batch64_greedy():
    """The headline batch at Qwen3-8B widths with two layers: 64 requests,
    prompts U[64, 512], randomly permuted pages, 8 steps, stride 4, argmax
    proposals, greedy verification. 448 block rows per step: the gate/up
    GEMM's SiLU epilogue at 448 token columns, the stream-K cut tiles of
    gate/up and the LM head, the tcgen05 attention fed by the QKV
    reduction's page writes and the bookkeeping of 64 requests, all against
    the oracle."""
    run_pair(synth.QWEN3_8B_2L, 64, 4, 8, oi.ARGMAX, oi.GREEDY, seed=2, len_lo=64, len_hi=512,
             max_near=WIDE_NEAR, min_request_steps=256, label="8B-2L B64 N4 argmax/greedy")


def test_qwen3_8b_widths_batch64_stochastic():
    """The same batch with stochastic verification (u < p/q): accept tests
    from acceptance-controlled uniforms (each draft passes with probability
    0.9 through the real p(d) > 0 test, or meets a uniform of 1 - 2^-24),
    and the new-token slot at 0 so the draw lands on the first token of
    nonzero weight (after a rejection the residual excludes the rejected
    draft). Every accept count A in 0..3 occurs, so full and restart steps,
    residual and bonus draws and the page hand-out for uneven advances all
    run at 448 rows."""
    rep = run_pair(synth.QWEN3_8B_2L, 64, 4, 6, oi.ARGMAX, oi.STOCHASTIC, seed=2, len_lo=64,
                   len_hi=512, max_near=WIDE_NEAR, min_request_steps=192, controlled=0.9,
                   draw_u=0.0, label="8B-2L B64 N4 argmax/stochastic")
    assert rep.decisions["accept"] >= 200, rep.line()


def test_qwen3_8b_widths_risd_batch32():
    """R-ISD at Qwen3-8B widths: the rank-128 gated LoRA (A, B ~ N(0, 0.01))
    on the MASK rows of 32 requests, two layers, stride 4, against the
    oracle's LoRA forward (whose gate and merged-weight identity are pinned
    on the CPU). Acceptance-controlled uniforms keep most steps full, so the
    adapter runs on MASK rows next to verify rows in the same GEMMs."""
    run_pair(synth.QWEN3_8B_2L, 32, 4, 5, oi.ARGMAX, oi.STOCHASTIC, seed=2, len_lo=64,
             len_hi=512, max_near=WIDE_NEAR, min_request_steps=96, controlled=0.9, draw_u=0.0,
             lora=True, lora_std=0.01, label="8B-2L R-ISD B32 N4")


@pytest.mark.parametrize("shape_name,Bn,N,verify,len_lo,len_hi", [
    ("TINY", 3, 2, oi.STOCHASTIC, 70, 200),       # 64-row chunks, 2 attention tiles per request
    ("QWEN3_8B_2L", 3, 4, oi.GREEDY, 90, 220),    # 64-row chunks, 4 attention tiles per request
])
def test_prefill_in_large_chunks(shape_name, Bn, N, verify, len_lo, len_hi):
    """Prefill passes of 64 rows per request, whose attention runs as several
    query tiles of the same request (pages shared): the oracle's prefill and
    the following steps must agree as with the small chunks."""
    shape = getattr(synth, shape_name)
    run_pair(shape, Bn, N, 3, oi.ARGMAX, verify, seed=5, len_lo=len_lo, len_hi=len_hi,
             max_near=TINY_NEAR if shape is synth.TINY else WIDE_NEAR, prefill_rows=64)


def test_qwen3_32b_widths_two_layers():
    """Qwen3-32B widths (hidden 5120, 64/8 heads x 128, intermediate 25600,
    vocab 151936) with two layers, batch 6, stride 4, greedy verification:
    eight query heads per KV head, so a request's block has 56 query rows per
    KV head, and the projections and the LM head run at the 32B shapes."""
    run_pair(synth.QWEN3_32B_2L, 6, 4, 3, oi.ARGMAX, oi.GREEDY, seed=3, len_lo=40, len_hi=200,
             max_near=WIDE_NEAR, min_request_steps=12, label="32B-2L B6 N4 argmax/greedy")
