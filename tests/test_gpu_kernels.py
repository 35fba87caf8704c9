"""GPU parity of the individual kernels, through the C ABI, against the oracle.

Inputs come from ``synth`` only; expected values from ``oracle`` (or, for
the GEMM, the fp64 product of the same bf16 operands, the definition of the
op). Shapes span several tiles with ragged tails and include the Qwen3-8B
batch-64 / stride-4 launch configuration the benchmark times.
"""
import math

import numpy as np
import pytest

import synth
from oracle import isd as oi
from oracle import model as om
from oracle import pages as op
from tests import _parity

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def _b(B):
    from strided_verify_propose_b200 import binding
    return binding


def _bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to("cuda").to(torch.bfloat16)


# ------------------------------------------------------------------- GEMM ---

@pytest.mark.parametrize("m,n,k,split", [
    (7, 256, 256, 1),          # decode b1 rows (single CTAs: no pairs at <= 32 token columns)
    (7, 384, 256, 1),          # odd tile count: single-CTA MMAs
    (28, 512, 1024, 3),        # ragged split-K
    (300, 384, 640, 1),        # ragged token count, n_pad not a multiple of 32
    (448, 1024, 512, 2),       # b64 x stride 4 rows, two MMAs per k-step
    (448, 1152, 1024, 1),      # the same rows over an odd tile count
    (96, 512, 256, 1),         # one MMA of 96 tokens split 48 / 48 over a pair
    (1000, 256, 256, 1),       # two token chunks (prefill chunk)
    (448, 6144, 4096, 3),      # Qwen3-8B QKV at b64, split 3
    (448, 4096, 12288, 4),     # Qwen3-8B down projection at b64
])
def test_gemm_matches_fp64_product(cuda_lib, m, n, k, split):
    B = _b(0)
    x = synth.bf16_round(synth.normal((m, k), 1, 1))
    w = synth.bf16_round(synth.normal((n, k), 1, 2, std=0.02))
    st = torch.zeros(1, device="cuda", dtype=torch.int32)
    y = B.gemm_bf16(_bf16(w), _bf16(x), split, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    got = y.double().sum(0).cpu().numpy()
    ref = x.astype(np.float64) @ w.astype(np.float64).T
    err = np.abs(got - ref).max()
    assert err <= 2e-4 * np.abs(ref).max(), err


@pytest.mark.parametrize("m,n,k", [
    (448, 19072, 256),         # 149 single-CTA tiles on 148 SMs: stream-K, cut tiles
    (448, 20480, 512),         # 80 pair tiles on 74 pairs: stream-K with 2-SM MMAs
    (7, 19072, 256),           # decode b1 rows through the same split
    (300, 2048, 256),          # fewer tiles than SMs: plain single slice
])
def test_gemm_single_slice_streamk(cuda_lib, m, n, k):
    """Stream-K parity with the fp64 product, and bitwise equal on a repeat
    (the cut tiles' fixups must not depend on which part finishes first)."""
    B = _b(0)
    x = synth.bf16_round(synth.normal((m, k), 3, 1))
    w = synth.bf16_round(synth.normal((n, k), 3, 2, std=0.02))
    wd, xd = _bf16(w), _bf16(x)
    ws = B.gemm_workspace(m, n, k)
    st = torch.zeros(1, device="cuda", dtype=torch.int32)
    y1 = B.gemm_bf16_single(wd, xd, ws, status=st)
    y2 = B.gemm_bf16_single(wd, xd, ws, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert torch.equal(y1, y2)
    if ws is not None:
        assert int(ws[:4096].count_nonzero().item()) == 0   # sync words left at zero
    got = y1.double().cpu().numpy()
    ref = x.astype(np.float64) @ w.astype(np.float64).T
    err = np.abs(got - ref).max()
    assert err <= 2e-4 * np.abs(ref).max(), err


# -------------------------------------------------------------- attention ---

def _attention_case(shape_args, lens, R, seed, pad_row=False):
    B_ = _b(0)
    hd, nq, nkv, P = shape_args
    Bn = len(lens)
    need = [op.pages_covering(L + R, P) for L in lens]
    maxp = max(need) + 2
    num_pages = int(sum(need)) + 5
    table, _ = synth.page_layout(need, num_pages, maxp, seed)
    pool_shape = (1, num_pages, nkv, P, hd)
    kp = synth.bf16_round(synth.normal(pool_shape, seed, 10))
    vp = synth.bf16_round(synth.normal(pool_shape, seed, 11))
    q = synth.bf16_round(synth.normal((Bn * R, nq, hd), seed, 12, std=2.0))
    pos = np.array([L + r for L in lens for r in range(R)], np.int32)
    if pad_row:
        pos[R - 1] = -1
    st = torch.zeros(1, device="cuda", dtype=torch.int32)
    out = B_.paged_attention(_bf16(q).view(Bn * R, nq, hd), torch.from_numpy(pos).cuda(),
                             _bf16(kp).view(pool_shape), _bf16(vp).view(pool_shape),
                             torch.from_numpy(table).cuda(), R, 0, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    got = out.float().cpu().numpy().reshape(Bn * R, nq, hd)
    return got, q, kp, vp, table, pos


def _oracle_attention(q, kp, vp, table, pos, lens, R, P, b):
    T = max(int(pos[b * R + r]) + 1 for r in range(R))
    T = max(T, 0)
    K = np.zeros((T, kp.shape[2], kp.shape[4]))
    V = np.zeros_like(K)
    for t in range(T):
        page, slot = op.slot_of(table, b, t, P)
        K[t] = kp[0, page, :, slot]
        V[t] = vp[0, page, :, slot]
    return om.causal_gqa_attention(q[b * R:(b + 1) * R].astype(np.float64), K, V,
                                   pos[b * R:(b + 1) * R], np.arange(T))


@pytest.mark.parametrize("shape_args,lens,R,pad", [
    ((64, 4, 2, 16), [0, 5, 17, 100], 3, False),           # tiny model, stride 2
    ((128, 32, 8, 64), [1, 63, 64, 700, 2100], 7, False),  # Qwen3-8B, stride 4, several splits
    ((128, 32, 8, 64), [130, 257], 16, False),              # prefill chunk: 64 query rows
    ((128, 8, 1, 64), [40, 300], 8, True),                  # 8:1 grouping, a row with no keys
    ((128, 16, 16, 32), [90, 33], 5, False),                # multi-head (1:1), page 32
    ((128, 8, 1, 64), [200, 5], 4, True),                   # 8:1, 32 rows, a row with no keys
    ((128, 16, 4, 64), [0, 127, 128, 129, 1000], 5, False),  # tile and page edges, 20 rows
])
def test_paged_attention_matches_oracle(cuda_lib, shape_args, lens, R, pad):
    hd, nq, nkv, P = shape_args
    got, q, kp, vp, table, pos = _attention_case(shape_args, lens, R, 3, pad)
    for b in range(len(lens)):
        ref = _oracle_attention(q, kp, vp, table, pos, lens, R, P, b)
        err = np.abs(got[b * R:(b + 1) * R] - ref).max()
        assert err < 2e-2, (b, err)
    if pad:
        assert np.all(got[R - 1] == 0)


def test_paged_attention_full_batch64(cuda_lib):
    """Qwen3-8B at batch 64 with prompt lengths U[512, 4096] (the benchmark's
    configuration): every request against the oracle. Most (request, KV
    head) pairs run whole in one CTA and the rest are split and merged by
    their last part, so both output paths are covered."""
    lens = synth.prompt_lengths(64, 512, 4096, 7).tolist()
    got, q, kp, vp, table, pos = _attention_case((128, 32, 8, 64), lens, 7, 7)
    for b in range(64):
        ref = _oracle_attention(q, kp, vp, table, pos, lens, 7, 64, b)
        err = np.abs(got[b * 7:(b + 1) * 7] - ref).max()
        assert err < 2e-2, (b, err)


def test_paged_attention_workspace_reuse(cuda_lib):
    """One workspace across launches of two batch sizes whose (request, KV
    head) pairs are split across CTAs: a repeat is bitwise equal (the merge
    takes a pair's parts in a fixed order, whichever CTA finished first)."""
    B_ = _b(0)
    hd, nq, nkv, P = 128, 32, 8, 64
    outs = {}
    ws = None
    for lens, R in [([3000, 2500, 1800, 4000], 7), ([900, 4000], 7), ([3000, 2500, 1800, 4000], 7)]:
        Bn = len(lens)
        need = [op.pages_covering(L + R, P) for L in lens]
        maxp = 72
        num_pages = int(sum(need)) + 5
        table, _ = synth.page_layout(need, num_pages, maxp, 5)
        pool_shape = (1, num_pages, nkv, P, hd)
        kp = _bf16(synth.bf16_round(synth.normal(pool_shape, 5, 10))).view(pool_shape)
        vp = _bf16(synth.bf16_round(synth.normal(pool_shape, 5, 11))).view(pool_shape)
        q = _bf16(synth.bf16_round(synth.normal((Bn * R, nq, hd), 5, 12, std=2.0))).view(Bn * R, nq, hd)
        pos = torch.tensor([L + r for L in lens for r in range(R)], dtype=torch.int32, device="cuda")
        if ws is None:
            ws = B_.attention_workspace(64, R, nq, nkv, hd, maxp, P)
        st = torch.zeros(1, device="cuda", dtype=torch.int32)
        out = B_.paged_attention(q, pos, kp, vp, torch.from_numpy(table).cuda(), R, 0, status=st,
                                 workspace=ws)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        key = tuple(lens)
        if key in outs:
            assert torch.equal(outs[key], out)
        outs[key] = out.clone()


# --------------------------------------------------------- accept/propose ---

def _accept_case(Bn, N, V, propose, verify, seed, boost=0.0, scale=1.0):
    B_ = _b(0)
    R = 2 * N - 1
    P = 16
    logits = synth.synthetic_logits(Bn * R, V, seed, scale=scale, boost=boost)
    n_draft = np.where(synth.integers(0, 4, (Bn,), seed, 1) == 0, 0, N - 1).astype(np.int32)
    pending = synth.integers(0, V, (Bn, N), seed, 2).astype(np.int32)
    # half the drafts are the row's argmax (likely accepted), half random
    pick = synth.integers(0, 2, (Bn, N), seed, 3)
    for b in range(Bn):
        for j in range(1, N):
            if pick[b, j]:
                pending[b, j] = int(np.argmax(logits[b * R + j - 1]))
    q_rows = None
    if propose == oi.SAMPLE:
        g = synth.normal((Bn, max(N - 1, 1), V), seed, 4, std=1.0)
        g = np.exp(g + 3.0 * (np.arange(V) == 0))
        q_rows = (g / g.sum(-1, keepdims=True)).astype(np.float32)
        for b in range(Bn):
            for j in range(1, N):
                if pick[b, j]:
                    q_rows[b, j - 1, pending[b, j]] += 0.5
            q_rows[b] /= q_rows[b].sum(-1, keepdims=True)
        q_rows = q_rows.astype(np.float32)
    u = synth.uniforms(Bn, R, seed, 0)
    seq = synth.integers(0, 500, (Bn,), seed, 5).astype(np.int32)
    need = [op.pages_covering(L + R, P) for L in seq]
    maxp = max(need) + 4
    num_pages = int(sum(need)) + 4 * Bn
    table, free = synth.page_layout(need, num_pages, maxp, seed)
    return dict(logits=logits, n_draft=n_draft, pending=pending, q_rows=q_rows, u=u, seq=seq,
                table=table, free=free, P=P, num_pages=num_pages, R=R)


def _run_accept_gpu(c, Bn, N, V, flags):
    B_ = _b(0)
    st = B_.StepState(Bn, N, V, sample=c["q_rows"] is not None)
    st.seq_len.copy_(torch.from_numpy(c["seq"]))
    st.n_draft.copy_(torch.from_numpy(c["n_draft"]))
    st.pending.copy_(torch.from_numpy(c["pending"]))
    if c["q_rows"] is not None:
        st.q_cache.copy_(torch.from_numpy(c["q_rows"]))
    shape = synth.ModelShape(1, 128, 1, 1, 64, 64, V, page_size=c["P"])
    kv = B_.KVCache(shape, c["num_pages"], c["table"], c["free"], n_layers=1)
    B_.accept_propose(torch.from_numpy(c["logits"]).cuda(), st, kv, c["P"],
                      torch.from_numpy(c["u"]).cuda(), flags)
    torch.cuda.synchronize()
    return st, kv


@pytest.mark.parametrize("Bn,N,V,propose,verify,boost,draw0", [
    (4, 2, 1024, oi.ARGMAX, oi.STOCHASTIC, 0.0, False),
    (16, 4, 1024, oi.SAMPLE, oi.STOCHASTIC, 2.0, False),
    (8, 3, 4096, oi.ARGMAX, oi.GREEDY, 0.0, False),
    (5, 1, 512, oi.ARGMAX, oi.STOCHASTIC, 0.0, False),       # N = 1: plain AR sampling
    (12, 4, 20000, oi.ARGMAX, oi.STOCHASTIC, 6.0, False),    # several vocab chunks, ragged tail
    (64, 4, 151936, oi.ARGMAX, oi.STOCHASTIC, 7.5, False),   # benchmark config, p_top ~ 0.9
    # the same with the new-token slot at u = 0 (R16): every draw then picks
    # the first token of nonzero weight, so whole requests compare exactly
    (64, 4, 151936, oi.ARGMAX, oi.STOCHASTIC, 7.5, True),
    (16, 4, 151936, oi.SAMPLE, oi.STOCHASTIC, 7.5, False),   # sampled proposals, full-vocabulary q rows
])
def test_accept_propose_matches_oracle(cuda_lib, Bn, N, V, propose, verify, boost, draw0):
    c = _accept_case(Bn, N, V, propose, verify, seed=Bn * 31 + N, boost=boost)
    if draw0:
        c["u"][:, N - 1] = 0.0
    flags = (1 if propose == oi.SAMPLE else 0) | (2 if verify == oi.GREEDY else 0)
    st, kv = _run_accept_gpu(c, Bn, N, V, flags)
    assert int(st.status.item()) == 0
    R = c["R"]
    gA = st.accepted.cpu().numpy()
    gpend = st.pending.cpu().numpy()
    gcomm = st.committed.cpu().numpy()
    gnd = st.n_draft.cpu().numpy()
    n_clear = n_accept = 0
    for b in range(Bn):
        n = int(c["n_draft"][b])
        drafts = [int(t) for t in c["pending"][b, 1:1 + n]]
        rows = c["logits"][b * R:(b + 1) * R].astype(np.float64)
        qr = None if c["q_rows"] is None else [c["q_rows"][b, j].astype(np.float64) for j in range(n)]
        dec = oi.decide(rows, drafts, qr, N, c["u"][b], propose, verify)
        # both sides saw the same logits: only fp32-vs-fp64 rounding separates them
        res = _parity.compare_decision(dec, int(gA[b]), int(gpend[b, 0]),
                                       [int(t) for t in gpend[b, 1:]], rows, rows, drafts, qr, qr,
                                       c["u"][b], N, propose, verify)
        if res.accept_clear:
            n_accept += 1
            A = dec.accepted
            assert list(gcomm[b, :A]) == drafts[:A]
            assert gnd[b] == (N - 1 if A == n else 0)
        if res.clear:
            n_clear += 1
            A = dec.accepted
            assert list(gcomm[b, :A + 1]) == drafts[:A] + [dec.new_token]
            assert gnd[b] == (N - 1 if A == n else 0)
            if propose == oi.SAMPLE and A == n and N > 1:
                gq = st.q_cache[b].double().cpu().numpy()
                for i in range(N - 1):
                    assert np.abs(gq[i] - dec.q_rows[i]).max() < 1e-6
    # accept decisions are compared exactly except within 1e-3 of p/q; draws
    # from flat tails (token mass ~1/vocab) often sit inside fp32 rounding of
    # a CDF boundary and are then checked for validity instead
    assert n_accept >= 0.9 * Bn, f"only {n_accept}/{Bn} accept decisions compared exactly"
    assert n_clear >= (0.9 if draw0 else 0.05) * Bn, f"only {n_clear}/{Bn} requests compared in full"
    print(f"accept[{Bn}x{V} N{N} {propose}/{verify}{' u0' if draw0 else ''}]: "
          f"{n_accept}/{Bn} accept decisions and {n_clear}/{Bn} whole requests compared exactly")
    # page bookkeeping (bit-exact) on the GPU's own accepted counts
    new_len, table2, head2, ok = op.bookkeep(c["seq"], gA, c["table"], c["free"], 0, N, c["P"])
    assert ok
    assert np.array_equal(st.seq_len.cpu().numpy(), new_len)
    assert np.array_equal(kv.page_table.cpu().numpy(), table2)
    assert int(kv.free_head.item()) == head2


def test_accept_all_when_u_zero_and_none_when_u_one(cuda_lib):
    """u = 0 accepts every draft with p > 0; u = 1 - 2^-24 rejects every
    draft with p < 1 - 2^-24 (a property, at the benchmark's sizes)."""
    Bn, N, V = 64, 4, 151936
    c = _accept_case(Bn, N, V, oi.ARGMAX, oi.STOCHASTIC, seed=5)
    c["n_draft"][:] = N - 1
    c["u"][:, :N - 1] = 0.0
    st, _ = _run_accept_gpu(c, Bn, N, V, 0)
    assert np.all(st.accepted.cpu().numpy() == N - 1)
    c["u"][:, :N - 1] = 1.0 - 2.0 ** -24
    st, _ = _run_accept_gpu(c, Bn, N, V, 0)
    assert np.all(st.accepted.cpu().numpy() == 0)


def test_bookkeep_pool_exhaustion_sets_status(cuda_lib):
    Bn, N, V = 4, 4, 1024
    c = _accept_case(Bn, N, V, oi.ARGMAX, oi.STOCHASTIC, seed=9)
    c["seq"][:] = 16 - 7          # every block ends on a page edge: each needs one page
    R = 7
    need = [op.pages_covering(L + R, 16) for L in c["seq"]]
    c["table"], _ = synth.page_layout(need, int(sum(need)), 8, 9)
    c["num_pages"] = int(sum(need)) + 2
    c["free"] = np.array([int(sum(need)), int(sum(need)) + 1], np.int32)   # two pages for four requests
    c["n_draft"][:] = 0
    st, kv = _run_accept_gpu(c, Bn, N, V, 0)
    from strided_verify_propose_b200 import binding
    assert int(st.status.item()) & binding.ISD_DEV_POOL_EXHAUSTED
    assert int(kv.free_head.item()) == 0
    assert np.array_equal(kv.page_table.cpu().numpy(), c["table"])
