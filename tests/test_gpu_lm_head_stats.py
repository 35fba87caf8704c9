"""The LM head's epilogue statistics against the logits it writes.

At Qwen3-8B widths (2 layers, random weights), batch 64, stride 4 (448
rows), the LM head runs stream-K over 1187 vocabulary tiles and writes,
beside the fp32 logits, the max, the sum of exp(z - max) and the first
argmax of every 32 logits; the accept step merges those statistics instead
of reading the logits a second time. Here every decision that depends only
on the argmax is checked exactly against torch.argmax of the returned
logits (first index on ties), and SAMPLE mode's stored proposal rows,
exp(z - max) / sum, against torch.softmax of the same rows.
"""
import numpy as np
import pytest

import synth
from oracle import pages as op

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")

SHAPE = synth.QWEN3_8B_2L
BN, N, STEPS, SEED = 64, 4, 4, 21


def _setup(sample):
    from strided_verify_propose_b200 import binding as B
    R, P = 2 * N - 1, SHAPE.page_size
    lens = synth.prompt_lengths(BN, 100, 400, SEED)
    prompts = synth.prompts(SHAPE, lens, SEED)
    maxp = op.pages_covering(int(lens.max()) + STEPS * N + R + 1, P) + 1
    need = [op.pages_covering(int(L) - 1 + R, P) for L in lens]
    num_pages = int(sum(need)) + BN * (op.pages_covering(STEPS * N, P) + 2)
    table, free = synth.page_layout(need, num_pages, maxp, SEED)
    model = B.Model(SHAPE, B.random_device_weights(SHAPE, seed=SEED), max_batch=BN,
                    max_rows=BN * 16, max_position=maxp * P)
    kv = B.KVCache(SHAPE, num_pages, table, free)
    st = B.StepState(BN, N, SHAPE.vocab, sample=sample)
    B.prefill(model, kv, st, prompts)
    torch.cuda.synchronize()
    assert int(st.status.item()) == 0
    return B, model, kv, st


def test_argmax_decisions_equal_the_logits_argmax():
    B, model, kv, st = _setup(sample=False)
    R = 2 * N - 1
    logits = torch.empty(BN * R, SHAPE.vocab, device="cuda", dtype=torch.float32)
    checked = 0
    for s in range(STEPS):
        n_before = st.n_draft.cpu().numpy().copy()
        pend_before = st.pending.cpu().numpy().copy()
        u = torch.from_numpy(synth.controlled_uniforms(BN, N, 0.9, SEED, s)).cuda()
        B.step(model, kv, st, u, B.VERIFY_GREEDY, logits_out=logits)
        torch.cuda.synchronize()
        assert int(st.status.item()) == 0
        am = logits.argmax(dim=1).view(BN, R).cpu().numpy()
        A = st.accepted.cpu().numpy()
        pend = st.pending.cpu().numpy()
        for b in range(BN):
            n, a = int(n_before[b]), int(A[b])
            # an accepted draft is the argmax of the row before it; the first
            # rejected one is not
            for j in range(1, a + 1):
                assert pend_before[b, j] == am[b, j - 1], (s, b, j)
            if a < n:
                assert pend_before[b, a + 1] != am[b, a], (s, b)
            assert pend[b, 0] == am[b, a], (s, b)
            if a == n:
                for i in range(1, N):
                    assert pend[b, i] == am[b, n + i], (s, b, i)
            checked += 1
    assert checked == STEPS * BN
    model.close()


def test_sampled_proposal_rows_equal_the_softmax_of_the_logits():
    B, model, kv, st = _setup(sample=True)
    R = 2 * N - 1
    logits = torch.empty(BN * R, SHAPE.vocab, device="cuda", dtype=torch.float32)
    rows = 0
    for s in range(STEPS):
        n_before = st.n_draft.cpu().numpy().copy()
        u = torch.from_numpy(synth.controlled_uniforms(BN, N, 0.9, SEED, s)).cuda()
        B.step(model, kv, st, u, B.PROPOSE_SAMPLE, logits_out=logits)
        torch.cuda.synchronize()
        assert int(st.status.item()) == 0
        A = st.accepted.cpu().numpy()
        lg = logits.view(BN, R, SHAPE.vocab)
        for b in np.nonzero(A == n_before)[0]:
            n = int(n_before[b])
            ref = torch.softmax(lg[b, n + 1:n + N], dim=1)
            torch.testing.assert_close(st.q_cache[b], ref, rtol=2e-5, atol=1e-10)
            rows += N - 1
    assert rows > 0
    model.close()
