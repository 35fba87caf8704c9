"""Whole ISD steps at the benchmark's full size, checked by properties.

The headline workload in the launch configuration bench.py times: Qwen3-8B
shape with all 36 layers (random weights drawn on the device), batch 64,
stride 4 (448 block rows), prompts U[512, 4096], pages randomly permuted;
and the Qwen3-32B shape (64 layers) at batch 64 with prompts U[1024, 8192].
The oracle cannot run this model, so each step is checked by what holds at
any size:

* page bookkeeping: the lengths, the page table and the free-list head after
  the step equal the oracle's bookkeeping (oracle/pages.py) applied to the
  GPU's own accepted counts, bit for bit;
* greedy verification with argmax proposals: every accepted draft, every
  rejected one, every new token and every proposal follows from
  torch.argmax of the step's returned logits (first index on ties);
* lengths advance by 1 + A, committed tokens are the accepted drafts and the
  new token, and the status word stays 0.
"""
import numpy as np
import pytest

import synth
from oracle import pages as op

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")

BN, N, STEPS, SEED = 64, 4, 3, 1000


@pytest.mark.parametrize("shape_name,len_lo,len_hi", [
    ("QWEN3_8B", 512, 4096),       # the headline workload
    ("QWEN3_32B", 1024, 8192),     # Qwen3-32B shape, 64 layers, 56 query rows per KV head
])
def test_full_size_steps_hold_their_invariants(shape_name, len_lo, len_hi):
    from strided_verify_propose_b200 import binding as B
    SHAPE = getattr(synth, shape_name)
    R, P, V = 2 * N - 1, SHAPE.page_size, SHAPE.vocab
    lens = synth.prompt_lengths(BN, len_lo, len_hi, SEED)
    prompts = synth.prompts(SHAPE, lens, SEED)
    maxp = op.pages_covering(int(lens.max()) + (STEPS + 1) * N + R + 1, P) + 1
    need = [op.pages_covering(int(L) - 1 + R, P) for L in lens]
    num_pages = int(sum(need)) + BN * (op.pages_covering((STEPS + 1) * N, P) + 2)
    table, free = synth.page_layout(need, num_pages, maxp, SEED)
    model = B.Model(SHAPE, B.random_device_weights(SHAPE, seed=SEED), max_batch=BN,
                    max_rows=BN * 16, max_position=maxp * P)
    kv = B.KVCache(SHAPE, num_pages, table, free)
    st = B.StepState(BN, N, V, sample=False)
    B.prefill(model, kv, st, prompts)
    torch.cuda.synchronize()
    assert int(st.status.item()) == 0
    assert np.array_equal(st.seq_len.cpu().numpy(), lens - 1)
    logits = torch.empty(BN * R, V, device="cuda", dtype=torch.float32)
    free_np = np.asarray(free)
    for s in range(STEPS):
        seq0 = st.seq_len.cpu().numpy().copy()
        n0 = st.n_draft.cpu().numpy().copy()
        pend0 = st.pending.cpu().numpy().copy()
        table0 = kv.page_table.cpu().numpy().copy()
        head0 = int(kv.free_head.item())
        u = torch.from_numpy(synth.controlled_uniforms(BN, N, 0.9, SEED, s)).cuda()
        B.step(model, kv, st, u, B.VERIFY_GREEDY, logits_out=logits)
        torch.cuda.synchronize()
        assert int(st.status.item()) == 0
        A = st.accepted.cpu().numpy()
        # bookkeeping, bit for bit, on the GPU's accepted counts
        new_len, table1, head1, ok = op.bookkeep(seq0, A, table0, free_np, head0, N, P)
        assert ok
        assert np.array_equal(st.seq_len.cpu().numpy(), new_len)
        assert np.array_equal(new_len, seq0 + 1 + A)
        assert np.array_equal(kv.page_table.cpu().numpy(), table1)
        assert int(kv.free_head.item()) == head1
        # every decision from the argmax of the returned logits
        am = logits.argmax(dim=1).view(BN, R).cpu().numpy()
        pend = st.pending.cpu().numpy()
        comm = st.committed.cpu().numpy()
        for b in range(BN):
            n, a = int(n0[b]), int(A[b])
            assert 0 <= a <= n
            for j in range(1, a + 1):
                assert pend0[b, j] == am[b, j - 1], (s, b, j)
            if a < n:
                assert pend0[b, a + 1] != am[b, a], (s, b)
            assert pend[b, 0] == am[b, a], (s, b)
            assert list(comm[b, :a + 1]) == [int(t) for t in pend0[b, 1:a + 1]] + [int(am[b, a])]
            if a == n:
                assert int(st.n_draft[b].item()) == N - 1
                for i in range(1, N):
                    assert pend[b, i] == am[b, n + i], (s, b, i)
            else:
                assert int(st.n_draft[b].item()) == 0
    model.close()
