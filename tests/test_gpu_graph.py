"""Steps replayed from a CUDA graph equal the same steps launched eagerly.

One or more isd_step calls are captured once (binding.StepGraph) and
replayed with new uniforms; from the same starting state (KV pools, page
table, free list, request state) the replays must reproduce the eager
steps bit for bit: the committed tokens, acceptance counts, lengths,
pending drafts, proposal rows, page bookkeeping and every KV byte.
"""
import numpy as np
import pytest

import synth

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


def _setup(shape, Bn, N, seed, len_lo, len_hi, steps, sample):
    from strided_verify_propose_b200 import binding as B
    R, P = 2 * N - 1, shape.page_size
    lens = synth.prompt_lengths(Bn, len_lo, len_hi, seed)
    prompts = synth.prompts(shape, lens, seed)
    maxp = -(-(int(lens.max()) + steps * N + R + 1) // P) + 1
    need = [-(-(int(L) - 1 + R) // P) for L in lens]
    num_pages = int(sum(need)) + Bn * (-(-steps * N // P) + 2)
    table, free = synth.page_layout(need, num_pages, maxp, seed)
    G = shape.n_q_heads // shape.n_kv_heads
    model = B.Model(shape, B.random_device_weights(shape, seed=seed), max_batch=Bn,
                    max_rows=max(Bn * R, Bn * (64 // G)), max_position=maxp * P)
    kv = B.KVCache(shape, num_pages, table, free)
    st = B.StepState(Bn, N, shape.vocab, sample=sample)
    B.prefill(model, kv, st, prompts)
    torch.cuda.synchronize()
    assert int(st.status.item()) == 0
    return B, model, kv, st


def _snapshot(kv, st):
    t = [kv.k_pool, kv.v_pool, kv.page_table, kv.free_list, kv.free_head, st.seq_len, st.n_draft,
         st.pending, st.accepted, st.committed, st.status]
    if st.q_cache is not None:
        t.append(st.q_cache)
    return t


@pytest.mark.parametrize("shape_name,Bn,N,per_graph,sample", [
    ("TINY", 4, 3, 1, False),
    ("TINY", 3, 4, 3, True),          # three steps per graph, sampled proposals (q rows)
    ("QWEN3_8B_2L", 16, 4, 2, False),  # stream-K GEMMs, tcgen05 attention
])
def test_graph_replay_equals_eager(cuda_lib, shape_name, Bn, N, per_graph, sample):
    shape = getattr(synth, shape_name)
    rounds = 3
    steps = rounds * per_graph
    B, model, kv, st = _setup(shape, Bn, N, 11, 40, 300, steps + 1, sample)
    flags = B.PROPOSE_SAMPLE if sample else 0
    R = 2 * N - 1
    u = torch.from_numpy(np.stack([synth.uniforms(Bn, R, 11, s) for s in range(steps + 1)])).cuda()
    # one eager step first (kernel attributes are set on first use), then the reference run
    B.step(model, kv, st, u[steps], flags)
    torch.cuda.synchronize()
    start = [x.clone() for x in _snapshot(kv, st)]
    eager = []
    for s in range(steps):
        B.step(model, kv, st, u[s], flags)
        eager.append([st.committed.clone(), st.accepted.clone(), st.seq_len.clone()])
    torch.cuda.synchronize()
    eager_end = [x.clone() for x in _snapshot(kv, st)]
    assert int(st.status.item()) == 0
    # restore the starting state into the same buffers, capture, replay
    for dst, src in zip(_snapshot(kv, st), start):
        dst.copy_(src)
    torch.cuda.synchronize()
    g = B.StepGraph(model, kv, st, per_graph, flags)
    # capturing launches nothing: the state is still the starting state
    torch.cuda.synchronize()
    for dst, src in zip(_snapshot(kv, st), start):
        assert torch.equal(dst, src)
    for r in range(rounds):
        g.replay(u[r * per_graph:(r + 1) * per_graph])
        torch.cuda.synchronize()
        last = r * per_graph + per_graph - 1
        for got, ref in zip([st.committed, st.accepted, st.seq_len], eager[last]):
            assert torch.equal(got, ref), f"round {r}"
    for got, ref in zip(_snapshot(kv, st), eager_end):
        assert torch.equal(got, ref)
