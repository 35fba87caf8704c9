"""Failure detection on the GPU, with every failure made on the host.

The library reports what it finds on the device through the caller's int32
status word (ISD_DEV_* bits) and keeps going; host-side argument errors
come back as negative return codes. Each test here injects one fault from
the host into otherwise valid inputs (a draft token outside the
vocabulary, a page id outside the pool, a draft count the layout does not
allow, a request that outgrows its page-table row, a stream-K partner flag
that nothing will set) and checks the reported bit. No test faults, traps
or hangs the GPU: every device wait is bounded, and the timeout test first
shortens that bound with isd_set_wait_limit. The resume test checks that
all step state lives in caller buffers: 8 steps, a copy of every buffer
through the host into fresh ones, 8 more steps equal 16 straight steps.
"""
import ctypes

import numpy as np
import pytest

import synth
from oracle import pages as op

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")

SHAPE = synth.TINY


def _run(Bn=2, N=3, len_lo=20, len_hi=40, seed=7, spare_pages=4, maxp_extra=4, lens=None):
    from strided_verify_propose_b200 import binding as B
    R, P = 2 * N - 1, SHAPE.page_size
    lens = synth.prompt_lengths(Bn, len_lo, len_hi, seed) if lens is None else np.asarray(lens)
    prompts = synth.prompts(SHAPE, lens, seed)
    need = [op.pages_covering(int(L) - 1 + R, P) for L in lens]
    maxp = max(need) + maxp_extra
    num_pages = int(sum(need)) + spare_pages
    table, free = synth.page_layout(need, num_pages, maxp, seed)
    model = B.Model(SHAPE, B.pack_weights(SHAPE, synth.decoder_weights(SHAPE, seed=seed)),
                    max_batch=Bn, max_rows=max(Bn * R, Bn * 32), max_position=maxp * P)
    kv = B.KVCache(SHAPE, num_pages, table, free)
    st = B.StepState(Bn, N, SHAPE.vocab, sample=False)
    B.prefill(model, kv, st, prompts)
    torch.cuda.synchronize()
    assert int(st.status.item()) == 0
    return B, model, kv, st


def _step(B, model, kv, st, s, flags=0, seed=3):
    u = synth.controlled_uniforms(st.B, st.N, 0.9, seed, s)
    B.step(model, kv, st, torch.from_numpy(u).cuda(), flags)
    torch.cuda.synchronize()
    return int(st.status.item())


def test_bad_draft_token_sets_bad_token():
    B, model, kv, st = _run()
    assert _step(B, model, kv, st, 0) == 0           # a restart step: drafts pending now
    assert int(st.n_draft[0].item()) == st.N - 1
    st.pending[0, 1] = SHAPE.vocab + 7               # host-injected draft outside the vocabulary
    status = _step(B, model, kv, st, 1)
    assert status & B.ISD_DEV_BAD_TOKEN
    # the bad draft is never accepted
    assert int(st.accepted[0].item()) == 0
    model.close()


def test_page_id_outside_the_pool_sets_bad_page():
    B, model, kv, st = _run()
    L = int(st.seq_len[0].item())
    kv.page_table[0, L // SHAPE.page_size] = kv.num_pages + 3   # the page the block writes into
    status = _step(B, model, kv, st, 0)
    assert status & B.ISD_DEV_BAD_PAGE
    model.close()


def test_draft_count_outside_the_layout_sets_bad_state():
    B, model, kv, st = _run(N=3)
    st.n_draft[1] = 1                                # neither 0 nor N - 1
    status = _step(B, model, kv, st, 0)
    assert status & B.ISD_DEV_BAD_STATE
    model.close()


def test_request_outgrowing_its_page_row_sets_table_full():
    # prompt of 28 tokens: L = 27 and L + 2N - 1 = 32 fills two 16-slot pages
    # exactly, so any step needs a third page, and the row has only two
    B, model, kv, st = _run(Bn=1, N=3, lens=[28], maxp_extra=0)
    assert kv.max_pages_per_req == 2
    before = kv.page_table.cpu().numpy().copy()
    status = _step(B, model, kv, st, 0)
    assert status & B.ISD_DEV_TABLE_FULL
    assert not status & B.ISD_DEV_POOL_EXHAUSTED
    # nothing was handed out
    assert np.array_equal(kv.page_table.cpu().numpy(), before)
    assert int(kv.free_head.item()) == 0
    model.close()


def test_step_refuses_bad_host_arguments():
    B, model, kv, st = _run()
    lib = B.lib()
    u = torch.zeros(st.B, 2 * st.N - 1, device="cuda")

    def call(batch=None, **kw):
        b = batch or B.Batch(st.B, st.N, kw.get("flags", 0), B._ptr(st.seq_len), B._ptr(st.n_draft),
                             None)
        return lib.isd_step(model.ctx, ctypes.byref(b), ctypes.byref(kv.c()), B._ptr(st.pending),
                            kw.get("q", None), B._ptr(u), B._ptr(st.accepted), B._ptr(st.committed),
                            B._ptr(st.status), B._stream())

    assert call(flags=0x80) == B.ISD_E_INVALID                      # unknown flag bit
    assert call(flags=B.USE_LORA) == B.ISD_E_INVALID                # no adapter loaded
    assert call(flags=B.PROPOSE_SAMPLE) == B.ISD_E_INVALID          # sampled proposals, no q rows
    assert call(B.Batch(0, st.N, 0, B._ptr(st.seq_len), B._ptr(st.n_draft), None)) == B.ISD_E_INVALID
    assert call(B.Batch(st.B, 9, 0, B._ptr(st.seq_len), B._ptr(st.n_draft), None)) == B.ISD_E_INVALID
    assert call(B.Batch(st.B, st.N, 0, None, B._ptr(st.n_draft), None)) == B.ISD_E_INVALID
    # more block rows than the context was sized for
    big = B.Batch(model.max_batch + 1, st.N, 0, B._ptr(st.seq_len), B._ptr(st.n_draft), None)
    assert call(big) == B.ISD_E_INVALID
    torch.cuda.synchronize()
    assert int(st.status.item()) == 0        # nothing was enqueued
    model.close()


def test_bounded_wait_runs_out_and_the_context_stays_usable():
    """A stream-K GEMM whose cut tiles find their partner's arrival already
    counted (the test writes 1 into every arrival word of the workspace):
    each part then waits for a ready flag that nothing sets. With the wait
    limit at 2e6 cycles (about 1 ms) the waits run out, ISD_DEV_TIMEOUT is
    set, and the kernel returns; the same call with a clean workspace and
    the default limit then gives the right product."""
    from strided_verify_propose_b200 import binding as B
    m, n, k = 448, 24576, 4096          # the MLP gate/up shape: stream-K with cut tiles
    plan = B.gemm_plan(m, n, k, single=True)
    assert plan["streamk"] == 1
    g = torch.Generator(device="cuda").manual_seed(5)
    w = (torch.randn(n, k, device="cuda", generator=g) * 0.02).to(torch.bfloat16)
    x = torch.randn(m, k, device="cuda", generator=g).to(torch.bfloat16)
    ws = B.gemm_workspace(m, n, k)
    slots = plan["units"] * (2 if plan["pair"] else 1)
    ws.view(torch.int32)[0:2 * slots:2] = 1          # arrival counts: "the partner came first"
    status = torch.zeros(1, device="cuda", dtype=torch.int32)
    try:
        B.set_wait_limit(2_000_000)
        B.gemm_bf16_single(w, x, ws, status=status)
        torch.cuda.synchronize()
    finally:
        B.set_wait_limit(0)
    assert int(status.item()) & B.ISD_DEV_TIMEOUT
    # the device is fine: a clean workspace and the default limit
    ws.zero_()
    status.zero_()
    y = B.gemm_bf16_single(w, x, ws, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref = x.float() @ w.float().t()
    assert (y - ref).abs().max().item() <= 2e-4 * ref.abs().max().item() + 1e-3


def _state_buffers(kv, st):
    # bf16 pools as their 16-bit patterns (numpy has no bfloat16)
    return [kv.k_pool.view(torch.int16), kv.v_pool.view(torch.int16), kv.page_table, kv.free_head,
            st.seq_len, st.n_draft, st.pending]


@pytest.mark.parametrize("shape_name,Bn", [("TINY", 4), ("QWEN3_8B_2L", 8)])
def test_resume_from_host_copies_equals_a_straight_run(shape_name, Bn):
    from strided_verify_propose_b200 import binding as B
    shape = getattr(synth, shape_name)
    N, seed, steps = 4, 13, 16
    R, P = 2 * N - 1, shape.page_size
    lens = synth.prompt_lengths(Bn, 30, 150, seed)
    prompts = synth.prompts(shape, lens, seed)
    maxp = op.pages_covering(int(lens.max()) + steps * N + R + 1, P) + 1
    need = [op.pages_covering(int(L) - 1 + R, P) for L in lens]
    num_pages = int(sum(need)) + Bn * (op.pages_covering(steps * N, P) + 2)
    table, free = synth.page_layout(need, num_pages, maxp, seed)
    G = shape.n_q_heads // shape.n_kv_heads
    w = B.random_device_weights(shape, seed=seed) if shape.hidden > 1024 else \
        B.pack_weights(shape, synth.decoder_weights(shape, seed=seed))
    model = B.Model(shape, w, max_batch=Bn, max_rows=max(Bn * R, Bn * (64 // G)),
                    max_position=maxp * P)

    def fresh():
        kv = B.KVCache(shape, num_pages, table, free)
        st = B.StepState(Bn, N, shape.vocab, sample=False)
        B.prefill(model, kv, st, prompts)
        return kv, st

    def run(kv, st, lo, hi):
        out = []
        for s in range(lo, hi):
            u = torch.from_numpy(synth.controlled_uniforms(Bn, N, 0.9, seed, s)).cuda()
            B.step(model, kv, st, u, 0)
            out.append(st.committed.cpu().numpy()[:, :].copy())
            out.append(st.accepted.cpu().numpy().copy())
        torch.cuda.synchronize()
        assert int(st.status.item()) == 0
        return out

    kv, st = fresh()
    straight = run(kv, st, 0, steps)
    final_straight = [t.cpu().numpy().copy() for t in _state_buffers(kv, st)]
    del kv, st
    kv, st = fresh()
    first = run(kv, st, 0, steps // 2)
    host = [t.cpu().numpy().copy() for t in _state_buffers(kv, st)]
    del kv, st
    kv2, st2 = fresh()                  # new buffers, then every byte of state restored
    for t, h in zip(_state_buffers(kv2, st2), host):
        t.copy_(torch.from_numpy(h))
    second = run(kv2, st2, steps // 2, steps)
    for a, b in zip(straight, first + second):
        assert np.array_equal(a, b)
    for a, t in zip(final_straight, _state_buffers(kv2, st2)):
        assert np.array_equal(a.view(np.uint8), t.cpu().numpy().view(np.uint8))
    model.close()
