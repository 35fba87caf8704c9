"""The no-allocation accept/propose entry point against the allocating one.

isd_accept_propose_noalloc serves callers that cannot allocate device
memory (their GPU memory is all handed out by a pool they do not own, or
they must not enter the allocator once serving). It runs the same kernels
with scratch from a fixed array inside the library, so its outputs must be
identical to isd_accept_propose's on the same inputs. Two calls in a row
with different inputs check that the shared array carries nothing from one
call into the next. This file is collected last so that a failure here
never hides the other tests.
"""
import numpy as np
import pytest

from oracle import isd as oi
from tests.test_gpu_kernels import _accept_case

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


def _state(c, Bn, N, V):
    from strided_verify_propose_b200 import binding as B
    st = B.StepState(Bn, N, V, sample=c["q_rows"] is not None)
    st.seq_len.copy_(torch.from_numpy(c["seq"]))
    st.n_draft.copy_(torch.from_numpy(c["n_draft"]))
    st.pending.copy_(torch.from_numpy(c["pending"]))
    if c["q_rows"] is not None:
        st.q_cache.copy_(torch.from_numpy(c["q_rows"]))
    import synth
    shape = synth.ModelShape(1, 128, 1, 1, 64, 64, V, page_size=c["P"])
    kv = B.KVCache(shape, c["num_pages"], c["table"], c["free"], n_layers=1)
    return st, kv


def _outputs(st, kv):
    out = {k: getattr(st, k).cpu().numpy().copy()
           for k in ("accepted", "committed", "pending", "n_draft", "seq_len", "status")}
    out["page_table"] = kv.page_table.cpu().numpy().copy()
    out["free_head"] = kv.free_head.cpu().numpy().copy()
    if st.q_cache is not None:
        out["q_cache"] = st.q_cache.cpu().numpy().copy()
    return out


@pytest.mark.parametrize("Bn,N,V,propose,boost", [
    (64, 4, 151936, oi.ARGMAX, 7.5),
    (16, 3, 4096, oi.SAMPLE, 2.0),
])
def test_noalloc_matches_allocating_entry_point(cuda_lib, Bn, N, V, propose, boost):
    from strided_verify_propose_b200 import binding as B
    flags = B.PROPOSE_SAMPLE if propose == oi.SAMPLE else 0
    for call in range(2):
        c = _accept_case(Bn, N, V, propose, oi.STOCHASTIC, seed=500 + 17 * call + Bn, boost=boost)
        logits = torch.from_numpy(c["logits"]).cuda()
        u = torch.from_numpy(c["u"]).cuda()
        st_a, kv_a = _state(c, Bn, N, V)
        B.accept_propose(logits, st_a, kv_a, c["P"], u, flags)
        st_n, kv_n = _state(c, Bn, N, V)
        B.accept_propose_noalloc(logits, st_n, kv_n, c["P"], u, flags)
        torch.cuda.synchronize()
        ref, got = _outputs(st_a, kv_a), _outputs(st_n, kv_n)
        assert int(ref["status"][0]) == 0
        for k in ref:
            # the same kernels on the same inputs: integers and q rows bit-identical
            assert np.array_equal(ref[k], got[k]), (call, k)


def test_noalloc_rejects_batches_beyond_its_scratch(cuda_lib):
    from strided_verify_propose_b200 import binding as B
    V, N, Bn = 151936, 8, 1024          # 1024 * 15 * 19 * 16 bytes > 4 MiB
    st = B.StepState(Bn, N, 4, sample=False)
    import synth
    shape = synth.ModelShape(1, 128, 1, 1, 64, 64, V, page_size=16)
    kv = B.KVCache(shape, 4, np.zeros((Bn, 1), np.int32), np.zeros(1, np.int32), n_layers=1)
    logits = torch.zeros(1, V, device="cuda")      # never read: the call is refused first
    u = torch.zeros(Bn, 2 * N - 1, device="cuda")
    with pytest.raises(RuntimeError, match="fixed array holds"):
        B.accept_propose_noalloc(logits, st, kv, 16, u, 0)


def test_noalloc_calls_after_the_first_allocate_nothing(cuda_lib):
    """The property the entry point is named for: once the first call on the
    device has placed the library's array, further calls leave both the
    device's free memory and PyTorch's allocator untouched."""
    from strided_verify_propose_b200 import binding as B
    Bn, N, V = 64, 4, 151936
    c = _accept_case(Bn, N, V, oi.ARGMAX, oi.STOCHASTIC, seed=777, boost=7.5)
    logits = torch.from_numpy(c["logits"]).cuda()
    u = torch.from_numpy(c["u"]).cuda()
    st, kv = _state(c, Bn, N, V)
    B.accept_propose_noalloc(logits, st, kv, c["P"], u, 0)      # first call: may load the module
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    alloc0, reserved0 = torch.cuda.memory_allocated(), torch.cuda.memory_reserved()
    for _ in range(5):
        B.accept_propose_noalloc(logits, st, kv, c["P"], u, 0)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert int(st.status.item()) & ~B.ISD_DEV_POOL_EXHAUSTED == 0
    assert torch.cuda.memory_allocated() == alloc0
    assert torch.cuda.memory_reserved() == reserved0
    assert free1 == free0, (free0, free1)
