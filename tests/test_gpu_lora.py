"""R-ISD: the rank-128 gated LoRA on MASK rows only.

* Verify rows are bitwise base-only: the same step with and without the
  adapter gives bit-identical logits on every non-MASK row (Bud's Wiki,
  Key claims and Method: verify positions use base weights, so the output
  is bit-for-bit the base AR model's).
* The adapter's effect on MASK rows matches the oracle's (x A) B update.
"""
import numpy as np
import pytest

import synth
from oracle import isd as oi
from oracle import model as om
from oracle import pages as op
from tests import _parity
from tests.test_gpu_step import TINY_NEAR, run_pair

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


def _setup(shape, Bn, N, seed, len_lo, len_hi, steps=4):
    from strided_verify_propose_b200 import binding as B
    R, P = 2 * N - 1, shape.page_size
    lens = synth.prompt_lengths(Bn, len_lo, len_hi, seed)
    prompts = synth.prompts(shape, lens, seed)
    maxp = op.pages_covering(int(lens.max()) + steps * N + R + 1, P) + 1
    need = [op.pages_covering(int(L) - 1 + R, P) for L in lens]
    num_pages = int(sum(need)) + Bn * (op.pages_covering(steps * N, P) + 2)
    table, free = synth.page_layout(need, num_pages, maxp, seed)
    return lens, prompts, maxp, num_pages, table, free


@pytest.mark.parametrize("shape,Bn,N,len_lo,len_hi", [
    (synth.TINY, 4, 3, 5, 40),
    (synth.QWEN3_8B_2L, 8, 4, 40, 200),     # Qwen3-8B widths, rank 128
])
def test_verify_rows_bitwise_base_only(shape, Bn, N, len_lo, len_hi):
    from strided_verify_propose_b200 import binding as B
    seed = 31
    R, V = 2 * N - 1, shape.vocab
    lens, prompts, maxp, num_pages, table, free = _setup(shape, Bn, N, seed, len_lo, len_hi)
    G = shape.n_q_heads // shape.n_kv_heads
    w = B.random_device_weights(shape, seed=seed) if shape.hidden > 1024 else \
        B.pack_weights(shape, synth.decoder_weights(shape, seed=seed))
    model = B.Model(shape, w, max_batch=Bn, max_rows=max(Bn * R, Bn * (64 // G)),
                    max_position=maxp * shape.page_size)
    model.load_lora(synth.lora_weights(shape, rank=128, seed=seed, std=0.05), rank=128)
    runs = []
    for flags in (0, B.USE_LORA):
        kv = B.KVCache(shape, num_pages, table, free)
        st = B.StepState(Bn, N, V, sample=False)
        B.prefill(model, kv, st, prompts)
        per_step = []
        for s in range(3):
            # identical inputs for both runs: greedy verify keeps the two
            # trajectories' verify rows comparable step after step
            u = torch.from_numpy(synth.uniforms(Bn, R, seed, s)).cuda()
            lg = torch.empty(Bn * R, V, device="cuda")
            nd = st.n_draft.cpu().numpy().copy()
            B.step(model, kv, st, u, flags | B.VERIFY_GREEDY, logits_out=lg)
            torch.cuda.synchronize()
            assert int(st.status.item()) == 0
            per_step.append((lg.cpu().numpy(), nd, st.pending.cpu().numpy().copy()))
        runs.append(per_step)
    model.close()
    n_rows = 0
    for (lb, ndb, pb), (ll, ndl, pl) in zip(*runs):
        if not np.array_equal(ndb, ndl):
            break      # the MASK-row proposals differ, so later blocks differ
        for b in range(Bn):
            for r in range(int(ndb[b]) + 1):          # x* and the pending drafts
                row = b * R + r
                assert np.array_equal(lb[row].view(np.uint32), ll[row].view(np.uint32)), (b, r)
                n_rows += 1
        # MASK rows must actually change under the adapter
        mask_rows = [b * R + r for b in range(Bn) for r in range(int(ndb[b]) + 1, R)]
        assert np.abs(lb[mask_rows] - ll[mask_rows]).max() > 1e-3
        if not np.array_equal(pb, pl):
            break
    assert n_rows >= Bn


def test_lora_mask_rows_match_oracle():
    """Tiny decoder with the adapter on: whole ISD steps against the oracle's
    LoRA forward (logits of every used row, decisions, bookkeeping)."""
    run_pair(synth.TINY, 4, 3, 5, oi.ARGMAX, oi.GREEDY, seed=41, len_lo=5, len_hi=40,
             max_near=TINY_NEAR, min_request_steps=8, lora=True)
