"""Planted mistakes in the oracle must each fail one of its pins.

A pin is only worth something if a plausible error in the code it guards
makes it fail. Each mutant below rewrites one expression of one oracle
function (a dropped term, a wrong row or index, a flipped sign or
comparison, an off-by-one), taken from that function's own source so the
mutant tracks the oracle as it changes; the rewritten function replaces the
original, in every oracle module that refers to it, for the length of one
test, on the CPU. The test passes when some pin of that part of the oracle
fails (an assertion, or an error raised inside the pin) and names the pin
that caught it. The gated-LoRA mutants live beside their pins in
test_oracle_lora.py.
"""
import inspect
import textwrap

import pytest

import oracle
from oracle import isd as oi
from oracle import model as om
from oracle import pages as op
from tests import test_oracle_forward as TF
from tests import test_oracle_golden as TG
from tests import test_oracle_isd as TI
from tests import test_oracle_pages as TP

MODULES = (om, oi, op)


def _mutant(module, name, old, new):
    """The function `name` of `module` with the one occurrence of `old` in
    its source replaced by `new`."""
    fn = getattr(module, name)
    src = textwrap.dedent(inspect.getsource(fn))
    assert src.count(old) == 1, f"{name}: expected one occurrence of {old!r}"
    ns = dict(vars(module))
    exec(compile(src.replace(old, new), f"<mutant of {module.__name__}.{name}>", "exec"), ns)
    return fn, ns[name]


def _with_monkeypatch(fn, *args):
    def run():
        mp = pytest.MonkeyPatch()
        try:
            fn(mp, *args)
        finally:
            mp.undo()
    return run


ISD_PINS = [
    ("inverse-CDF and argmax rules", TI.test_inverse_cdf_rules),
    ("residual falls back to p", TI.test_residual_with_identical_p_q_falls_back_to_p),
    ("zero-probability draft rejected", TI.test_a_draft_of_probability_zero_is_never_accepted),
    ("printed speedups", lambda: [TG.test_printed_speedup_numbers(c) for c in TG.CASES]),
    ("exact p, argmax proposals",
     lambda: [TI.test_accept_resample_reproduces_p_exactly(oi.ARGMAX, s) for s in range(3)]),
    ("exact p, sampled proposals",
     lambda: [TI.test_accept_resample_reproduces_p_exactly(oi.SAMPLE, s) for s in range(3)]),
    ("exact p at the second draft",
     lambda: [TI.test_second_draft_reproduces_its_row_exactly(pr, s)
              for pr in (oi.ARGMAX, oi.SAMPLE) for s in range(2)]),
    ("q = p accepts every draft", TI.test_q_equal_p_accepts_every_draft),
    ("N = 1 is AR", TI.test_stride_one_is_plain_ar),
    ("greedy ISD = greedy AR", lambda: [TI.test_greedy_isd_equals_greedy_ar(N) for N in (2, 3, 4)]),
    ("KV history = committed tokens", TI.test_kv_history_matches_committed_tokens),
    ("TPF renewal = formula",
     lambda: [TI.test_layout_tpf_equals_pages_formula_exactly(N) for N in (2, 3, 4, 5)]),
    ("perfect predictor", lambda: [_with_monkeypatch(
        TI.test_a_perfect_predictor_accepts_every_draft, N)() for N in (2, 3, 4)]),
    ("trajectory distribution = AR",
     lambda: [TI.test_isd_trajectory_distribution_equals_ar(N, pr, 3)
              for N, pr in ((2, oi.ARGMAX), (3, oi.ARGMAX), (2, oi.SAMPLE))]),
]

MODEL_PINS = [
    ("RMSNorm closed form", TF.test_rms_norm_closed_form),
    ("RMSNorm = library norm", TF.test_rms_norm_matches_the_library_norm_at_large_eps),
    ("RoPE closed forms", TF.test_rope_closed_forms),
    ("single visible key", TF.test_single_key_attention_returns_value),
    ("causal rows", TF.test_block_rows_are_causal),
    ("independent Qwen3 forward", TF.test_forward_matches_independent_qwen3),
    ("KV history = committed tokens", TI.test_kv_history_matches_committed_tokens),
]

PAGE_PINS = [
    ("covers and never shares",
     lambda: [TP.test_bookkeep_covers_and_never_shares(s) for s in range(5)]),
    ("exhausted pool", TP.test_bookkeep_exhausted_pool_assigns_nothing),
    ("table row too short", TP.test_bookkeep_table_row_too_short_assigns_nothing),
]

# (module, function, expression, its mutant, pins)
MUTANTS = {
    # accept / resample / propose
    "accept test drops q": (oi, "decide", "float(u[j - 1]) * qd < p[d]", "float(u[j - 1]) < p[d]", ISD_PINS),
    "accept test <= instead of <": (oi, "decide", "float(u[j - 1]) * qd < p[d]",
                                    "float(u[j - 1]) * qd <= p[d]", ISD_PINS),
    "draft scored by its own row": (oi, "decide", "z = logits[j - 1]", "z = logits[j]", ISD_PINS),
    "new token from the row after A": (oi, "decide", "z = logits[A]\n", "z = logits[min(A + 1, len(logits) - 1)]\n",
                                       ISD_PINS),
    "residual removes the wrong draft": (oi, "decide", "q[int(drafts[A])] = 1.0", "q[int(drafts[A - 1])] = 1.0",
                                         ISD_PINS),
    "no residual after a rejection": (oi, "decide", "w = residual(p, q)", "w = p", ISD_PINS),
    "new token reuses the first uniform": (oi, "decide", "inverse_cdf(w, float(u[N - 1]))",
                                           "inverse_cdf(w, float(u[0]))", ISD_PINS),
    "proposals read one MASK row early": (oi, "decide", "zi = logits[n + i]", "zi = logits[n + i - 1]", ISD_PINS),
    "proposals kept after a rejection": (oi, "decide", "    if A == n:\n        for i in range(1, N):",
                                         "    if True:\n        for i in range(1, N):", ISD_PINS),
    "verification continues past a rejection": (oi, "decide", "            A = j - 1\n            break",
                                                "            A = j - 1", ISD_PINS),
    "residual is max(0, q - p)": (oi, "residual", "np.maximum(0.0, p - q)", "np.maximum(0.0, q - p)", ISD_PINS),
    "residual never falls back to p": (oi, "residual", "return r if r.sum() > 0 else p", "return r", ISD_PINS),
    "inverse CDF with >=": (oi, "inverse_cdf", "np.flatnonzero(c > t)", "np.flatnonzero(c >= t)", ISD_PINS),
    "argmax takes the last maximum": (oi, "argmax_lowest", "(z == z.max())[0]", "(z == z.max())[-1]", ISD_PINS),
    "TPF denominator uses a^N": (oi, "tpf_formula", "a ** (n_stride - 1))", "a ** n_stride)", ISD_PINS),
    # block layout and commit
    "block positions start at L + 1": (oi, "block_tokens", "st.seq_len + np.arange(R)",
                                       "st.seq_len + 1 + np.arange(R)", ISD_PINS),
    "one MASK row too few": (oi, "block_tokens", "[mask_token] * (R - 1 - n)", "[mask_token] * max(R - 2 - n, 0)",
                             ISD_PINS),
    "KV of x* not committed": (oi, "isd_step", "commit_kv(st.kv, bk, bv, A + 1)",
                               "commit_kv(st.kv, bk, bv, max(A, 1))", ISD_PINS),
    "rejected draft committed": (oi, "isd_step", "committed = list(st.drafts[:A]) + [dec.new_token]",
                                 "committed = list(st.drafts[:A + 1]) + [dec.new_token]", ISD_PINS),
    "x* left out of the history": (oi, "isd_step", "st.history.extend([st.x_star] + list(st.drafts[:A]))",
                                   "st.history.extend(list(st.drafts[:A + 1]))", ISD_PINS),
    # decoder forward
    "RMSNorm over |x|": (om, "rms_norm", "np.mean(x * x,", "np.mean(np.abs(x),", MODEL_PINS),
    "RMSNorm eps outside the root": (om, "rms_norm", "np.sqrt(ms + eps)", "(np.sqrt(ms) + eps)", MODEL_PINS),
    "RoPE rotates the wrong way": (om, "rope_neox", "x1 * c - x2 * s, x2 * c + x1 * s",
                                   "x1 * c + x2 * s, x2 * c - x1 * s", MODEL_PINS),
    "RoPE frequencies without the 2": (om, "rope_neox", "(2.0 * np.arange(half, dtype=np.float64))",
                                       "(np.arange(half, dtype=np.float64))", MODEL_PINS),
    "RoPE pairs adjacent lanes": (om, "rope_neox", "x1, x2 = x[..., :half], x[..., half:]",
                                  "x1, x2 = x[..., 0::2], x[..., 1::2]", MODEL_PINS),
    "query head reads KV head h mod n_kv": (om, "causal_gqa_attention", "g = hq // G", "g = hq % K.shape[1]",
                                            MODEL_PINS),
    "attention without 1/sqrt(d)": (om, "causal_gqa_attention", "scale = 1.0 / np.sqrt(d)", "scale = 1.0",
                                    MODEL_PINS),
    "row cannot see itself": (om, "causal_gqa_attention", "visible = k_pos <= q_pos[r]",
                              "visible = k_pos < q_pos[r]", MODEL_PINS),
    "row sees the next row": (om, "causal_gqa_attention", "visible = k_pos <= q_pos[r]",
                              "visible = k_pos <= q_pos[r] + 1", MODEL_PINS),
    "no QK-norm on k": (om, "block_forward", 'rope_neox(rms_norm(k, lw["k_norm"], s.rms_eps), pos, s.rope_theta)',
                        "rope_neox(k, pos, s.rope_theta)", MODEL_PINS),
    "RoPE on v as well": (om, "block_forward",
                          'v = _proj(m, l, "v", "wv", h, lora_rows).reshape(R, s.n_kv_heads, s.head_dim)',
                          'v = rope_neox(_proj(m, l, "v", "wv", h, lora_rows).reshape(R, s.n_kv_heads, '
                          's.head_dim), pos, s.rope_theta)', MODEL_PINS),
    "attention output replaces the residual": (om, "block_forward", 'x = x + _proj(m, l, "o", "wo"',
                                               'x = 0 * x + _proj(m, l, "o", "wo"', MODEL_PINS),
    "gate and up swapped": (om, "block_forward",
                            'silu(_proj(m, l, "gate", "w_gate", h, lora_rows)) * _proj(m, l, "up", "w_up", h, '
                            'lora_rows)',
                            'silu(_proj(m, l, "up", "w_up", h, lora_rows)) * _proj(m, l, "gate", "w_gate", h, '
                            'lora_rows)', MODEL_PINS),
    "MLP norm reads the pre-attention stream": (om, "block_forward", 'h = rms_norm(x, lw["mlp_norm"], s.rms_eps)',
                                                'h = rms_norm(x - _proj(m, l, "o", "wo", att.reshape(R, s.q_dim), '
                                                'lora_rows), lw["mlp_norm"], s.rms_eps)', MODEL_PINS),
    "no final norm": (om, "block_forward", "rms_norm(x, m.final_norm, s.rms_eps) @ m.lm_head.T",
                      "x @ m.lm_head.T", MODEL_PINS),
    "SiLU is the sigmoid": (om, "silu", "x / (1.0 + np.exp(-x))", "1.0 / (1.0 + np.exp(-x))", MODEL_PINS),
    "commit keeps the last rows": (om, "commit_kv", "block_k[l][:n_rows]", "block_k[l][len(block_k[l]) - n_rows:]",
                                   MODEL_PINS + ISD_PINS[6:9]),
    # page bookkeeping
    "held pages counted without the block": (op, "bookkeep", "have = np.array([pages_covering(L + R, page_size)",
                                             "have = np.array([pages_covering(L + 1, page_size)", PAGE_PINS),
    "length grows by A only": (op, "bookkeep", "new_len = seq_len + 1 + accepted", "new_len = seq_len + accepted",
                               PAGE_PINS),
    "inclusive offsets": (op, "bookkeep", "np.concatenate([[0], np.cumsum(count)[:-1]])", "np.cumsum(count)",
                          PAGE_PINS),
    "exact fit refused": (op, "bookkeep", "free_head + total <= len(free_list)", "free_head + total < len(free_list)",
                          PAGE_PINS),
    "row width never checked": (op, "bookkeep", " and bool(np.all(want <= table.shape[1]))", "", PAGE_PINS),
    "pages rounded down": (op, "pages_covering", "-(-int(length) // int(page_size))",
                           "int(length) // int(page_size)", PAGE_PINS),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_fails_a_pin(name, monkeypatch):
    module, fname, old, new, pins = MUTANTS[name]
    original, mutant = _mutant(module, fname, old, new)
    for mod in MODULES + (oracle,):
        for attr, val in list(vars(mod).items()):
            if val is original:
                monkeypatch.setattr(mod, attr, mutant)
    for pin_name, pin in pins:
        try:
            pin()
        except Exception as e:          # an assertion, or an error inside the pin
            print(f"{name}: caught by '{pin_name}' ({type(e).__name__})")
            return
    pytest.fail(f"planted mistake '{name}' passed every pin")
