"""CPU oracle for one Introspective Strided Decoding (ISD) step.

TEST INFRASTRUCTURE ONLY. Nothing on the product path imports, links or runs
this package: it is used by ``tests/``, by ``__graft_entry__.smoke()`` and by
the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py``. It shares no
code with the CUDA library; the two meet only through the seeded inputs of
the ``synth`` module.

Plain, slow, fp64 numpy. Every function restates a step of the method as
the pages describe it, in their notation (stride N, anchor p, proposal q,
acceptance min(1, p/q), MASK positions). Sources, cited by short tag:

  [wiki]  Bud's Wiki, "Introspective Diffusion Language Models"
          (sections TL;DR, Key claims, Method, Results)
  [blog]  Agentic Commons blog, "Introspective Diffusion Language Models"
          (sections "Introspective Consistency: AR's Hidden Advantage",
          "How Introspective Strided Decoding Works", "Why Dropping into SGLang Matters")
  [gn-hi] GeekNews (hi), "I-DLM - Introspective Diffusion Language Models"
          (sections Throughput, Speedup Factor Explorer, Inference & ISD, Lossless R-ISD)
  [gn-pt] GeekNews (pt), the Portuguese mirror of [gn-hi]

Where the pages leave a step open the oracle takes one fixed reading; each
reading is listed in the docstring of the function that applies it.

Parity status: the model forward is pinned to an independent Qwen3 decoder
implementation (HF transformers) on tiny shapes; the accept / resample rule by
exact enumeration; the ISD layout by the pages' TPF formula, the TPF and
efficiency values the pages print, and brute-force trajectory distributions;
the gated LoRA by bitwise base-only verify rows and by a merged-weight model
on the MASK rows; page bookkeeping by brute-force invariants; which MASK
row proposes which draft position (reading R4 of isd.py), which no
distribution-level test can see, by a predictor that is perfect for a token
sequence: every draft accepted, tokens per forward N as the pages' formula
gives at acceptance 1.
"""
