"""Plain fp64 CPU oracle for one Introspective Strided Decoding (ISD) step.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports, calls or
links this package: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.  It
shares no code, constant table or helper with the CUDA library; the two
meet only through the seeded input generators, which hold none of the
method's arithmetic.

Sources.  The method is described on the pages collected for
"Introspective Diffusion Language Models" (arXiv 2604.11035): the abstract
(fugumt.com page, "Abstract"), and the project summary on the hada.io pages,
sections "Méthodologie d'I-DLM", "Throughput", "Speedup Factor Explorer",
"Inference & ISD" and "Serving (SGLang)".  Those pages fix the p/q
acceptance rule min(1, p(x)/q(x)), the claim that it preserves the AR
distribution, strict causal attention with logit shift, the paged KV
cache, and the tokens-per-forward closed form.  Where they are silent
(row layout of a stride, residual rule, bonus token, RNG, rollback) the
module docstrings state the reading taken.

Modules
-------
philox     Philox4x32-10 (Salmon et al., SC'11) and the uniform stream U.
attention  strided-query causal GQA attention over a paged KV cache.
vocab      softmax statistics, probabilities and the inverse CDF.
step       the accept / resample / bonus / draft step and the KV commit.
tpf        the tokens-per-forward closed form, the Markov chain behind it,
           and a finite-horizon expectation.
lm_head    the LM head that makes the logits, the R-ISD gated LoRA at MASK
           rows, bfloat16 rounding and sub-chunk vocabulary statistics.

Every floating-point quantity is computed in float64 with plain numpy.
"""
