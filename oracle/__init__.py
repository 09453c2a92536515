"""fp64 CPU oracle of the block-diffusion MoE denoising step.

TEST INFRASTRUCTURE ONLY.  Only `tests/`, `__graft_entry__.smoke()` and the
`cpu_baseline` / `--impl reference` legs of `bench.py` may import this
package.  The product path (the C-ABI library and its Python binding) never
imports, calls or falls back to it, and this package imports nothing from the
product: the two share no code.  The only shared module is `synth`, which
draws seeded random inputs and holds none of the method's arithmetic.

It is a plain, slow, obviously correct restatement of what the pages say a
denoising step computes, in float64 NumPy, in the order the pages give.

Pages cited (by title; the section follows in each citation):
  [P1] "Google open-sources DiffusionGemma: H100 reaches 1000 TPS" (openai-hub.net)
  [P2] "DiffusionGemma hits ~1,500 TPS on one H100: when a diffusion LLM beats
       autoregressive serving" (saify.me)
  [P3] "DiffusionGemma Hits 1,000 Tokens per Second - But Its Benchmarks Reveal
       the Real Tradeoff" (carussignal.com)
  [P4] "DiffusionGemma: Google open-sources a diffusion-based 26B MoE text model
       hitting 1,000+ tokens per second on H100" (modeldex.dev)
  [SC11] Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers: As Easy as 1, 2, 3",
       SC'11 (the Philox generator).

Where the pages are silent the plainest reading is taken; each reading is named
where it is used.  Pinned by tests/test_oracle_*.py (brute force, closed forms,
invariants, a library cross-check of the Philox round structure, of the E4M3
codec against the library float8 type, an exact rational brute force and a
chi-square test of the candidate draw, closed forms and invariances of the
self-conditioning term).  Model-level
end-to-end values have no printed worked example in the pages: that level is
pinned only through the invariants (frozen tokens, >= min_accept accepted per
step, convergence within the step cap, commit == prefill, permutation
equivariance) and through the per-part pins.
"""
from . import layers, model, philox, quant, sampler  # noqa: F401
