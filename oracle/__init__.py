"""CPU oracle for the SureLock decoding step -- TEST INFRASTRUCTURE ONLY.

Only the test-suite, the smoke check and the benchmark's CPU-baseline leg may
import this package.  The product path (the CUDA library and its Python
binding) never imports, calls or links anything here, and this package never
imports the product: the two share no code.  Both receive their inputs from
`workloads`, which draws random numbers and holds none of the method's
arithmetic.

The oracle restates, in plain NumPy, what the pages on SureLock ("Stopping
Computation for Converged Tokens in Masked Diffusion-LM Decoding", Oba,
Bollegala, Kaneko, Okazaki) say one decoding step computes: a bidirectional
masked-diffusion transformer run on the active rows only, the step-to-step KL
"sure" test with its optional confidence gate, stable compaction of the active
set, and the semi-autoregressive unmasking sampler that drives it.  Arithmetic
is float64 unless the caller passes float32 arrays (used only where an 8B-shaped
case would not fit the CPU time budget).

Modules:
  model     -- the denoiser restricted to active rows (RMSNorm, RoPE, attention
               over cached + fresh K/V, SwiGLU, LM head)
  surelock  -- sure test, confidence gate, compaction, unmasking, the sampler with
               locking, the plain sampler without locking, a teacher-forced step
  brute     -- scalar-loop restatements for tiny shapes (pins for the above)

Pins: every function here is checked by `tests/test_oracle_*.py` against closed
forms, invariants the pages state, special cases that reduce to a library
routine, or brute force on tiny inputs.  Two parts carry no such pin
("parity unpinned"): the error bound of Theorem 1, whose constants the pages do
not define (nothing here computes it), and full-model values at the LLaDA-8B
shape, which no page prints.
"""
