"""CPU oracle for the ReplaySSM decode path -- TEST INFRASTRUCTURE ONLY.

This package is the plain, slow, obviously-correct statement of what the
decode path computes, written in float64 numpy from the sources it cites.  It
exists to check the CUDA library, and only the test suite, the package smoke
check and the benchmark's CPU-baseline leg may import it.  The product path
(the C-ABI library and its Python binding) never imports, calls or links
anything here, and nothing here imports the product path.

Sources, cited in each module by page title and section:

* "Hybrid-model decoding has a new bottleneck: stop writing the SSM state every
  step, and speculative throughput reaches 2.10x" (ai4snews news page about
  the ReplaySSM paper), sections Synopsis, Interpretation, Perspective.
* "NVIDIA and Dao AI Lab speed up hybrid-model decoding" (aimodeltracker).
* "SSM decoding stops writing state every step: caching recent inputs halves
  state traffic and matches vLLM speculation" (ai4snews), sections Synopsis,
  Interpretation, Perspective.
* The published Mamba-2 recurrence (Dao & Gu, "Transformers are SSMs", 2024)
  and gated delta rule (Yang, Kautz & Hatamizadeh, "Gated Delta Networks",
  2024), which the pages name but do not print.
* Philox4x32-10 (Salmon, Moraes, Dror & Shaw, "Parallel random numbers: as easy
  as 1, 2, 3", SC'11).
* The IEEE binary16 format and the OCP microscaling formats E4M3 and E2M1 used
  by NVFP4.

Modules:

* ``recurrence`` -- step-by-step Mamba-2 and Gated DeltaNet recurrences, the
  explicit replay formulas and the fold.
* ``lowprec`` -- FP16 stochastic rounding, E4M3 / E2M1 rounding and the NVFP4
  read-copy quantiser.
* ``philox`` -- Philox4x32-10.
* ``decoder`` -- the checkpoint + input-buffer bookkeeping (step, verify,
  commit, flush) and the separate-precision modes.

Pins: every function is checked by tests marked ``not gpu`` against closed
forms, invariants stated by the pages, brute force on tiny shapes, library
routines on special cases, or published test vectors.
"""
