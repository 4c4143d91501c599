"""FP64 CPU oracle for the merged-LoRA refiner hot path.

TEST INFRASTRUCTURE ONLY.  This package is the plain, slow, obviously correct
reference that the CUDA kernels are checked against.  Only ``tests/``,
``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference``
legs of ``bench.py`` may import it.  The product path (``lora_gemm_b200``)
never imports, calls or links anything here, and this package imports nothing
from the product path: the two share no code.

Sources (the pages are cited by title and section):

* "Open-H3-Regenerate-2K: High-Resolution Video Refinement with Few-Step
  Diffusion" (agientry.com, English article) -- sections "Training: learn what
  degradation removed" (flow-matching path and velocity target), "Three steps
  instead of dozens" (partial re-noise at sigma0 = 0.909 and the Euler update
  on the schedule 0.909 -> 0.857 -> 0.667 -> 0), "From any low-resolution
  draft to native 4K" and "Why upscaling happens in latent space" (latent
  grids).
* "Open-H3-Regenerate-2K：MiniMax H3 的开源 4K 精修方案" (comfyui-wiki.com
  news) -- section "三个步如何完成工作" (three adapters merged by
  concatenating their factors along the rank axis, 384 + 128 + 64 = 576,
  FP32, 312 linear layers, relative merge error 2.2e-8).
* "Open-H3-Regenerate-2K-IC" (wujieai.com) -- section
  "三步接着放大的草稿画，八步从噪声重画" (IC starts sigma = 0.835 and 0.923).
* Philox4x32-10: Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers: As
  Easy as 1, 2, 3", SC'11 (the pages name no generator).
* Box-Muller: Box and Muller, "A Note on the Generation of Random Normal
  Deviates", Ann. Math. Statist. 29 (1958) (the pages only say eps ~ N(0, I)).
* MXFP8: Open Compute Project, "OCP Microscaling Formats (MX) v1.0" and "OCP
  8-bit Floating Point (OFP8)" (the pages only name MXFP8 linear layers,
  section "Where the 3.9x speedup comes from" of the English article).

Pins (tests/test_oracle_*.py, run with ``-m "not gpu"``):

* philox      -- cuRAND's host-side Philox4_32_10 generator (an independent
                 library implementation) for several keys and offsets.
* noise       -- closed-form inverse of Box-Muller (radius and angle), exact
                 special words (u1 = 1, u2 = 0, u2 = 1/4), distribution tests.
* flow        -- exact recovery of z0 along the linear flow path with the
                 exact velocity; sigma = 0 / 1 special cases; Sterbenz
                 exactness of the schedule coefficients in FP32; the
                 projection with the Euler update by brute-force loops over
                 the latent's flat index and by exact recovery of z0 with
                 x = I (a wrong token-to-cell map misses).
* lora        -- brute-force pure-Python loops on tiny shapes, rank 0 reduces
                 to a plain GEMM, associativity through the dense merged
                 delta, merge identity B_cat A_cat = sum_i s_i B_i A_i and the
                 pages' 2.2e-8 merge-error figure.
* mxfp8       -- the E4M3 bit layout, PyTorch's independent float8_e4m3fn
                 conversion, round-to-nearest-even at every midpoint,
                 saturation, the block-exponent definition, the 3-bit-mantissa
                 error bound and brute-force loops on a tiny layer; SiLU
                 against PyTorch's and its limits, SwiGLU by brute force.

Every function here has a pin; none is "parity unpinned".
"""

from . import flow, lora, mxfp8, noise, philox  # noqa: F401
