"""CPU oracle for the fine-grained block-scaled FP8 GEMM.

TEST INFRASTRUCTURE ONLY.  This package is the slow, obviously correct reference
that the CUDA path is checked against.  Only the test suite, the smoke check in
``__graft_entry__`` and the ``cpu_baseline`` / ``--impl reference`` legs of
``bench.py`` may import it.  The product library never calls it, shares no code
with it, and has no CPU fallback.

Everything here is plain numpy in float64 (float32 only where the method itself
fixes float32: the scale factors and the quotient that is rounded to E4M3).

Sources (the web pages this library is built from):

* "Lesson 13: DeepSeek DeepGEMM core architecture and Hopper FP8 kernel
  breakdown" (hpc.payai.win, cuda/lesson13_deepgemm) -- cited as *Lesson 13*:
  Fig. 13-1 (the 1x128 / 128x128 scaling and the per-K-block formula),
  Fig. 13-3 (contiguous and masked MoE layouts), the practice exercise (block
  GEMM simulator and its test) and the answers to Q1 and Q3.
* "DeepGEMM architecture deep dive" (blog.123qwe.co.kr, 2026-10) -- cited as
  *Deep dive*: section 3 (NT convention, scale layout, contiguous alignment,
  the three grouped GEMM families).

Modules
-------
``e4m3``   the 256-code E4M3 table and round-to-nearest-even encoding.
``bf16``   round-to-nearest-even of float64 values to bfloat16.
``quant``  1x128 activation and 128x128 weight quantization (FP32 or
           power-of-two scales).
``gemm``   the block-scaled NT GEMM, its accumulating form, its m-grouped
           contiguous and masked forms and the k-grouped contiguous form.
``ue8m0``  UE8M0 (power-of-two) scale codes and the packed 4-per-int32,
           MN-major scale layout.

Every function is pinned by ``tests/test_oracle_*.py`` against something other
than itself (closed forms, brute force, library conversions, the page's worked
exercise).  No function here is "parity unpinned".
"""

from . import bf16, e4m3, gemm, quant, ue8m0  # noqa: F401
