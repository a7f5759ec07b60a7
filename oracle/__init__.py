"""CPU oracle for the routed-expert FFN over packed STQ1_0 / MXFP4 weights.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  The CUDA library never calls it and shares no code with it: every
value here is computed from the format definitions in plain numpy, with float64
arithmetic, in the order the definitions state.

Sources (page titles as they appear in the reference material):

* "Hy4-preview-GGUF" (AngelSlim), section 3 "STQ1_0 and the mixed-precision
  strategy": ternary {-d, 0, +d}, exactly one zero per four lanes, a 5-bit
  pattern per group, one FP16 scale per 256 weights, 42 bytes per 256 weights;
  the upstream quantizer sets d = amax and zeroes argmin |x|.
* "Hy4-preview-FlashMoE-STQ1_0" (anemll), "How the STQ1_0 packing works":
  64 four-weight groups per block, 4 x 2^3 = 32 patterns, five bits each;
  "Package details": hidden 6144, MoE intermediate 2048, 256 experts, top-8,
  one shared expert.
* "Hy4-preview-SF-WFP4AFP8" (siliconflow), "Quant Diff" table: routed experts
  are FP4 E2M1 weights with FP8 E4M3 activations, group 32, UE8M0 scales.

The bit-level definitions of E4M3 / E2M1 / UE8M0 follow the OCP Microscaling
specification (the pages name the formats but not their bits).

Parity status: every function here is pinned by the ``-m "not gpu"`` tests in
``tests/test_oracle_*.py`` (closed forms, brute force, invariants, library
routines for IEEE rounding, and the byte totals the pages print).
"""

from . import formats, moe  # noqa: F401
