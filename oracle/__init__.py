"""CPU oracle for the FP8 per-tensor delayed-scaling linear.

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import, call or
execute this package: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.

It is a plain, slow, obviously-correct restatement of what the method
computes, written with numpy in float64 (float32 only where the method fixes
float32: the product ``x * scale`` and the two scale divisions).  It shares
no code with the CUDA path.

Sources (the AstrAI commit-log pages):

* "AstrAI commits, branch main, tests/extension" -- the FP8 recipe/ring
  commit (last block folds amax into the history window and publishes the
  next scale), the quantize split commit (E4M3/E5M2 fmt enum, bf16/fp16/fp32
  inputs), the snapshot commit (the GEMM dequantises with the scale that
  quantize used), the bias-fusion commit (fp32 bias added before one bf16
  rounding), the batched commit (stride-0 broadcast), the bias_scale commit
  (FP8 bias storage dequantised in the epilogue) and the FP8-in/FP8-out
  GEMM commit.
* "AstrAI commit 69f35c46 csrc/kernels/fp8_mm.cu" -- amax is taken over the
  raw, unscaled values.
* "AstrAI commit 5244f1a8 (te-style scaled fp8 training)" on the same page
  -- the amax history ring of 16 steps.  Recipe constants read from it:
  margin 0, FP8_MAX = the largest finite value of the format (448 for
  E4M3, 57344 for E5M2), a zero history maximum keeps the previous scale,
  saturating round-to-nearest-even conversion.
* The FP8 encodings themselves (E4M3 with no infinities, E5M2 IEEE-like)
  follow the OCP 8-bit floating point specification (OFP8).

Modules:
  fp8_formats -- decode table and encoder (RNE + saturation) per format.
  recipe      -- amax, quantize in row/transposed/dual layout, ring fold,
                 current scaling, and the shard cast of data-parallel scaling.
  gemm        -- fp64 scaled GEMM, |a.b| sums and the acceptance bound;
                 FP8 bias dequantisation and the acceptance interval of
                 FP8 output codes and of the output amax.
  bias_grad   -- column sums of the output gradient (the bias gradient).

Parity status: every function is pinned by ``tests/test_oracle_*.py``
except the treatment of NaN inputs and of a non-finite history maximum,
which no workload exercises ("parity unpinned" for those two cases).
"""

from . import fp8_formats, recipe, gemm, bias_grad  # noqa: F401
