"""CPU oracle for the SVDQuant inference linear.

TEST INFRASTRUCTURE ONLY. This package is a plain, slow, float64 restatement
of what the operator computes, written from the defining pages:

* "SVDQuant Smoothing, Low-rank and Residual Quantization" (paperleet.com):
  the function contracts (smooth_inputs, split_weight, svdquant_linear,
  fake_quantize, _check_smoothing, _check_rank) and "Formula and conventions"
  items 1-3 with the two-branch equation Y = (X_hat L1) L2 + Q(X_hat) Q(R).
* "flashinfer.gemm.svdquant_linear" (docs.flashinfer.ai): the NVFP4 operator's
  parameter list (packed e2m1 residual, ue4m3 block scales in a 128x4 swizzled
  layout, per-tensor fp32 scales, bf16 factors with the smoothing folded in).

Only the tests, the package entry point's smoke check and the bench's CPU
baseline leg may import it. The CUDA library never does, shares no code with
it, and has no CPU fallback that could route through it.

Modules
-------
svdquant   page-1 contract in float64 (exact mode)
codes      the fp32 op order that integer codes are compared in bit-exactly
nvfp4      e2m1 / e4m3 formats, block quantisation, the 128x4 scale layout
prepared   the linear evaluated from prepared (stored) operands

Parity pins live in tests/test_oracle_*.py. The NVFP4 global/block scale
recipe (gs = 448*6/amax, sf = e4m3(amax_b/6*gs)) is not printed on any page:
it is pinned only by format definitions and internal consistency, i.e.
"parity unpinned" as far as the pages go.
"""

from . import svdquant, codes, nvfp4, prepared  # noqa: F401
