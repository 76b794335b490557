// gemm.cu - the residual GEMM with the low-rank epilogue: argument checks
// shared by both kernels and the choice between them.
//
// "SVDQuant Smoothing, Low-rank and Residual Quantization", Formula item 3:
//   Y = (X_hat L1) L2 + Q(X_hat) Q(R)
// evaluated from prepared operands ("flashinfer.gemm.svdquant_linear", step 3:
// residual GEMM with the low-rank up-projection and bias in the epilogue).
//
// INT grid:   Y[b, n] = s_x s_w sum_k cx[b, k] cw[n, k] + sum_j down[b, j] lu[n, j] (+ bias)
//   the integer product on tcgen05 kind::i8 (exact int32 accumulation), the
//   up-projection on kind::f16 into a separate fp32 accumulator.
// NVFP4:      Y[b, n] = (1 / (gs_x gs_w)) (sum_blocks (a sfa)(w sfw) + sum_j down'[b, j] lu[n, j])
//   with down' = down gs_x gs_w written by the activation pass (the alpha fold
//   of the NVFP4 operator's l1_scaled, applied to the down side because gs_x is
//   per call), so both branches share one fp32 accumulator: kind::mxf4nvf4 with
//   scale_vec::4X, the ue4m3 scales copied to TMEM by tcgen05.cp.
// `down` holds hi | lo bf16 halves of the fp32 down-projection and `lu` holds
// the up factor twice, so one K = 2 r MMA chain sums hi.lu + lo.lu.
//
//   B <= 128   gemm_skinny.cu: weight rows on the MMA's M side, split-K
//              clusters over all SMs (the weight stream is the cost)
//   B >  128   gemm_pair.cu: persistent CTA pairs, 256 x 256 tiles
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "gemm_common.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace svdq {

namespace {

// Shared host part: tensor maps, launch geometry, argument block.
template <int kKind>
cudaError_t launch_gemm(const svdq_weight* w, const void* act_codes, const uint8_t* act_sf,
                        const float* s_x, const void* down2, int64_t B, const void* bias, void* y,
                        svdq_dtype ydt, int64_t ldy, bool raw_i32, bool pdl, cudaStream_t stream,
                        bool* bad_args, void* split_ws) {
  *bad_args = false;
  if (B == 0) return cudaSuccess;
  const int64_t M = w->M, N = w->N;
  const int rp = w->rank_pad;
  const bool has_lr = !raw_i32 && rp > 0 && down2 != nullptr;
  GemmArgs args{};
  args.B = static_cast<int>(B);
  args.N = static_cast<int>(N);
  args.M = static_cast<int>(M);
  args.lr_steps = has_lr ? static_cast<int>(ceil_div(2 * rp, 64)) : 0;
  args.s_x = s_x;
  args.s_w = w->w_scale;
  args.bias = static_cast<const __nv_bfloat16*>(raw_i32 ? nullptr : bias);
  args.y = y;
  args.ldy = ldy;
  const int elem = raw_i32 ? 4 : (ydt == SVDQ_F32 ? 4 : 2);
  args.vec_ok = ((reinterpret_cast<uintptr_t>(y) & 15) == 0 && (ldy * elem) % 16 == 0) ? 1 : 0;
  args.sfa = act_sf;
  args.sfb = static_cast<const uint8_t*>(w->sf);
  args.katoms = static_cast<int>(kKind == kKindMxfp4 ? ceil_div(M, 128) : ceil_div(M, 64));
  args.status = device_status_word();
  const int out = raw_i32 ? kOutI32 : (ydt == SVDQ_F32 ? kOutF32 : kOutBF16);
  cudaError_t err = cudaSuccess;
  const bool launched =
      B > 128 ? launch_gemm_pair(kKind, out, args, act_codes, has_lr ? down2 : nullptr, w, split_ws, stream, &err)
              : launch_gemm_skinny(kKind, out, args, act_codes, act_sf, has_lr ? down2 : nullptr, w, pdl, stream,
                                   &err);
  if (!launched) *bad_args = true;
  return err;
}

}  // namespace

cudaError_t launch_gemm_int(const svdq_weight* w, const int8_t* act_codes, const float* s_x,
                            const void* down2, int64_t B, const void* bias, void* y,
                            svdq_dtype ydt, int64_t ldy, bool raw_i32, bool pdl, cudaStream_t stream,
                            bool* bad_args, void* split_ws) {
  return launch_gemm<kKindInt>(w, act_codes, nullptr, s_x, down2, B, bias, y, ydt, ldy, raw_i32, pdl,
                               stream, bad_args, split_ws);
}

cudaError_t launch_gemm_fp4(const svdq_weight* w, const uint8_t* act_codes,
                            const uint8_t* act_sf, const float* gs_x, const void* down2,
                            int64_t B, const void* bias, void* y, svdq_dtype ydt,
                            int64_t ldy, bool pdl, cudaStream_t stream, bool* bad_args, void* split_ws) {
  if (!act_sf || !w->sf || (reinterpret_cast<uintptr_t>(act_sf) & 15) ||
      (reinterpret_cast<uintptr_t>(w->sf) & 15)) {
    *bad_args = true;
    return cudaSuccess;
  }
  if (w->fmt.kind == SVDQ_KIND_MXFP4)
    return launch_gemm<kKindMxfp4>(w, act_codes, act_sf, gs_x, down2, B, bias, y, ydt, ldy, false, pdl,
                                   stream, bad_args, split_ws);
  return launch_gemm<kKindNvfp4>(w, act_codes, act_sf, gs_x, down2, B, bias, y, ydt, ldy, false, pdl,
                                 stream, bad_args, split_ws);
}

}  // namespace svdq
