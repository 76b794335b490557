// gemm.cu - the residual GEMM with the low-rank epilogue.
//
// "SVDQuant Smoothing, Low-rank and Residual Quantization", Formula item 3:
//   Y = (X_hat L1) L2 + Q(X_hat) Q(R)
// evaluated from prepared operands ("flashinfer.gemm.svdquant_linear", step 3:
// residual GEMM with the low-rank up-projection and bias in the epilogue).
//
// INT grid:   Y[b, n] = s_x s_w sum_k cx[b, k] cw[n, k] + sum_j down[b, j] lu[n, j] (+ bias)
//   the integer product runs on tcgen05 kind::i8 (exact int32 in TMEM columns
//   [0, 256)) and the up-projection on kind::f16 into its own fp32 accumulator
//   (columns [256, 512)).
// NVFP4:      Y[b, n] = (1 / (gs_x gs_w)) (sum_blocks (a sfa)(w sfw) + sum_j down'[b, j] lu[n, j])
//   with down' = down gs_x gs_w written by the activation pass (the alpha fold
//   of the NVFP4 operator's l1_scaled, applied to the down side because gs_x
//   is per call), so both branches share one fp32 accumulator (columns
//   [0, 256)) and the block scales take columns [256, 304): kind::mxf4nvf4
//   with scale_vec::4X, the scales copied from shared memory by tcgen05.cp.
// `down` holds hi | lo bf16 halves of the fp32 down-projection and `lu` holds
// the up factor twice, so one K = 2 r MMA chain sums hi.lu + lo.lu.
//
// Persistent kernel, one CTA per SM, 128 x 256 output tiles, 6 warps:
//   warp 0     TMA / bulk-copy producer (4-stage ring)
//   warp 1     TMEM allocation and the single MMA-issuing thread
//   warps 2-5  epilogue: TMEM -> registers -> dequantise (+ up) + bias -> global
// The low-rank K steps go through the same ring as the residual K steps.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "gemm_common.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace svdq {

namespace {

constexpr int kBM = 128;
constexpr int kBN = 256;
constexpr int kStages = 4;
constexpr int kABytes = kBM * 128;
constexpr int kBBytes = kBN * 128;
constexpr int kSfaBytes = 4 * 512;       // 4 scale atoms (128 rows x 4 blocks each)
constexpr int kSfbBytes = 2 * 4 * 512;   // two 128-row tiles of B
constexpr int kGemmThreads = 192;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSfaCol = 256;        // NVFP4: scale factors of A, 4 columns per MMA
constexpr uint32_t kSfbCol = 272;        // NVFP4: scale factors of B, 8 columns per MMA

template <int kKind>
struct Cfg {
  static constexpr int kStageBytes =
      kABytes + kBBytes + (kKind == kKindNvfp4 ? kSfaBytes + kSfbBytes : 0);
};

template <int kKind, int kOut>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                const __grid_constant__ CUtensorMap tm_da, const __grid_constant__ CUtensorMap tm_lu,
                const GemmArgs args) {
  constexpr int kStageBytes = Cfg<kKind>::kStageBytes;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[kStages];
  __shared__ __align__(8) uint64_t empty_bar[kStages];
  __shared__ __align__(8) uint64_t tmem_full_bar;
  __shared__ __align__(8) uint64_t tmem_empty_bar;
  __shared__ __align__(8) uint64_t mma_done_bar;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int B = args.B, N = args.N, M = args.M, lr_steps = args.lr_steps;
  unsigned* status = args.status;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int tiles_m = (B + kBM - 1) / kBM;
  const int tiles_n = (N + kBN - 1) / kBN;
  const int total = tiles_m * tiles_n;
  // K elements per 128-byte stage row: 128 int8 or 256 e2m1
  constexpr int kStageK = kKind == kKindNvfp4 ? 256 : 128;
  const int ksteps = (M + kStageK - 1) / kStageK;
  const int steps_per_tile = lr_steps + ksteps;
  const int n_rows_p = ((N + 127) / 128) * 128;  // rows of the weight scale layout

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    mbar_init(&tmem_full_bar, 1);
    mbar_init(&tmem_empty_bar, 4);
    mbar_init(&mma_done_bar, 1);
    fence_mbar_init();
    abort_sh = 0;
    tma_prefetch_desc(&tm_a);
    tma_prefetch_desc(&tm_b);
    if (lr_steps) {
      tma_prefetch_desc(&tm_da);
      tma_prefetch_desc(&tm_lu);
    }
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base_sh, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
        const int m0 = (t % tiles_m) * kBM;
        const int n0 = (t / tiles_m) * kBN;
        for (int j = 0; j < steps_per_tile && ok; ++j, ++it) {
          const int s = it % kStages;
          const uint32_t ph = (it / kStages) & 1;
          ok = mbar_wait(&empty_bar[s], ph ^ 1, status, &abort_sh);
          if (!ok) break;
          uint8_t* st = smem + s * kStageBytes;
          if (j < lr_steps) {
            mbar_arrive_expect_tx(&full_bar[s], kABytes + kBBytes);
            tma_load_2d(st, &tm_da, &full_bar[s], 64 * j, m0);
            tma_load_2d(st + kABytes, &tm_lu, &full_bar[s], 64 * j, n0);
          } else {
            const int k = j - lr_steps;
            if constexpr (kKind == kKindNvfp4) {
              // scale atoms of this stage: one per 64 K elements that exist
              const int a0 = 4 * k;
              const int na = min(4, args.katoms - a0);
              const int nrt = (n0 + 128 < n_rows_p) ? 2 : 1;
              mbar_arrive_expect_tx(&full_bar[s], kABytes + kBBytes + na * 512 * (1 + nrt));
              tma_load_2d(st, &tm_a, &full_bar[s], 128 * k, m0);
              tma_load_2d(st + kABytes, &tm_b, &full_bar[s], 128 * k, n0);
              uint8_t* sfa_s = st + kABytes + kBBytes;
              uint8_t* sfb_s = sfa_s + kSfaBytes;
              bulk_load(sfa_s, args.sfa + (static_cast<int64_t>(m0 / 128) * args.katoms + a0) * 512,
                        na * 512, &full_bar[s]);
              for (int rt = 0; rt < nrt; ++rt)
                bulk_load(sfb_s + rt * 2048,
                          args.sfb + (static_cast<int64_t>(n0 / 128 + rt) * args.katoms + a0) * 512,
                          na * 512, &full_bar[s]);
            } else {
              mbar_arrive_expect_tx(&full_bar[s], kABytes + kBBytes);
              tma_load_2d(st, &tm_a, &full_bar[s], 128 * k, m0);
              tma_load_2d(st + kABytes, &tm_b, &full_bar[s], 128 * k, n0);
            }
          }
        }
      }
      // let the last loads land before this block's shared memory is released
      const uint32_t first = it > static_cast<uint32_t>(kStages) ? it - kStages : 0u;
      for (uint32_t i = first; i < it; ++i)
        mbar_wait(&full_bar[i % kStages], (i / kStages) & 1, status, nullptr);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA
    if (lane == 0) {
      const uint32_t id_i8 = idesc_i8(kBM, kBN);
      const uint32_t id_bf = idesc_bf16(kBM, kBN);
      const uint32_t id_f4 = idesc_nvf4(kBM, kBN);
      // INT: low-rank into its own fp32 accumulator; NVFP4: everything into one
      const uint32_t lr_acc = kKind == kKindNvfp4 ? tmem : tmem + 256;
      {
        // throwaway MMA: the first tcgen05.mma of a kernel takes microseconds
        // longer than the rest; issued now, that start-up overlaps the first
        // loads (the first real MMA of the tile overwrites the accumulator)
        const uint64_t d0 = smem_desc_sw128(smem_u32(smem));
        if constexpr (kKind == kKindNvfp4)
          mma_nvf4(tmem, d0, d0, id_f4, 0u, tmem + kSfaCol, tmem + kSfbCol);
        else
          mma_i8(tmem, d0, d0, id_i8, 0u);
      }
      uint32_t it = 0, lt = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x, ++lt) {
        ok = mbar_wait(&tmem_empty_bar, (lt & 1) ^ 1, status, &abort_sh);
        if (!ok) break;
        tc_fence_after();
        const int n0 = (t / tiles_m) * kBN;
        for (int j = 0; j < steps_per_tile; ++j, ++it) {
          const int s = it % kStages;
          const uint32_t ph = (it / kStages) & 1;
          ok = mbar_wait(&full_bar[s], ph, status, &abort_sh);
          if (!ok) break;
          tc_fence_after();
          const uint32_t a0 = smem_u32(smem + s * kStageBytes);
          const uint32_t b0 = a0 + kABytes;
          if (j < lr_steps) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_f16(lr_acc, smem_desc_sw128(a0 + 32 * kk), smem_desc_sw128(b0 + 32 * kk), id_bf,
                      (j > 0 || kk > 0) ? 1u : 0u);
          } else {
            const int k = j - lr_steps;
            if constexpr (kKind == kKindNvfp4) {
              const int na = min(4, args.katoms - 4 * k);
              const int nrt = (n0 + 128 < n_rows_p) ? 2 : 1;
              const uint32_t sfa_s = b0 + kBBytes;
              const uint32_t sfb_s = sfa_s + kSfaBytes;
              // scale atoms -> TMEM; tcgen05.cp and tcgen05.mma issued by one
              // thread execute in order, so the columns can be reused per stage
              for (int kk = 0; kk < na; ++kk) {
                tmem_cp_32x128b_warpx4(tmem + kSfaCol + 4 * kk, smem_desc_plain(sfa_s + 512 * kk));
                for (int rt = 0; rt < nrt; ++rt)
                  tmem_cp_32x128b_warpx4(tmem + kSfbCol + 8 * kk + 4 * rt,
                                         smem_desc_plain(sfb_s + 2048 * rt + 512 * kk));
              }
              for (int kk = 0; kk < na; ++kk)
                mma_nvf4(tmem, smem_desc_sw128(a0 + 32 * kk), smem_desc_sw128(b0 + 32 * kk), id_f4,
                         (lr_steps > 0 || k > 0 || kk > 0) ? 1u : 0u, tmem + kSfaCol + 4 * kk,
                         tmem + kSfbCol + 8 * kk);
            } else {
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                mma_i8(tmem, smem_desc_sw128(a0 + 32 * kk), smem_desc_sw128(b0 + 32 * kk), id_i8,
                       (k > 0 || kk > 0) ? 1u : 0u);
            }
          }
          mma_commit(&empty_bar[s]);
        }
        if (!ok) break;
        mma_commit(&tmem_full_bar);
      }
      // wait for every MMA this thread issued before TMEM is released
      mma_commit(&mma_done_bar);
      mbar_wait(&mma_done_bar, 0, status, nullptr);
    }
  } else {
    // ----------------------------------------------------------- epilogue
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    const int r_in = q * 32 + lane;
    const float alpha = epilogue_alpha<kKind, kOut>(args);
    const bool sep_lr = kKind == kKindInt && kOut != kOutI32 && lr_steps > 0;
    uint32_t lt = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x, ++lt) {
      if (!mbar_wait_warp(&tmem_full_bar, lt & 1, status, &abort_sh)) break;
      tc_fence_after();
      const int m0 = (t % tiles_m) * kBM;
      const int n0 = (t / tiles_m) * kBN;
      const uint32_t lane_addr = tmem + (static_cast<uint32_t>(q * 32) << 16);
      epilogue_slab<kKind, kOut>(args, lane_addr, m0 + r_in, n0, alpha, sep_lr);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tmem_empty_bar);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int kKind, int kOut>
cudaError_t launch_one(const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& da,
                       const CUtensorMap& lu, const GemmArgs& args, int grid, cudaStream_t st) {
  const size_t smem = static_cast<size_t>(kStages) * Cfg<kKind>::kStageBytes + 1024;
  cudaError_t err = cudaFuncSetAttribute(gemm_kernel<kKind, kOut>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
  if (err != cudaSuccess) return err;
  gemm_kernel<kKind, kOut><<<grid, kGemmThreads, smem, st>>>(a, b, da, lu, args);
  return cudaGetLastError();
}

// Shared host part: tensor maps, launch geometry, argument block.
template <int kKind>
cudaError_t launch_gemm(const svdq_weight* w, const void* act_codes, const uint8_t* act_sf,
                        const float* s_x, const void* down2, int64_t B, const void* bias, void* y,
                        svdq_dtype ydt, int64_t ldy, bool raw_i32, bool pdl, cudaStream_t stream,
                        bool* bad_args) {
  *bad_args = false;
  if (B == 0) return cudaSuccess;
  const int64_t M = w->M, N = w->N;
  const int rp = w->rank_pad;
  const bool has_lr = !raw_i32 && rp > 0 && down2 != nullptr;
  // codes rows are 128 bytes per K step: M int8 or M/2 packed e2m1 bytes
  const int64_t row_bytes = kKind == kKindNvfp4 ? M / 2 : M;
  CUtensorMap tm_a, tm_b, tm_da, tm_lu;
  bool ok =
      make_tmap_2d(&tm_a, act_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, row_bytes, B, row_bytes, 128, kBM, true) &&
      make_tmap_2d(&tm_b, w->codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, row_bytes, N, row_bytes, 128, kBN, true);
  if (ok && has_lr) {
    ok = make_tmap_2d(&tm_da, down2, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, 2 * rp, B, 2 * rp, 64, kBM, true) &&
         make_tmap_2d(&tm_lu, w->lu, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, 2 * rp, N, 2 * rp, 64, kBN, true);
  } else {
    tm_da = tm_a;
    tm_lu = tm_b;
  }
  if (!ok) {
    *bad_args = true;
    return cudaSuccess;
  }
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
  args.katoms = static_cast<int>(ceil_div(M, 64));
  args.status = device_status_word();
  // more than one 128-row block: CTA pairs (256 x 256 tiles)
  if (B > kBM) {
    cudaError_t err = cudaSuccess;
    const int out = raw_i32 ? kOutI32 : (ydt == SVDQ_F32 ? kOutF32 : kOutBF16);
    if (launch_gemm_pair(kKind, out, args, act_codes, has_lr ? down2 : nullptr, w, stream, &err))
      return err;
    *bad_args = true;
    return cudaSuccess;
  }
  {
    // short batch: split-K clusters over all SMs (gemm_skinny.cu)
    cudaError_t err = cudaSuccess;
    const int out = raw_i32 ? kOutI32 : (ydt == SVDQ_F32 ? kOutF32 : kOutBF16);
    if (launch_gemm_skinny(kKind, out, args, act_codes, act_sf, has_lr ? down2 : nullptr, w, pdl, stream, &err))
      return err;
    *bad_args = true;
    return cudaSuccess;
  }
  const int64_t tiles = ceil_div(B, kBM) * ceil_div(N, kBN);
  const int grid = static_cast<int>(std::min<int64_t>(tiles, num_sms()));
  if (raw_i32) {
    if constexpr (kKind == kKindInt) {
      return launch_one<kKind, kOutI32>(tm_a, tm_b, tm_da, tm_lu, args, grid, stream);
    } else {
      *bad_args = true;
      return cudaSuccess;
    }
  }
  if (ydt == SVDQ_F32) return launch_one<kKind, kOutF32>(tm_a, tm_b, tm_da, tm_lu, args, grid, stream);
  return launch_one<kKind, kOutBF16>(tm_a, tm_b, tm_da, tm_lu, args, grid, stream);
}

}  // namespace

cudaError_t launch_gemm_int(const svdq_weight* w, const int8_t* act_codes, const float* s_x,
                            const void* down2, int64_t B, const void* bias, void* y,
                            svdq_dtype ydt, int64_t ldy, bool raw_i32, bool pdl, cudaStream_t stream,
                            bool* bad_args) {
  return launch_gemm<kKindInt>(w, act_codes, nullptr, s_x, down2, B, bias, y, ydt, ldy, raw_i32, pdl,
                               stream, bad_args);
}

cudaError_t launch_gemm_nvfp4(const svdq_weight* w, const uint8_t* act_codes,
                              const uint8_t* act_sf, const float* gs_x, const void* down2,
                              int64_t B, const void* bias, void* y, svdq_dtype ydt,
                              int64_t ldy, bool pdl, cudaStream_t stream, bool* bad_args) {
  if (!act_sf || !w->sf || (reinterpret_cast<uintptr_t>(act_sf) & 15) ||
      (reinterpret_cast<uintptr_t>(w->sf) & 15)) {
    *bad_args = true;
    return cudaSuccess;
  }
  return launch_gemm<kKindNvfp4>(w, act_codes, act_sf, gs_x, down2, B, bias, y, ydt, ldy, false, pdl,
                                 stream, bad_args);
}

}  // namespace svdq
