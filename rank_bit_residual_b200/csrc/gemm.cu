// gemm.cu - the residual GEMM with the low-rank epilogue (INT grid).
//
// "SVDQuant Smoothing, Low-rank and Residual Quantization", Formula item 3:
//   Y = (X_hat L1) L2 + Q(X_hat) Q(R)
// evaluated from prepared operands as
//   Y[b, n] = s_x s_w * sum_k cx[b, k] cw[n, k] + sum_j down[b, j] lu[n, j] (+ bias[n])
// where the integer product runs on tcgen05 kind::i8 (int8 x int8 -> exact int32
// in TMEM) and the up-projection down . lu^T is a second, small kind::f16 MMA
// into its own fp32 TMEM accumulator, so the low-rank branch costs no pass
// over Y. `down` holds hi | lo bf16 halves of the fp32 down-projection and `lu`
// holds the up factor twice, so one K = 2 r MMA chain sums hi.lu + lo.lu.
//
// Persistent kernel, one CTA per SM, 128 x 256 output tiles, 6 warps:
//   warp 0     TMA producer (4-stage ring of 48 KB: A 128x128 B, B 256x128 B)
//   warp 1     TMEM allocation and the single MMA-issuing thread
//   warps 2-5  epilogue: TMEM -> registers -> dequantise + up + bias -> global
// The low-rank K steps go through the same ring as the integer K steps.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "internal.h"
#include "ptx.cuh"

namespace svdq {

namespace {

constexpr int kBM = 128;
constexpr int kBN = 256;
constexpr int kStages = 4;
constexpr int kABytes = kBM * 128;
constexpr int kBBytes = kBN * 128;
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kGemmThreads = 192;
constexpr uint32_t kTmemCols = 512;  // [0,256) int32 residual acc, [256,512) fp32 low-rank acc

enum OutKind { kOutF32 = 0, kOutBF16 = 1, kOutI32 = 2 };

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);  // a -> low half
  return *reinterpret_cast<const uint32_t*>(&h);
}

template <int kOut>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_int_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                    const __grid_constant__ CUtensorMap tm_da, const __grid_constant__ CUtensorMap tm_lu,
                    int B, int N, int M, int lr_steps, const float* __restrict__ s_x,
                    const float* __restrict__ s_w, const __nv_bfloat16* __restrict__ bias,
                    void* __restrict__ y, int64_t ldy, int vec_ok, unsigned* status) {
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
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int tiles_m = (B + kBM - 1) / kBM;
  const int tiles_n = (N + kBN - 1) / kBN;
  const int total = tiles_m * tiles_n;
  const int ksteps = (M + 127) / 128;
  const int steps_per_tile = lr_steps + ksteps;

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
          mbar_arrive_expect_tx(&full_bar[s], kStageBytes);
          if (j < lr_steps) {
            tma_load_2d(st, &tm_da, &full_bar[s], 64 * j, m0);
            tma_load_2d(st + kABytes, &tm_lu, &full_bar[s], 64 * j, n0);
          } else {
            const int k = j - lr_steps;
            tma_load_2d(st, &tm_a, &full_bar[s], 128 * k, m0);
            tma_load_2d(st + kABytes, &tm_b, &full_bar[s], 128 * k, n0);
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
      uint32_t it = 0, lt = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x, ++lt) {
        ok = mbar_wait(&tmem_empty_bar, (lt & 1) ^ 1, status, &abort_sh);
        if (!ok) break;
        tc_fence_after();
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
              mma_f16(tmem + 256, smem_desc_sw128(a0 + 32 * kk), smem_desc_sw128(b0 + 32 * kk),
                      id_bf, (j > 0 || kk > 0) ? 1u : 0u);
          } else {
            const int k = j - lr_steps;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_i8(tmem, smem_desc_sw128(a0 + 32 * kk), smem_desc_sw128(b0 + 32 * kk), id_i8,
                     (k > 0 || kk > 0) ? 1u : 0u);
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
    const float alpha = kOut == kOutI32 ? 0.0f : __ldg(s_x) * __ldg(s_w);
    uint32_t lt = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x, ++lt) {
      if (!mbar_wait(&tmem_full_bar, lt & 1, status, &abort_sh)) break;
      tc_fence_after();
      const int m0 = (t % tiles_m) * kBM;
      const int n0 = (t / tiles_m) * kBN;
      const int row = m0 + r_in;
      const uint32_t lane_addr = tmem + (static_cast<uint32_t>(q * 32) << 16);
      for (int c0 = 0; c0 < kBN; c0 += 32) {
        __syncwarp();  // the TMEM loads below are warp-collective
        uint32_t acc[32], up[32];
        tmem_ld_32x32b_x32(lane_addr + c0, acc);
        if (kOut != kOutI32 && lr_steps) tmem_ld_32x32b_x32(lane_addr + 256 + c0, up);
        tmem_ld_wait();
        const int n = n0 + c0;
        if (row >= B || n >= N) continue;
        const bool full = vec_ok && (n + 32 <= N);
        if (kOut == kOutI32) {
          int32_t* dst = static_cast<int32_t*>(y) + static_cast<int64_t>(row) * ldy + n;
          if (full) {
#pragma unroll
            for (int j = 0; j < 32; j += 4)
              *reinterpret_cast<uint4*>(dst + j) = make_uint4(acc[j], acc[j + 1], acc[j + 2], acc[j + 3]);
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (n + j < N) dst[j] = static_cast<int32_t>(acc[j]);
          }
          continue;
        }
        float v[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          v[j] = alpha * static_cast<float>(static_cast<int32_t>(acc[j]));
          if (lr_steps) v[j] += __uint_as_float(up[j]);
        }
        if (bias != nullptr) {
          if (n + 32 <= N) {
            const uint4* bp = reinterpret_cast<const uint4*>(bias + n);
#pragma unroll
            for (int g = 0; g < 4; ++g) {
              const uint4 bb = __ldg(bp + g);
              const uint32_t w4[4] = {bb.x, bb.y, bb.z, bb.w};
#pragma unroll
              for (int h = 0; h < 4; ++h) {
                v[8 * g + 2 * h] += __uint_as_float(w4[h] << 16);
                v[8 * g + 2 * h + 1] += __uint_as_float(w4[h] & 0xFFFF0000u);
              }
            }
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (n + j < N) v[j] += __bfloat162float(bias[n + j]);
          }
        }
        if (kOut == kOutF32) {
          float* dst = static_cast<float*>(y) + static_cast<int64_t>(row) * ldy + n;
          if (full) {
#pragma unroll
            for (int j = 0; j < 32; j += 4)
              *reinterpret_cast<float4*>(dst + j) = make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (n + j < N) dst[j] = v[j];
          }
        } else {
          __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(y) + static_cast<int64_t>(row) * ldy + n;
          if (full) {
#pragma unroll
            for (int j = 0; j < 32; j += 8)
              *reinterpret_cast<uint4*>(dst + j) =
                  make_uint4(pack_bf16x2(v[j], v[j + 1]), pack_bf16x2(v[j + 2], v[j + 3]),
                             pack_bf16x2(v[j + 4], v[j + 5]), pack_bf16x2(v[j + 6], v[j + 7]));
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (n + j < N) dst[j] = __float2bfloat16_rn(v[j]);
          }
        }
      }
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

}  // namespace

cudaError_t launch_gemm_int(const svdq_weight* w, const int8_t* act_codes, const float* s_x,
                            const void* down2, int64_t B, const void* bias, void* y,
                            svdq_dtype ydt, int64_t ldy, bool raw_i32, cudaStream_t stream,
                            bool* bad_args) {
  *bad_args = false;
  if (B == 0) return cudaSuccess;
  const int64_t M = w->M, N = w->N;
  const int rp = w->rank_pad;
  const bool has_lr = !raw_i32 && rp > 0 && down2 != nullptr;
  CUtensorMap tm_a, tm_b, tm_da, tm_lu;
  bool ok = make_tmap_2d(&tm_a, act_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, M, B, M, 128, kBM, true) &&
            make_tmap_2d(&tm_b, w->codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, M, N, M, 128, kBN, true);
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
  const int lr_steps = has_lr ? static_cast<int>(ceil_div(2 * rp, 64)) : 0;
  const int elem = raw_i32 ? 4 : (ydt == SVDQ_F32 ? 4 : 2);
  const int vec_ok = ((reinterpret_cast<uintptr_t>(y) & 15) == 0 && (ldy * elem) % 16 == 0) ? 1 : 0;
  const int64_t tiles = ceil_div(B, kBM) * ceil_div(N, kBN);
  const int grid = static_cast<int>(std::min<int64_t>(tiles, num_sms()));
  const size_t smem = static_cast<size_t>(kStages) * kStageBytes + 1024;
  unsigned* status = device_status_word();
  const float* sw = w->w_scale;
  const __nv_bfloat16* bb = static_cast<const __nv_bfloat16*>(raw_i32 ? nullptr : bias);
  cudaError_t err;
#define SVDQ_LAUNCH_GEMM(K)                                                                        \
  err = cudaFuncSetAttribute(gemm_int_kernel<K>, cudaFuncAttributeMaxDynamicSharedMemorySize,       \
                             static_cast<int>(smem));                                               \
  if (err != cudaSuccess) return err;                                                               \
  gemm_int_kernel<K><<<grid, kGemmThreads, smem, stream>>>(                                         \
      tm_a, tm_b, tm_da, tm_lu, static_cast<int>(B), static_cast<int>(N), static_cast<int>(M),      \
      lr_steps, s_x, sw, bb, y, ldy, vec_ok, status);
  if (raw_i32) {
    SVDQ_LAUNCH_GEMM(kOutI32)
  } else if (ydt == SVDQ_F32) {
    SVDQ_LAUNCH_GEMM(kOutF32)
  } else {
    SVDQ_LAUNCH_GEMM(kOutBF16)
  }
#undef SVDQ_LAUNCH_GEMM
  return cudaGetLastError();
}

}  // namespace svdq
