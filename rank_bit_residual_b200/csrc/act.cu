// act.cu - the activation pass of the SVDQuant linear.
//
// "SVDQuant Smoothing, Low-rank and Residual Quantization", Formula items 1
// and 3: X_hat = x / scale is quantised per tensor (INT grid, or NVFP4 blocks
// for the variant of "flashinfer.gemm.svdquant_linear" step 1), and the
// low-rank branch needs X_hat L1 = x ld^T (step 2 of that page) in the same
// pass over x.
//
// Two kernels:
//   act_stats_kernel  reads x once through TMA (128-byte swizzled tiles). Per
//                     tile it issues the down-projection MMA (tcgen05, bf16 or
//                     tf32 in, fp32 in TMEM) and takes column maxima of |x|
//                     from the same shared-memory tile. Since fl(a / s) is
//                     monotone in a, max_b fl(|x_bk| / s_k) = fl(max_b |x_bk| / s_k):
//                     one IEEE division per column instead of per element.
//                     Grid = row blocks of 128 x K splits; each CTA writes a
//                     partial max and a partial down tile (fp32).
//   act_quant_*       re-reads x (L2-resident after the first kernel), reduces
//                     the partial maxima to the per-tensor scale and writes the
//                     codes; it also sums the partial down tiles and writes them
//                     as bf16 hi | lo for the GEMM's low-rank MMA.
// fp32 evaluation order (the one the oracle's fp32 code mode repeats): the
// per-element divisions of the definition are multiplies by correctly rounded
// reciprocals, r_k = fl(1 / scale_k) once per column and u = fl(1 / s) once
// per tensor: X_hat = fl(x r_k), code = rint(fl(X_hat u)).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "internal.h"
#include "ptx.cuh"

namespace svdq {

namespace {

constexpr int kActThreads = 128;
constexpr int kActStages = 4;
constexpr int kRowsPerBlock = 128;
constexpr int kTileBytes = kRowsPerBlock * 128;  // one 128 x 128-byte x tile
constexpr int kRowsPerThread = 8;     // INT quantise: rows in flight per thread
constexpr int kRowsPerThreadF4 = 4;   // NVFP4 quantise: rows in flight per thread

__host__ __device__ constexpr uint32_t pow2_cols(int n) {
  return n <= 32 ? 32u : n <= 64 ? 64u : n <= 128 ? 128u : 256u;
}

// Column maxima of |x| over the 128-row tile for this thread's 16-byte chunk
// (rows rg, rg+16, ..., rg+112), then fold fl(colmax / scale) into `run`.
template <typename TIn>
__device__ __forceinline__ float tile_absmax(const uint8_t* tile, const float* __restrict__ scale,
                                             int kbase, int M, float run) {
  const int tid = threadIdx.x;
  const int c = tid & 7;     // logical 16-byte chunk of the 128-byte row
  const int rg = tid >> 3;   // row group 0..15
  const int p = c ^ (rg & 7);  // physical chunk position under the 128-byte swizzle
  uint32_t mx0 = 0, mx1 = 0, mx2 = 0, mx3 = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int r = rg + 16 * i;
    const uint4 v = *reinterpret_cast<const uint4*>(tile + r * 128 + p * 16);
    if constexpr (sizeof(TIn) == 2) {
      mx0 = __vmaxu2(mx0, v.x & 0x7FFF7FFFu);
      mx1 = __vmaxu2(mx1, v.y & 0x7FFF7FFFu);
      mx2 = __vmaxu2(mx2, v.z & 0x7FFF7FFFu);
      mx3 = __vmaxu2(mx3, v.w & 0x7FFF7FFFu);
    } else {
      mx0 = max(mx0, v.x & 0x7FFFFFFFu);
      mx1 = max(mx1, v.y & 0x7FFFFFFFu);
      mx2 = max(mx2, v.z & 0x7FFFFFFFu);
      mx3 = max(mx3, v.w & 0x7FFFFFFFu);
    }
  }
  const uint32_t mx[4] = {mx0, mx1, mx2, mx3};
  if constexpr (sizeof(TIn) == 2) {
#pragma unroll
    for (int w = 0; w < 4; ++w) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int k = kbase + 8 * c + 2 * w + h;
        if (k < M) {
          const uint32_t bits = h ? (mx[w] & 0xFFFF0000u) : (mx[w] << 16);
          run = fmaxf(run, __fmul_rn(__uint_as_float(bits), __frcp_rn(__ldg(scale + k))));
        }
      }
    }
  } else {
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const int k = kbase + 4 * c + w;
      if (k < M) run = fmaxf(run, __fmul_rn(__uint_as_float(mx[w]), __frcp_rn(__ldg(scale + k))));
    }
  }
  return run;
}

template <typename TIn>
__global__ void __launch_bounds__(kActThreads, 1)
    act_stats_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_ld,
                     const float* __restrict__ scale, int B, int M, int nsteps, int ksplit,
                     int rank_pad, int has_ld, float* __restrict__ ws_down,
                     float* __restrict__ ws_max, unsigned* status) {
  constexpr int kTileK = 128 / static_cast<int>(sizeof(TIn));
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[kActStages];
  __shared__ __align__(8) uint64_t mma_bar[kActStages];
  __shared__ __align__(8) uint64_t final_bar;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;
  __shared__ float red_sh[kActThreads / 32];

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int ld_bytes = rank_pad * 128;
  const int stage_bytes = kTileBytes + (has_ld ? ld_bytes : 0);
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int m0 = blockIdx.x * kRowsPerBlock;
  const int sp = blockIdx.y;
  const int k_lo = static_cast<int>((static_cast<int64_t>(nsteps) * sp) / ksplit);
  const int k_hi = static_cast<int>((static_cast<int64_t>(nsteps) * (sp + 1)) / ksplit);
  const int n = k_hi - k_lo;
  const uint32_t tcols = pow2_cols(rank_pad);

  if (tid == 0) {
    for (int s = 0; s < kActStages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&mma_bar[s], 1);
    }
    mbar_init(&final_bar, 1);
    fence_mbar_init();
    abort_sh = 0;
    tma_prefetch_desc(&tm_x);
    if (has_ld) tma_prefetch_desc(&tm_ld);
  }
  if (has_ld && warp == 0) {
    tmem_alloc(&tmem_base_sh, tcols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = has_ld ? tmem_base_sh : 0u;

  auto issue = [&](int i) {
    const int s = i % kActStages;
    uint8_t* st = smem + s * stage_bytes;
    mbar_arrive_expect_tx(&full_bar[s], stage_bytes);
    const int kc = (k_lo + i) * kTileK;
    tma_load_2d(st, &tm_x, &full_bar[s], kc, m0);
    if (has_ld) tma_load_2d(st + kTileBytes, &tm_ld, &full_bar[s], kc, 0);
  };

  if (tid == 0) {
    for (int i = 0; i < min(n, kActStages); ++i) issue(i);
  }

  const uint32_t idesc = sizeof(TIn) == 2 ? idesc_bf16(128, rank_pad) : idesc_tf32(128, rank_pad);
  float run = 0.0f;
  int issued = min(n, kActStages);
  int consumed = 0;
  bool ok_all = true;
  // Every thread runs every iteration (and its __syncthreads) even after a
  // failed wait: a failure only turns the work of the remaining steps off.
  for (int i = 0; i < n; ++i) {
    const int s = i % kActStages;
    const uint32_t ph = (i / kActStages) & 1;
    ok_all = ok_all && mbar_wait(&full_bar[s], ph, status, &abort_sh);
    if (ok_all) consumed = i + 1;
    uint8_t* st = smem + s * stage_bytes;
    if (ok_all && has_ld && tid == 0) {
      tc_fence_after();
      const uint32_t a0 = smem_u32(st);
      const uint32_t b0 = smem_u32(st + kTileBytes);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint64_t ad = smem_desc_sw128(a0 + 32 * kk);
        const uint64_t bd = smem_desc_sw128(b0 + 32 * kk);
        if (sizeof(TIn) == 2)
          mma_f16(tmem, ad, bd, idesc, (i > 0 || kk > 0) ? 1u : 0u);
        else
          mma_tf32(tmem, ad, bd, idesc, (i > 0 || kk > 0) ? 1u : 0u);
      }
      mma_commit(&mma_bar[s]);
    }
    if (ok_all) run = tile_absmax<TIn>(st, scale, (k_lo + i) * kTileK, M, run);
    __syncthreads();
    if (tid == 0 && ok_all && issued < n && !abort_sh) {
      bool ok = true;
      if (has_ld) ok = mbar_wait(&mma_bar[s], ph, status, &abort_sh);
      if (ok) {
        issue(issued);
        ++issued;
      }
    }
  }

  // After a failed wait, let the loads already issued land before the shared
  // memory they target is released (bounded like every other wait).
  if (tid == 0) {
    for (int i = consumed; i < issued; ++i)
      mbar_wait(&full_bar[i % kActStages], (i / kActStages) & 1, status, nullptr);
  }

  // Partial down tile: TMEM lane = row, one fp32 column per factor column.
  if (has_ld) {
    if (tid == 0) mma_commit(&final_bar);
    const bool ok = mbar_wait(&final_bar, 0, status, nullptr) && ok_all;
    tc_fence_after();
    const int row = m0 + warp * 32 + lane;
    float* dst = ws_down + (static_cast<int64_t>(sp) * B + row) * rank_pad;
    for (int c0 = 0; c0 < rank_pad; c0 += 32) {
      uint32_t v[32];
      tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(warp * 32) << 16) + c0, v);
      tmem_ld_wait();
      if (ok && row < B) {
        const int cnt = min(32, rank_pad - c0);
        for (int j = 0; j < cnt; j += 4) {
          *reinterpret_cast<float4*>(dst + c0 + j) =
              make_float4(__uint_as_float(v[j]), __uint_as_float(v[j + 1]),
                          __uint_as_float(v[j + 2]), __uint_as_float(v[j + 3]));
        }
      }
    }
  }

  // Partial per-tensor maximum of |X_hat|.
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) run = fmaxf(run, __shfl_xor_sync(0xffffffffu, run, o));
  if (lane == 0) red_sh[warp] = run;
  tc_fence_before();
  __syncthreads();
  if (tid == 0) {
    float m = red_sh[0];
    for (int w = 1; w < kActThreads / 32; ++w) m = fmaxf(m, red_sh[w]);
    ws_max[static_cast<int64_t>(sp) * gridDim.x + blockIdx.x] = m;
  }
  if (has_ld && warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, tcols);
  }
}

__device__ __forceinline__ float block_max_of_parts(const float* __restrict__ parts, int nparts,
                                                    float* red) {
  float m = 0.0f;
  for (int i = threadIdx.x; i < nparts; i += blockDim.x) m = fmaxf(m, parts[i]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = red[0];
    for (int w = 1; w < static_cast<int>(blockDim.x >> 5); ++w) t = fmaxf(t, red[w]);
    red[0] = t;
  }
  __syncthreads();
  return red[0];
}

template <typename TIn>
__device__ __forceinline__ void load8(const TIn* __restrict__ p, float (&v)[8]) {
  if constexpr (sizeof(TIn) == 2) {
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      v[2 * j] = __uint_as_float(w[j] << 16);
      v[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
    }
  } else {
    const float4 a = __ldg(reinterpret_cast<const float4*>(p));
    const float4 b = __ldg(reinterpret_cast<const float4*>(p + 4));
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  }
}

__device__ __forceinline__ void load8_scale(const float* __restrict__ p, float (&v)[8]) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(p));
  const float4 b = __ldg(reinterpret_cast<const float4*>(p + 4));
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

// Sum the K-split partial down tiles, multiply by `mult` and store bf16 hi | lo.
__device__ __forceinline__ void finalize_down(const float* __restrict__ ws_down, int ksplit,
                                              int B, int rank_pad, __nv_bfloat16* down,
                                              float mult) {
  const int64_t total = static_cast<int64_t>(B) * rank_pad;
  const int64_t nblk = static_cast<int64_t>(gridDim.x) * gridDim.y;
  const int64_t bid = static_cast<int64_t>(blockIdx.y) * gridDim.x + blockIdx.x;
  for (int64_t i = bid * blockDim.x + threadIdx.x; i < total; i += nblk * blockDim.x) {
    const int64_t row = i / rank_pad;
    const int j = static_cast<int>(i - row * rank_pad);
    float v = 0.0f;
    for (int sp = 0; sp < ksplit; ++sp) v += ws_down[(static_cast<int64_t>(sp) * B + row) * rank_pad + j];
    v = __fmul_rn(v, mult);
    const __nv_bfloat16 hi = __float2bfloat16_rn(v);
    const __nv_bfloat16 lo = __float2bfloat16_rn(v - __bfloat162float(hi));
    down[row * 2 * rank_pad + j] = hi;
    down[row * 2 * rank_pad + rank_pad + j] = lo;
  }
}

// 2-D grid: blockIdx.x picks 32 chunks of 8 columns (one per lane), blockIdx.y a
// band of rows; warp ty takes rows ty, ty + 8, ... of the band. A warp reads one
// 512-byte run of a row per step; the reciprocals are taken once per thread.
template <typename TIn>
__global__ void __launch_bounds__(256)
    act_quant_int_kernel(const TIn* __restrict__ x, int64_t ldx, const float* __restrict__ scale,
                         int B, int M, int qmax, int rows_per_block,
                         const float* __restrict__ ws_max, int nparts,
                         const float* __restrict__ ws_down, int ksplit, int rank_pad,
                         int8_t* __restrict__ codes, __nv_bfloat16* __restrict__ down,
                         float* __restrict__ act_scale) {
  __shared__ float red[8];
  const float m = block_max_of_parts(ws_max, nparts, red);
  const float s = __fdiv_rn(m, static_cast<float>(qmax));
  const float u = s > 0.0f ? __frcp_rn(s) : 0.0f;
  if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) *act_scale = s;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  const int cc = blockIdx.x * 32 + tx;
  if (cc < M / 8) {
    const int k0 = cc * 8;
    float r[8];
    load8_scale(scale + k0, r);
#pragma unroll
    for (int j = 0; j < 8; ++j) r[j] = __frcp_rn(r[j]);
    const int row0 = blockIdx.y * rows_per_block + ty;
    // rows row0, row0 + 8, ... : all loads of a group are in flight before the math
    for (int g = 0; g < rows_per_block; g += 8 * kRowsPerThread) {
      float xv[kRowsPerThread][8];
#pragma unroll
      for (int i = 0; i < kRowsPerThread; ++i) {
        const int row = row0 + g + 8 * i;
        if (row < B) load8<TIn>(x + static_cast<int64_t>(row) * ldx + k0, xv[i]);
      }
#pragma unroll
      for (int i = 0; i < kRowsPerThread; ++i) {
        const int row = row0 + g + 8 * i;
        if (row >= B) continue;
        uint32_t packed[2] = {0u, 0u};
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          int q = __float2int_rn(__fmul_rn(__fmul_rn(xv[i][j], r[j]), u));
          q = min(max(q, -qmax), qmax);
          packed[j >> 2] |= (static_cast<uint32_t>(q) & 0xFFu) << (8 * (j & 3));
        }
        *reinterpret_cast<uint2*>(codes + static_cast<int64_t>(row) * M + k0) =
            make_uint2(packed[0], packed[1]);
      }
    }
  }
  if (rank_pad > 0 && down != nullptr) finalize_down(ws_down, ksplit, B, rank_pad, down, 1.0f);
}

// ------------------------------------------------------------------ NVFP4
__device__ __forceinline__ uint8_t f32_to_ue4m3(float v) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(v));
  return static_cast<uint8_t>(r & 0xFFu);
}

// Exact value of a non-negative e4m3 byte (bias 7; exponent 0 is subnormal).
__device__ __forceinline__ float ue4m3_to_f32(uint8_t b) {
  const uint32_t e = (b >> 3) & 0xFu, m = b & 7u;
  return e == 0 ? static_cast<float>(m) * 0.001953125f  // m * 2^-9
                : __uint_as_float(((e + 120u) << 23) | (m << 20));
}

// Eight floats -> eight e2m1 nibbles, element j in nibble j (low nibble first).
__device__ __forceinline__ uint32_t f32x8_to_e2m1(const float (&v)[8]) {
  uint32_t out;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(out)
      : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
  // a code whose magnitude is zero is stored as +0
  const uint32_t mag = out & 0x77777777u;
  const uint32_t nz = (mag + 0x77777777u) & 0x88888888u;
  return out & (0x77777777u | nz);
}

__device__ __forceinline__ int64_t sf_swizzle_offset(int64_t row, int64_t col, int64_t kbp) {
  return ((row >> 7) * (kbp >> 2) + (col >> 2)) * 512 + (row & 31) * 16 + ((row & 127) >> 5) * 4 +
         (col & 3);
}

// 2-D grid like the INT kernel, one thread per 16-element block of a row.
template <typename TIn>
__global__ void __launch_bounds__(256)
    act_quant_nvfp4_kernel(const TIn* __restrict__ x, int64_t ldx, const float* __restrict__ scale,
                           int B, int M, int rows_per_block, const float* __restrict__ ws_max,
                           int nparts, const float* __restrict__ gs_given,
                           const float* __restrict__ gs_w, const float* __restrict__ ws_down,
                           int ksplit, int rank_pad, uint8_t* __restrict__ codes,
                           uint8_t* __restrict__ sf, __nv_bfloat16* __restrict__ down,
                           float* __restrict__ act_scale) {
  __shared__ float red[8];
  const float m = block_max_of_parts(ws_max, nparts, red);
  float gs;
  if (gs_given != nullptr)
    gs = __ldg(gs_given);
  else
    gs = m > 0.0f ? __fdiv_rn(2688.0f, m) : 1.0f;
  if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) *act_scale = gs;
  const int kb = M / 16;
  const int64_t kbp = (kb + 3) / 4 * 4;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  const int b = blockIdx.x * 32 + tx;
  if (b < kb) {
    const int k0 = b * 16;
    float r[16];
    {
      float t[8];
      load8_scale(scale + k0, t);
#pragma unroll
      for (int j = 0; j < 8; ++j) r[j] = __frcp_rn(t[j]);
      load8_scale(scale + k0 + 8, t);
#pragma unroll
      for (int j = 0; j < 8; ++j) r[8 + j] = __frcp_rn(t[j]);
    }
    const int row0 = blockIdx.y * rows_per_block + ty;
    for (int g = 0; g < rows_per_block; g += 8 * kRowsPerThreadF4) {
      float xv[kRowsPerThreadF4][16];
#pragma unroll
      for (int i = 0; i < kRowsPerThreadF4; ++i) {
        const int row = row0 + g + 8 * i;
        if (row < B) {
          load8<TIn>(x + static_cast<int64_t>(row) * ldx + k0, *reinterpret_cast<float(*)[8]>(&xv[i][0]));
          load8<TIn>(x + static_cast<int64_t>(row) * ldx + k0 + 8, *reinterpret_cast<float(*)[8]>(&xv[i][8]));
        }
      }
#pragma unroll
      for (int i = 0; i < kRowsPerThreadF4; ++i) {
        const int row = row0 + g + 8 * i;
        if (row >= B) continue;
        float xs[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) xs[j] = __fmul_rn(xv[i][j], r[j]);
        float amax = 0.0f;
#pragma unroll
        for (int j = 0; j < 16; ++j) amax = fmaxf(amax, fabsf(xs[j]));
        const uint8_t sfb = f32_to_ue4m3(__fmul_rn(__fdiv_rn(amax, 6.0f), gs));
        const float d = ue4m3_to_f32(sfb);
        const float enc = d > 0.0f ? __fdiv_rn(gs, d) : 0.0f;
        float lo[8], hi[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          lo[j] = __fmul_rn(xs[j], enc);
          hi[j] = __fmul_rn(xs[8 + j], enc);
        }
        *reinterpret_cast<uint2*>(codes + static_cast<int64_t>(row) * (M / 2) + b * 8) =
            make_uint2(f32x8_to_e2m1(lo), f32x8_to_e2m1(hi));
        sf[sf_swizzle_offset(row, b, kbp)] = sfb;
      }
    }
  }
  // zero the scale padding (rows up to a multiple of 128, columns up to 4)
  const int64_t rows_p = (static_cast<int64_t>(B) + 127) / 128 * 128;
  const int64_t nblk = static_cast<int64_t>(gridDim.x) * gridDim.y;
  const int64_t bid = static_cast<int64_t>(blockIdx.y) * gridDim.x + blockIdx.x;
  for (int64_t i = bid * blockDim.x + threadIdx.x; i < rows_p * kbp; i += nblk * blockDim.x) {
    const int64_t row = i / kbp;
    const int64_t c = i - row * kbp;
    if (row >= B || c >= kb) sf[sf_swizzle_offset(row, c, kbp)] = 0;
  }
  // down in the units of the NVFP4 GEMM accumulator: x ld^T gs_x gs_w (gs_w when given)
  if (rank_pad > 0 && down != nullptr)
    finalize_down(ws_down, ksplit, B, rank_pad, down,
                  gs_w != nullptr ? __fmul_rn(gs, __ldg(gs_w)) : gs);
}

}  // namespace

ActPlan plan_act(int64_t B, int64_t M, int32_t rank_pad, svdq_dtype xdt) {
  ActPlan p{};
  p.B = B;
  p.M = M;
  p.rank_pad = rank_pad;
  p.tile_k = xdt == SVDQ_BF16 ? 64 : 32;
  p.nrb = static_cast<int>(ceil_div(B, kRowsPerBlock));
  p.nsteps = static_cast<int>(ceil_div(M, p.tile_k));
  // one wave: two CTAs per SM (shared memory allows two), split K to fill it
  const int target = 2 * num_sms();
  int ks = target / std::max(p.nrb, 1);
  ks = std::max(1, std::min(ks, p.nsteps));
  p.ksplit = ks;
  p.nparts = p.nrb * p.ksplit;
  return p;
}

size_t act_scratch_bytes(const ActPlan& p) {
  size_t b = static_cast<size_t>(round_up(static_cast<int64_t>(p.nparts) * 4, 256));
  if (p.rank_pad > 0)
    b += static_cast<size_t>(round_up(static_cast<int64_t>(p.ksplit) * p.B * p.rank_pad * 4, 256));
  return b + 256;
}

cudaError_t launch_act(const ActPlan& p, const void* x, svdq_dtype xdt, int64_t ldx,
                       const float* scale, svdq_fmt fmt, const float* act_global_scale,
                       const float* w_global_scale, const void* ld, void* codes, void* sf,
                       float* act_scale, void* down, void* scratch, cudaStream_t stream,
                       bool* bad_args) {
  *bad_args = false;
  if (p.B == 0) return cudaSuccess;
  const bool has_ld = ld != nullptr && p.rank_pad > 0 && down != nullptr;
  Carver cv(scratch, ~size_t(0));
  float* ws_max = static_cast<float*>(cv.take(static_cast<size_t>(p.nparts) * 4));
  float* ws_down =
      has_ld ? static_cast<float*>(cv.take(static_cast<size_t>(p.ksplit) * p.B * p.rank_pad * 4))
             : nullptr;
  const int esz = xdt == SVDQ_BF16 ? 2 : 4;
  const CUtensorMapDataType cdt =
      xdt == SVDQ_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  CUtensorMap tm_x, tm_ld;
  if (!make_tmap_2d(&tm_x, x, cdt, esz, p.M, p.B, ldx, p.tile_k, kRowsPerBlock, true)) {
    *bad_args = true;
    return cudaSuccess;
  }
  if (has_ld) {
    if (!make_tmap_2d(&tm_ld, ld, cdt, esz, p.M, p.rank_pad, p.M, p.tile_k, p.rank_pad, true)) {
      *bad_args = true;
      return cudaSuccess;
    }
  } else {
    tm_ld = tm_x;
  }
  unsigned* status = device_status_word();
  const int stage_bytes = kTileBytes + (has_ld ? p.rank_pad * 128 : 0);
  const size_t smem = static_cast<size_t>(kActStages) * stage_bytes + 1024;
  dim3 grid(p.nrb, p.ksplit);
  cudaError_t err;
  if (xdt == SVDQ_BF16) {
    err = cudaFuncSetAttribute(act_stats_kernel<__nv_bfloat16>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (err != cudaSuccess) return err;
    act_stats_kernel<__nv_bfloat16><<<grid, kActThreads, smem, stream>>>(
        tm_x, tm_ld, scale, static_cast<int>(p.B), static_cast<int>(p.M), p.nsteps, p.ksplit,
        p.rank_pad, has_ld ? 1 : 0, ws_down, ws_max, status);
  } else {
    err = cudaFuncSetAttribute(act_stats_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(smem));
    if (err != cudaSuccess) return err;
    act_stats_kernel<float><<<grid, kActThreads, smem, stream>>>(
        tm_x, tm_ld, scale, static_cast<int>(p.B), static_cast<int>(p.M), p.nsteps, p.ksplit,
        p.rank_pad, has_ld ? 1 : 0, ws_down, ws_max, status);
  }
  err = cudaGetLastError();
  if (err != cudaSuccess) return err;

  // quantise: 32 column chunks per block along x, a band of rows along y, sized
  // for about eight blocks per SM
  const int chunk = fmt.kind == SVDQ_KIND_INT ? 8 : 16;
  const int gx = static_cast<int>(ceil_div(p.M / chunk, 32));
  const int64_t want_blocks = static_cast<int64_t>(num_sms()) * 8;
  const int64_t rows_step = 8 * (fmt.kind == SVDQ_KIND_INT ? kRowsPerThread : kRowsPerThreadF4);
  int64_t rows_per_block =
      round_up(std::max<int64_t>(1, ceil_div(p.B * gx, want_blocks)), rows_step);
  const int gy = static_cast<int>(ceil_div(p.B, rows_per_block));
  dim3 qgrid(gx, gy);
  const int threads = 256;
  __nv_bfloat16* down_bf = has_ld ? static_cast<__nv_bfloat16*>(down) : nullptr;
  const int rp = has_ld ? p.rank_pad : 0;
  const int rpb = static_cast<int>(rows_per_block);
  if (fmt.kind == SVDQ_KIND_INT) {
    const int qmax = (1 << (fmt.bits - 1)) - 1;
    if (xdt == SVDQ_BF16)
      act_quant_int_kernel<__nv_bfloat16><<<qgrid, threads, 0, stream>>>(
          static_cast<const __nv_bfloat16*>(x), ldx, scale, static_cast<int>(p.B),
          static_cast<int>(p.M), qmax, rpb, ws_max, p.nparts, ws_down, p.ksplit, rp,
          static_cast<int8_t*>(codes), down_bf, act_scale);
    else
      act_quant_int_kernel<float><<<qgrid, threads, 0, stream>>>(
          static_cast<const float*>(x), ldx, scale, static_cast<int>(p.B), static_cast<int>(p.M),
          qmax, rpb, ws_max, p.nparts, ws_down, p.ksplit, rp, static_cast<int8_t*>(codes),
          down_bf, act_scale);
  } else {
    if (xdt == SVDQ_BF16)
      act_quant_nvfp4_kernel<__nv_bfloat16><<<qgrid, threads, 0, stream>>>(
          static_cast<const __nv_bfloat16*>(x), ldx, scale, static_cast<int>(p.B),
          static_cast<int>(p.M), rpb, ws_max, p.nparts, act_global_scale, w_global_scale,
          ws_down, p.ksplit, rp, static_cast<uint8_t*>(codes), static_cast<uint8_t*>(sf), down_bf,
          act_scale);
    else
      act_quant_nvfp4_kernel<float><<<qgrid, threads, 0, stream>>>(
          static_cast<const float*>(x), ldx, scale, static_cast<int>(p.B), static_cast<int>(p.M),
          rpb, ws_max, p.nparts, act_global_scale, w_global_scale, ws_down, p.ksplit, rp,
          static_cast<uint8_t*>(codes), static_cast<uint8_t*>(sf), down_bf, act_scale);
  }
  return cudaGetLastError();
}

}  // namespace svdq
