// act.cu - the activation pass of the SVDQuant linear, one cooperative kernel.
//
// "SVDQuant Smoothing, Low-rank and Residual Quantization", Formula items 1
// and 3: X_hat = x / scale is quantised per tensor (INT grid, or NVFP4 blocks
// for the variant of "flashinfer.gemm.svdquant_linear" step 1), and the
// low-rank branch needs X_hat L1 = x ld^T (step 2 of that page) from the same
// read of x.
//
// Work unit = 128 rows x a range of 128-byte K tiles. Phase 1 streams the
// unit's x tiles in by TMA (128-byte swizzle), runs the down-projection on
// tcgen05 (bf16, or tf32 for fp32 x, accumulated in TMEM) and takes column
// maxima of |x| from the same shared-memory tiles; it writes a partial down
// tile and a partial maximum. Since fl(a r) is monotone in a, the tensor
// maximum of |X_hat| is max_k fl(colmax_k r_k). A bounded grid barrier then
// makes the per-tensor scale known everywhere, and phase 2 writes the codes:
// from the tiles still held in shared memory when the unit fits there (x is
// then read from HBM exactly once), else by re-reading the unit from global
// memory. Phase 2 also sums the partial down tiles into bf16 hi | lo.
//
// fp32 evaluation order (the one the oracle's fp32 code mode repeats): the
// per-element divisions of the definition are multiplies by correctly rounded
// reciprocals, r_k = fl(1 / scale_k) once per column and u = fl(1 / s) once
// per tensor: X_hat = fl(x r_k), INT code = rint(fl(x c_k)) with the per-column
// constant c_k = fl(r_k u).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "internal.h"
#include "ptx.cuh"

namespace svdq {

namespace {

constexpr int kThreads = 512;
constexpr int kRows = 128;                  // rows per unit (MMA M)
constexpr int kTileBytes = kRows * 128;     // one 128 x 128-byte x tile
constexpr int kRing = 4;                    // ring depth for ld tiles (and x tiles when not held)
constexpr int kMaxHold = 12;                // x tiles a unit may keep in shared memory
constexpr int kSmemBudget = 224 * 1024;

__host__ __device__ constexpr uint32_t pow2_cols(int n) {
  return n <= 32 ? 32u : n <= 64 ? 64u : n <= 128 ? 128u : 256u;
}

struct ActArgs {
  int B, M;
  int64_t ldx;
  int nsteps, ksplit, nrb, nunits, rank_pad, has_ld, hold, xbuf, fmt_kind, qmax;
  const void* x;
  const float* scale;
  const float* gs_given;
  const float* gs_w;
  float* ws_down;   // [ksplit][B][rank_pad]
  float* ws_max;    // [gridDim.x]
  unsigned* sync;   // [0] barrier counter, [1] abort flag (zeroed before launch)
  void* codes;
  uint8_t* sf;
  __nv_bfloat16* down;
  float* act_scale;
  unsigned* status;
};

// ------------------------------------------------------------- small helpers
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

// Eight floats -> eight e2m1 nibbles, element j in nibble j (low nibble first);
// a code whose magnitude is zero is stored as +0.
__device__ __forceinline__ uint32_t f32x8_to_e2m1(const float* v) {
  uint32_t out;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(out)
      : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
  const uint32_t mag = out & 0x77777777u;
  const uint32_t nz = (mag + 0x77777777u) & 0x88888888u;
  return out & (0x77777777u | nz);
}

__device__ __forceinline__ int64_t sf_swizzle_offset(int64_t row, int64_t col, int64_t kbp) {
  return ((row >> 7) * (kbp >> 2) + (col >> 2)) * 512 + (row & 31) * 16 + ((row & 127) >> 5) * 4 +
         (col & 3);
}

// 16 bytes of x as floats: 8 bf16 or 4 fp32
template <typename TIn>
__device__ __forceinline__ void unpack16(const uint4 u, float* v) {
  if constexpr (sizeof(TIn) == 2) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      v[2 * j] = __uint_as_float(w[j] << 16);
      v[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
    }
  } else {
    v[0] = __uint_as_float(u.x);
    v[1] = __uint_as_float(u.y);
    v[2] = __uint_as_float(u.z);
    v[3] = __uint_as_float(u.w);
  }
}

// Column maxima of |x| over a 128 x 128-byte swizzled tile. Thread t owns the
// logical 16-byte chunk c = t % 8 of rows t/8 and t/8 + 64; it folds
// fl(colmax r_k) of its chunk's columns into `run` (rcp: reciprocals of the
// tile's columns, 0 past M).
template <typename TIn>
__device__ __forceinline__ float tile_absmax(const uint8_t* tile, const float* rcp, float run) {
  const int tid = threadIdx.x;
  const int c = tid & 7;
  const int rg = tid >> 3;
  const int p = c ^ (rg & 7);  // rows rg + 64 i share rg & 7
  uint32_t mx[4] = {0u, 0u, 0u, 0u};
#pragma unroll
  for (int i = 0; i < kRows / (kThreads / 8); ++i) {
    const uint4 v = *reinterpret_cast<const uint4*>(tile + (rg + (kThreads / 8) * i) * 128 + p * 16);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      if constexpr (sizeof(TIn) == 2)
        mx[q] = __vmaxu2(mx[q], w[q] & 0x7FFF7FFFu);
      else
        mx[q] = max(mx[q], w[q] & 0x7FFFFFFFu);
    }
  }
  if constexpr (sizeof(TIn) == 2) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      run = fmaxf(run, __fmul_rn(__uint_as_float(mx[q] << 16), rcp[8 * c + 2 * q]));
      run = fmaxf(run, __fmul_rn(__uint_as_float(mx[q] & 0xFFFF0000u), rcp[8 * c + 2 * q + 1]));
    }
  } else {
#pragma unroll
    for (int q = 0; q < 4; ++q) run = fmaxf(run, __fmul_rn(__uint_as_float(mx[q]), rcp[4 * c + q]));
  }
  return run;
}

// -------------------------------------------------------------- the kernel
template <typename TIn>
__global__ void __launch_bounds__(kThreads, 1)
    act_fused_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_ld,
                     const ActArgs a) {
  constexpr int kTileK = 128 / static_cast<int>(sizeof(TIn));   // elements per 128-byte row
  constexpr int kPerChunk = 16 / static_cast<int>(sizeof(TIn)); // elements per 16 bytes
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t xfull[kMaxHold];
  __shared__ __align__(8) uint64_t ldfull[kRing];
  __shared__ __align__(8) uint64_t mmadone[kRing];
  __shared__ __align__(8) uint64_t final_bar;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;
  __shared__ float red[kThreads / 32];

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int ld_bytes = a.rank_pad * 128;
  uint8_t* xbuf = smem;                                               // a.xbuf tiles
  uint8_t* ldbuf = smem + static_cast<size_t>(a.xbuf) * kTileBytes;   // kRing ld tiles
  float* rcp = reinterpret_cast<float*>(ldbuf + (a.has_ld ? kRing * ld_bytes : 0));
  const uint32_t tcols = pow2_cols(a.rank_pad);
  unsigned* status = a.status;

  if (tid == 0) {
    for (int s = 0; s < kMaxHold; ++s) mbar_init(&xfull[s], 1);
    for (int s = 0; s < kRing; ++s) {
      mbar_init(&ldfull[s], 1);
      mbar_init(&mmadone[s], 1);
    }
    mbar_init(&final_bar, 1);
    fence_mbar_init();
    abort_sh = 0;
    tma_prefetch_desc(&tm_x);
    if (a.has_ld) tma_prefetch_desc(&tm_ld);
  }
  if (a.has_ld && warp == 0) {
    tmem_alloc(&tmem_base_sh, tcols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = a.has_ld ? tmem_base_sh : 0u;
  const uint32_t idesc = sizeof(TIn) == 2 ? idesc_bf16(128, a.rank_pad) : idesc_tf32(128, a.rank_pad);

  // barrier uses so far (phase parities carry across units)
  uint32_t xuse[kMaxHold] = {};
  uint32_t lduse = 0;
  uint32_t final_use = 0;
  float run = 0.0f;
  bool ok = true;

  // ================================================================ phase 1
  for (int unit = blockIdx.x; unit < a.nunits; unit += gridDim.x) {
    const int rb = unit % a.nrb, sp = unit / a.nrb;
    const int m0 = rb * kRows;
    const int k_lo = static_cast<int>((static_cast<int64_t>(a.nsteps) * sp) / a.ksplit);
    const int k_hi = static_cast<int>((static_cast<int64_t>(a.nsteps) * (sp + 1)) / a.ksplit);
    const int n = k_hi - k_lo;
    for (int j = tid; j < n * kTileK; j += kThreads) {
      const int col = k_lo * kTileK + j;
      rcp[j] = col < a.M ? __frcp_rn(__ldg(a.scale + col)) : 0.0f;
    }
    __syncthreads();
    const uint32_t ld0 = lduse;
    auto issue_x = [&](int i) {
      const int b = i % a.xbuf;
      mbar_arrive_expect_tx(&xfull[b], kTileBytes);
      tma_load_2d(xbuf + static_cast<size_t>(b) * kTileBytes, &tm_x, &xfull[b], (k_lo + i) * kTileK, m0);
    };
    auto issue_ld = [&](int i) {
      const uint32_t q = (ld0 + i) % kRing;
      mbar_arrive_expect_tx(&ldfull[q], ld_bytes);
      tma_load_2d(ldbuf + static_cast<size_t>(q) * ld_bytes, &tm_ld, &ldfull[q], (k_lo + i) * kTileK, 0);
    };
    if (tid == 0 && ok) {
      for (int i = 0; i < min(n, a.xbuf); ++i) issue_x(i);
      if (a.has_ld)
        for (int i = 0; i < min(n, kRing); ++i) issue_ld(i);
    }
    // Step i reads x buffer i % xbuf and ld slot (ld0 + i) % kRing. At step i,
    // thread 0 refills the buffers step i - 1 used (its MMA was issued a step
    // ago, so the wait for it is normally already satisfied).
    for (int i = 0; i < n; ++i) {
      const int b = i % a.xbuf;
      const uint32_t q = (ld0 + i) % kRing;
      ok = ok && mbar_wait(&xfull[b], xuse[b] & 1, status, &abort_sh);
      ++xuse[b];
      if (a.has_ld && tid == 0) {
        ok = ok && mbar_wait(&ldfull[q], ((ld0 + i) / kRing) & 1, status, &abort_sh);
        if (ok) {
          tc_fence_after();
          const uint32_t a0 = smem_u32(xbuf + static_cast<size_t>(b) * kTileBytes);
          const uint32_t b0 = smem_u32(ldbuf + static_cast<size_t>(q) * ld_bytes);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ad = smem_desc_sw128(a0 + 32 * kk);
            const uint64_t bd = smem_desc_sw128(b0 + 32 * kk);
            if (sizeof(TIn) == 2)
              mma_f16(tmem, ad, bd, idesc, (i > 0 || kk > 0) ? 1u : 0u);
            else
              mma_tf32(tmem, ad, bd, idesc, (i > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(&mmadone[q]);
        }
      }
      if (ok) run = tile_absmax<TIn>(xbuf + static_cast<size_t>(b) * kTileBytes, rcp + i * kTileK, run);
      __syncthreads();
      if (tid == 0 && ok && i >= 1) {
        const int jl = i - 1 + kRing;     // ld step that takes over slot of step i - 1
        const int jx = i - 1 + a.xbuf;    // x step that takes over buffer of step i - 1
        const bool need_ld = a.has_ld && jl < n;
        const bool need_x = !a.hold && jx < n;
        if (a.has_ld && (need_ld || need_x))
          ok = mbar_wait(&mmadone[(ld0 + i - 1) % kRing], ((ld0 + i - 1) / kRing) & 1, status,
                         &abort_sh);
        if (ok && need_ld) issue_ld(jl);
        if (ok && need_x) issue_x(jx);
      }
    }
    if (a.has_ld) lduse += n;
    if (a.has_ld) {
      if (tid == 0) mma_commit(&final_bar);
      const bool fin = mbar_wait(&final_bar, final_use & 1, status, nullptr);
      ++final_use;
      tc_fence_after();
      // TMEM lane = row; warps 0-3 cover the 128 lanes (one lane quarter each)
      if (warp < 4) {
        const int row = m0 + warp * 32 + lane;
        float* dst = a.ws_down + (static_cast<int64_t>(sp) * a.B + row) * a.rank_pad;
        for (int c0 = 0; c0 < a.rank_pad; c0 += 32) {
          uint32_t v[32];
          tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(warp * 32) << 16) + c0, v);
          tmem_ld_wait();
          if (fin && ok && row < a.B) {
            const int cnt = min(32, a.rank_pad - c0);
            for (int j = 0; j < cnt; j += 4)
              *reinterpret_cast<float4*>(dst + c0 + j) =
                  make_float4(__uint_as_float(v[j]), __uint_as_float(v[j + 1]),
                              __uint_as_float(v[j + 2]), __uint_as_float(v[j + 3]));
          }
        }
      }
      tc_fence_before();
      __syncthreads();
    }
  }
  // a failed wait: let loads already issued land before the block moves on
  if (tid == 0 && !ok) {
    for (int s = 0; s < min(a.xbuf, kMaxHold); ++s)
      mbar_wait(&xfull[s], xuse[s] & 1, status, nullptr, 1000000ull);
  }
  // per-CTA maximum -> ws_max[blockIdx.x]
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) run = fmaxf(run, __shfl_xor_sync(0xffffffffu, run, o));
  if (lane == 0) red[warp] = run;
  __syncthreads();
  if (tid == 0) {
    float m = red[0];
    for (int w = 1; w < kThreads / 32; ++w) m = fmaxf(m, red[w]);
    a.ws_max[blockIdx.x] = m;
  }

  // ======================================================== grid barrier
  GridSync gs{a.sync, a.sync + 1, status, 0};
  ok = grid_sync(gs, &abort_sh) && ok;

  // ================================================================ phase 2
  if (ok) {
    float m = 0.0f;
    for (int i = tid; i < static_cast<int>(gridDim.x); i += kThreads) m = fmaxf(m, a.ws_max[i]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    __syncthreads();
    if (lane == 0) red[warp] = m;
    __syncthreads();
    m = red[0];
    for (int w = 1; w < kThreads / 32; ++w) m = fmaxf(m, red[w]);
    const bool nv = a.fmt_kind == SVDQ_KIND_NVFP4;
    float s = 0.0f, u = 0.0f, gs_x = 1.0f;
    if (nv) {
      gs_x = a.gs_given != nullptr ? __ldg(a.gs_given) : (m > 0.0f ? __fdiv_rn(2688.0f, m) : 1.0f);
    } else {
      s = __fdiv_rn(m, static_cast<float>(a.qmax));
      u = s > 0.0f ? __frcp_rn(s) : 0.0f;
    }
    if (blockIdx.x == 0 && tid == 0) *a.act_scale = nv ? gs_x : s;
    const int kb = a.M / 16;
    const int64_t kbp = (kb + 3) / 4 * 4;

    for (int unit = blockIdx.x; unit < a.nunits; unit += gridDim.x) {
      const int rb = unit % a.nrb, sp = unit / a.nrb;
      const int m0 = rb * kRows;
      const int k_lo = static_cast<int>((static_cast<int64_t>(a.nsteps) * sp) / a.ksplit);
      const int k_hi = static_cast<int>((static_cast<int64_t>(a.nsteps) * (sp + 1)) / a.ksplit);
      const int n = k_hi - k_lo;
      if (!a.hold) {
        __syncthreads();
        for (int j = tid; j < n * kTileK; j += kThreads) {
          const int col = k_lo * kTileK + j;
          rcp[j] = col < a.M ? __frcp_rn(__ldg(a.scale + col)) : 0.0f;
        }
        __syncthreads();
      }
      const int rows = min(kRows, a.B - m0);
      // the unit's 16-byte chunk (row r, logical chunk c) of tile t
      auto chunk = [&](int t, int r, int c) -> uint4 {
        if (a.hold)
          return *reinterpret_cast<const uint4*>(xbuf + static_cast<size_t>(t) * kTileBytes + r * 128 +
                                                 ((c ^ (r & 7)) * 16));
        return __ldg(reinterpret_cast<const uint4*>(static_cast<const TIn*>(a.x) +
                                                    static_cast<int64_t>(m0 + r) * a.ldx +
                                                    (k_lo + t) * kTileK + c * kPerChunk));
      };
      if (!nv) {
        // thread -> chunk c of rows r0, r0 + 64 of every tile; c_k = fl(r_k u) per column
        const int c = tid & 7, r0 = tid >> 3;
        for (int t = 0; t < n; ++t) {
          const int col = (k_lo + t) * kTileK + c * kPerChunk;
          if (col >= a.M) continue;
          float ck[kPerChunk];
#pragma unroll
          for (int j = 0; j < kPerChunk; ++j) ck[j] = __fmul_rn(rcp[t * kTileK + c * kPerChunk + j], u);
          uint4 raw[kRows / (kThreads / 8)];
#pragma unroll
          for (int i = 0; i < kRows / (kThreads / 8); ++i) {
            const int r = r0 + (kThreads / 8) * i;
            if (r < rows) raw[i] = chunk(t, r, c);
          }
#pragma unroll
          for (int i = 0; i < kRows / (kThreads / 8); ++i) {
            const int r = r0 + (kThreads / 8) * i;
            if (r >= rows) continue;
            float v[kPerChunk];
            unpack16<TIn>(raw[i], v);
            uint32_t packed[2] = {0u, 0u};
#pragma unroll
            for (int j = 0; j < kPerChunk; ++j) {
              int qv = __float2int_rn(__fmul_rn(v[j], ck[j]));
              qv = min(max(qv, -a.qmax), a.qmax);
              packed[j >> 2] |= (static_cast<uint32_t>(qv) & 0xFFu) << (8 * (j & 3));
            }
            int8_t* dst = static_cast<int8_t*>(a.codes) + static_cast<int64_t>(m0 + r) * a.M + col;
            if constexpr (kPerChunk == 8)
              *reinterpret_cast<uint2*>(dst) = make_uint2(packed[0], packed[1]);
            else
              *reinterpret_cast<uint32_t*>(dst) = packed[0];
          }
        }
      } else {
        // thread -> 16-element block b of row r of every tile
        constexpr int kBlk = kTileK / 16;                 // blocks per tile row
        constexpr int kChunksPerBlk = 16 / kPerChunk;
        constexpr int kRowsPerPass = kThreads / kBlk;     // rows covered per pass
        const int bk = tid % kBlk, r0 = tid / kBlk;
        for (int t = 0; t < n; ++t) {
          const int col = (k_lo + t) * kTileK + bk * 16;
          if (col >= a.M) continue;
          for (int r = r0; r < rows; r += kRowsPerPass) {
            float xs[16];
#pragma unroll
            for (int h = 0; h < kChunksPerBlk; ++h) {
              unpack16<TIn>(chunk(t, r, bk * kChunksPerBlk + h), xs + h * kPerChunk);
            }
            float amax = 0.0f;
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              xs[j] = __fmul_rn(xs[j], rcp[t * kTileK + bk * 16 + j]);
              amax = fmaxf(amax, fabsf(xs[j]));
            }
            const uint8_t sfb = f32_to_ue4m3(__fmul_rn(__fdiv_rn(amax, 6.0f), gs_x));
            const float d = ue4m3_to_f32(sfb);
            const float enc = d > 0.0f ? __fdiv_rn(gs_x, d) : 0.0f;
#pragma unroll
            for (int j = 0; j < 16; ++j) xs[j] = __fmul_rn(xs[j], enc);
            const int row = m0 + r;
            *reinterpret_cast<uint2*>(static_cast<uint8_t*>(a.codes) + static_cast<int64_t>(row) * (a.M / 2) +
                                      col / 2) = make_uint2(f32x8_to_e2m1(xs), f32x8_to_e2m1(xs + 8));
            a.sf[sf_swizzle_offset(row, col / 16, kbp)] = sfb;
          }
        }
      }
      // down: this unit's share of the row block's rows, all K splits summed
      if (a.has_ld && a.down != nullptr) {
        const int r_lo = (kRows * sp) / a.ksplit, r_hi = (kRows * (sp + 1)) / a.ksplit;
        const float mult = nv ? (a.gs_w != nullptr ? __fmul_rn(gs_x, __ldg(a.gs_w)) : gs_x) : 1.0f;
        const int cnt = (r_hi - r_lo) * a.rank_pad;
        for (int i = tid; i < cnt; i += kThreads) {
          const int rr = r_lo + i / a.rank_pad, j = i % a.rank_pad;
          const int row = m0 + rr;
          if (row >= a.B) continue;
          float acc = 0.0f;
          for (int z = 0; z < a.ksplit; ++z)
            acc += a.ws_down[(static_cast<int64_t>(z) * a.B + row) * a.rank_pad + j];
          acc = __fmul_rn(acc, mult);
          const __nv_bfloat16 hi = __float2bfloat16_rn(acc);
          const __nv_bfloat16 lo = __float2bfloat16_rn(acc - __bfloat162float(hi));
          a.down[static_cast<int64_t>(row) * 2 * a.rank_pad + j] = hi;
          a.down[static_cast<int64_t>(row) * 2 * a.rank_pad + a.rank_pad + j] = lo;
        }
      }
    }
    // NVFP4: zero the scale padding (rows up to a multiple of 128, columns up to 4)
    if (nv) {
      const int64_t rows_p = (static_cast<int64_t>(a.B) + 127) / 128 * 128;
      const int64_t pad_cols = kbp - kb;
      const int64_t n_pad = (rows_p - a.B) * kbp + static_cast<int64_t>(a.B) * pad_cols;
      for (int64_t i = static_cast<int64_t>(blockIdx.x) * kThreads + tid; i < n_pad;
           i += static_cast<int64_t>(gridDim.x) * kThreads) {
        int64_t row, c;
        if (i < static_cast<int64_t>(a.B) * pad_cols) {
          row = i / pad_cols;
          c = kb + (i - row * pad_cols);
        } else {
          const int64_t j = i - static_cast<int64_t>(a.B) * pad_cols;
          row = a.B + j / kbp;
          c = j - (j / kbp) * kbp;
        }
        a.sf[sf_swizzle_offset(row, c, kbp)] = 0;
      }
    }
  }

  __syncthreads();
  if (a.has_ld && warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, tcols);
  }
}

size_t smem_for(const ActPlan& p, int xbuf) {
  const int ld_bytes = p.rank_pad * 128;
  const int steps_max = (p.nsteps + p.ksplit - 1) / p.ksplit;
  return static_cast<size_t>(xbuf) * kTileBytes + (p.rank_pad > 0 ? kRing * ld_bytes : 0) +
         static_cast<size_t>(steps_max) * p.tile_k * sizeof(float) + 1024;
}

// Resident CTAs per SM for a given dynamic shared memory size (at most two:
// each may hold TMEM for its down accumulator).
int resident_per_sm(size_t smem, bool bf16) {
  int n = 0;
  cudaError_t e;
  // the occupancy query honours the kernel's opt-in shared memory limit
  int dev = 0, optin = 0;
  if (cudaGetDevice(&dev) == cudaSuccess &&
      cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) == cudaSuccess &&
      optin > 4096) {
    const int lim = optin - 2048;
    if (bf16)
      cudaFuncSetAttribute(act_fused_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, lim);
    else
      cudaFuncSetAttribute(act_fused_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, lim);
  }
  if (bf16)
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, act_fused_kernel<__nv_bfloat16>, kThreads,
                                                      smem);
  else
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, act_fused_kernel<float>, kThreads, smem);
  if (e != cudaSuccess || n <= 0) n = smem > 110 * 1024 ? 1 : 2;
  return std::max(1, std::min(n, 2));
}

}  // namespace

void finish_act_plan(ActPlan& p) {
  p.nunits = p.nrb * p.ksplit;
  const int steps_max = (p.nsteps + p.ksplit - 1) / p.ksplit;
  // hold the unit's x tiles when they fit and every unit gets a CTA of its own
  p.hold = 0;
  p.xbuf = kRing;
  if (steps_max <= kMaxHold) {
    const size_t sm = smem_for(p, steps_max);
    if (sm <= static_cast<size_t>(kSmemBudget) && p.nunits <= num_sms() * resident_per_sm(sm, p.bf16)) {
      p.hold = 1;
      p.xbuf = steps_max;
    }
  }
  p.smem = smem_for(p, p.xbuf);
  p.grid = std::min(p.nunits, num_sms() * resident_per_sm(p.smem, p.bf16));
  p.nparts = p.grid;
}

ActPlan plan_act(int64_t B, int64_t M, int32_t rank_pad, svdq_dtype xdt) {
  ActPlan p{};
  p.B = B;
  p.M = M;
  p.rank_pad = rank_pad;
  p.bf16 = xdt == SVDQ_BF16;
  p.tile_k = p.bf16 ? 64 : 32;
  p.nrb = static_cast<int>(ceil_div(B, kRows));
  p.nsteps = static_cast<int>(ceil_div(M, p.tile_k));
  // one unit per SM; split K further when that lets each unit's tiles stay in
  // shared memory (then two units share an SM)
  const int sms = num_sms();
  int ks = std::max(1, std::min(p.nsteps, sms / std::max(p.nrb, 1)));
  while (ks < p.nsteps && ceil_div(p.nsteps, ks) > kMaxHold && p.nrb * (ks + 1) <= 2 * sms) ++ks;
  p.ksplit = ks;
  finish_act_plan(p);
  return p;
}

size_t act_scratch_bytes(const ActPlan& p) {
  size_t b = static_cast<size_t>(round_up(static_cast<int64_t>(std::max(p.grid, 1)) * 4, 256));
  b += 256;  // grid barrier words
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
  float* ws_max = static_cast<float*>(cv.take(static_cast<size_t>(std::max(p.grid, 1)) * 4));
  unsigned* sync = static_cast<unsigned*>(cv.take(256));
  float* ws_down =
      has_ld ? static_cast<float*>(cv.take(static_cast<size_t>(p.ksplit) * p.B * p.rank_pad * 4))
             : nullptr;
  const int esz = xdt == SVDQ_BF16 ? 2 : 4;
  const CUtensorMapDataType cdt =
      xdt == SVDQ_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  CUtensorMap tm_x, tm_ld;
  if (!make_tmap_2d(&tm_x, x, cdt, esz, p.M, p.B, ldx, p.tile_k, kRows, true)) {
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
  cudaError_t err = cudaMemsetAsync(sync, 0, 2 * sizeof(unsigned), stream);
  if (err != cudaSuccess) return err;
  ActArgs a{};
  a.B = static_cast<int>(p.B);
  a.M = static_cast<int>(p.M);
  a.ldx = ldx;
  a.nsteps = p.nsteps;
  a.ksplit = p.ksplit;
  a.nrb = p.nrb;
  a.nunits = p.nunits;
  a.rank_pad = has_ld ? p.rank_pad : 0;
  a.has_ld = has_ld ? 1 : 0;
  a.hold = p.hold;
  a.xbuf = p.xbuf;
  a.fmt_kind = fmt.kind;
  a.qmax = fmt.kind == SVDQ_KIND_INT ? (1 << (fmt.bits - 1)) - 1 : 0;
  a.x = x;
  a.scale = scale;
  a.gs_given = fmt.kind == SVDQ_KIND_NVFP4 ? act_global_scale : nullptr;
  a.gs_w = fmt.kind == SVDQ_KIND_NVFP4 ? w_global_scale : nullptr;
  a.ws_down = ws_down;
  a.ws_max = ws_max;
  a.sync = sync;
  a.codes = codes;
  a.sf = static_cast<uint8_t*>(sf);
  a.down = has_ld ? static_cast<__nv_bfloat16*>(down) : nullptr;
  a.act_scale = act_scale;
  a.status = device_status_word();
  // without the down factor the launch needs no ld ring (plan keeps its grid)
  ActPlan q = p;
  if (!has_ld) q.rank_pad = 0;
  const size_t smem = smem_for(q, p.xbuf);
  void* args[] = {&tm_x, &tm_ld, &a};
  if (xdt == SVDQ_BF16) {
    err = cudaFuncSetAttribute(act_fused_kernel<__nv_bfloat16>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (err != cudaSuccess) return err;
    err = cudaLaunchCooperativeKernel(reinterpret_cast<void*>(act_fused_kernel<__nv_bfloat16>),
                                      dim3(p.grid), dim3(kThreads), args, smem, stream);
  } else {
    err = cudaFuncSetAttribute(act_fused_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(smem));
    if (err != cudaSuccess) return err;
    err = cudaLaunchCooperativeKernel(reinterpret_cast<void*>(act_fused_kernel<float>), dim3(p.grid),
                                      dim3(kThreads), args, smem, stream);
  }
  return err;
}

}  // namespace svdq
