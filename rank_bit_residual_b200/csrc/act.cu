// act.cu - the activation pass of the SVDQuant linear for batches of more
// than 128 rows: a stats kernel and a codes kernel.
//
// "SVDQuant Smoothing, Low-rank and Residual Quantization", Formula items 1
// and 3: X_hat = x / scale is quantised per tensor (INT grid, or NVFP4 blocks
// for the variant of "flashinfer.gemm.svdquant_linear" step 1, or MXFP4 blocks
// of 32 with power-of-two scales for the "mxfp4" per-block format of the
// SVDQuant parameter configuration guide), and the
// low-rank branch needs X_hat L1 = x ld^T (step 2 of that page) from the same
// read of x.
//
// Work unit = 128 rows x a range of columns; the per-tensor scale needs every
// unit's maximum before any code is written, and the boundary between the
// two kernels is that grid-wide barrier (an in-kernel barrier would need its
// counter zeroed before every launch, a graph node that costs more than the
// barrier itself).
//   stats kernel  streams the unit's rows with coalesced 16-byte loads (whole
//                 row segments: DRAM pages are read front to back), takes the
//                 column maxima of |x| from registers, and runs the unit's
//                 down-projection x ld^T with warp-level MMAs from padded
//                 shared-memory tiles; it writes one partial maximum per CTA
//                 and one partial down tile per unit. Since fl(a / c) is
//                 monotone in a, the tensor maximum of |X_hat|, rounded to
//                 fp32, is max_k fl(colmax_k / scale_k) (IEEE quotients).
//   codes kernel  takes the per-tensor scale from the partial maxima, writes
//                 the codes from a second read of x (from L2 when x fits
//                 there) and sums each row block's partial down tiles in split
//                 order into bf16 hi | lo.
//
// Rounding: the stored scalars carry one fp32 rounding each (s = fl(m / qmax)
// with m the fp32 maximum above; the NVFP4 / MXFP4 block maxima and scales),
// and every code is the exactly rounded value of its real quotient. The codes
// kernel estimates each quotient with multiplies by the reciprocals
// r_k = fl(1 / scale_k) and u = fl(1 / s) (INT: rint(fl(x c_k)), c_k =
// fl(r_k u)) and decides the rare elements next to a rounding boundary again
// in exact arithmetic (encode.cuh).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "encode.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace svdq {

namespace {

constexpr int kWorkWarps = 16;
constexpr int kWork = 32 * kWorkWarps;      // threads of both kernels
constexpr int kRows = 128;                  // rows per unit
constexpr int kTileBytes = 128;             // bytes of a row per column tile (64 bf16 / 32 fp32)
constexpr int kSub = 256;                   // bytes of a row per stats sub-chunk (two tiles)
constexpr int kMaxStages = 6;
constexpr int kScaleBytes = 512;            // a stage's scale values (at most 128 columns)

// Bytes of one stats-kernel stage: x and ld as two 128-byte K blocks each, then
// the scale values; a multiple of 1024 so every block keeps the swizzle atom.
__host__ __device__ constexpr int stats_stage_bytes(int rank_pad) {
  return (2 * kRows * kTileBytes + 2 * rank_pad * kTileBytes + kScaleBytes + 1023) / 1024 * 1024;
}

// TMEM columns for a rank_pad-column fp32 accumulator (a power of two >= 32).
__host__ __device__ constexpr uint32_t tmem_cols_for(int rank_pad) {
  return rank_pad <= 32 ? 32u : rank_pad <= 64 ? 64u : rank_pad <= 128 ? 128u : 256u;
}
constexpr size_t kStatsSmemBudget = 220 * 1024;

struct ActArgs {
  int B, M;
  int64_t ldx;
  int nsteps, ksplit, nrb, nunits, rank_pad, has_ld, fmt_kind, qmax;
  int nparts;       // partial maxima written by the stats kernel
  int stages;       // stats kernel: shared-memory stages
  int nacc;         // stats kernel: MMA issuers, each with its own TMEM accumulator
  int chained;      // stats kernel: launched as a programmatic dependent of the previous kernel
  const void* x;
  const float* scale;
  const float* gs_given;
  const float* gs_w;
  const void* ld;   // [rank_pad][M], x's dtype
  float* ws_down;   // [ksplit][B][rank_pad]
  float* ws_max;    // [nparts]
  void* codes;
  uint8_t* sf;
  __nv_bfloat16* down;
  float* act_scale;
  unsigned* status;   // bounded waits record a timeout here
};


// Eight consecutive elements of x (16 bytes of bf16, or 32 of fp32) from
// global memory; cl: column within the unit, a multiple of 8.
template <typename TIn>
__device__ __forceinline__ void load8(const void* x, int64_t ldx, int64_t row, int64_t col0, int cl,
                                      uint4 (&u)[2]) {
  constexpr int kPerChunk = 16 / static_cast<int>(sizeof(TIn));
  constexpr int kChunks = 8 / kPerChunk;   // 1 (bf16) or 2 (fp32)
  const uint4* g = reinterpret_cast<const uint4*>(static_cast<const TIn*>(x) + row * ldx + col0 + cl);
#pragma unroll
  for (int h = 0; h < kChunks; ++h) u[h] = __ldg(g + h);
}

template <typename TIn>
__device__ __forceinline__ void unpack8(const uint4 (&u)[2], float (&v)[8]) {
  if constexpr (sizeof(TIn) == 2) {
    unpack16<TIn>(u[0], v);
  } else {
    unpack16<TIn>(u[0], v);
    unpack16<TIn>(u[1], v + 4);
  }
}

// Wait until at most stages - 2 groups are pending (stages in [2, kMaxStages]).
__device__ __forceinline__ void cp_async_wait_ring(int stages) {
  switch (stages) {
    case 2: cp_async_wait<0>(); break;
    case 3: cp_async_wait<1>(); break;
    case 4: cp_async_wait<2>(); break;
    case 5: cp_async_wait<3>(); break;
    default: cp_async_wait<4>(); break;
  }
}

// Running maximum of |x| over one 32-bit word of a row: two bf16 lanes (the
// packed 16-bit magnitudes, one SIMD max) or one fp32 (its magnitude bits);
// for non-negative values both orders agree with the float order.
template <typename TIn>
__device__ __forceinline__ uint32_t abs_max_word(uint32_t m, uint32_t w) {
  if constexpr (sizeof(TIn) == 2)
    return __vmaxu2(m, w & 0x7FFF7FFFu);
  else
    return max(m, w & 0x7FFFFFFFu);
}
template <typename TIn>
__device__ __forceinline__ uint32_t max_word(uint32_t m, uint32_t w) {
  if constexpr (sizeof(TIn) == 2)
    return __vmaxu2(m, w);
  else
    return max(m, w);
}

// ------------------------------------------------------------ stats kernel
// A unit is streamed in sub-chunks of kSub bytes per row through a ring of
// `stages` shared-memory stages filled by cp.async (stages - 1 sub-chunks in
// flight while one is consumed). A stage holds the x rows and the ld rows as
// two 128-byte-wide K blocks each, in the 128-byte-swizzled K-major layout the
// tensor core reads (16-byte chunk c of row r at chunk c ^ (r & 7) of the
// row's 128 bytes), then the sub-chunk's scale values.
//   copies        thread t moves the 16-byte piece t % 16 of rows t / 16 + 32 i
//                 (i < 4): a warp moves two whole 256-byte row segments;
//   column maxima warp w scans 32-bit words 4 w .. 4 w + 3 of rows l / 4 + 8 i
//                 (lane l, i < 16; conflict-free under the swizzle), the eight
//                 row slices meet by shuffles, and each column's fl(colmax / scale_k)
//                 is taken once;
//   down tile     one thread issues the sub-chunk's tcgen05 MMAs (M = 128 rows,
//                 N = rank_pad, kind::f16 for bf16 x, kind::tf32 for fp32 x)
//                 into a TMEM accumulator that lives across the unit; their
//                 commit frees the stage for the copies of a later sub-chunk;
//                 at the unit's end warps 0-3 drain it (TMEM lane = row).
template <typename TIn>
__global__ void __launch_bounds__(kWork, 1) act_stats_kernel(const ActArgs a) {
  constexpr int kEsz = static_cast<int>(sizeof(TIn));
  constexpr int kSubCols = kSub / kEsz;             // 128 bf16 or 64 fp32 columns
  constexpr int kPer16 = 16 / kEsz;                 // elements per 16-byte piece
  constexpr int kTileK = kTileBytes / kEsz;         // columns per K tile
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ float red[kWorkWarps];
  __shared__ __align__(8) uint64_t mma_bar[kMaxStages];
  __shared__ uint32_t tmem_sh;
  __shared__ int abort_sh;

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int rp = a.rank_pad;                        // 0 without the down factor
  const int stages = a.stages;
  const int stage_bytes = stats_stage_bytes(rp);
  const int ld_off = 2 * kRows * kTileBytes;        // the ld blocks follow the x blocks
  const int sc_off = ld_off + 2 * rp * kTileBytes;  // then the scale values
  const int piece = tid & 15, rg = tid >> 4;
  const int wi = warp * 4 + (lane & 3), rs = lane >> 2;   // column-max word and row slice
  const TIn* x = static_cast<const TIn*>(a.x);
  const TIn* ld = static_cast<const TIn*>(a.ld);
  const uint32_t idesc = kEsz == 2 ? idesc_bf16(kRows, rp > 0 ? rp : 16) : idesc_tf32(kRows, rp > 0 ? rp : 16);
  float run = 0.0f;

  const int nacc = a.nacc;
  const uint32_t acc_cols = tmem_cols_for(rp);
  if (tid == 0) {
    for (int s = 0; s < kMaxStages; ++s) mbar_init(&mma_bar[s], nacc);
    fence_mbar_init();
    abort_sh = 0;
  }
  // chained after another linear: x is that linear's output, complete and
  // visible once the kernel before this one has finished. Waited for before the
  // tensor-memory allocation, so a CTA of this kernel that shares an SM with
  // one of that kernel's never holds columns that kernel is waiting for.
  if (a.chained) pdl_wait();
  if (rp > 0 && warp == 0) {
    tmem_alloc(&tmem_sh, acc_cols * nacc);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_sh;

  // 16-byte chunk c (0..15) of row r of a two-block region with `rows` rows
  auto swz = [](int r, int c, int rows) -> int {
    return (c >> 3) * rows * kTileBytes + r * kTileBytes + (((c & 7) ^ (r & 7)) << 4);
  };
  uint32_t g = 0;   // sub-chunks begun so far: stage g % stages, barrier phase (g / stages) & 1
  for (int unit = blockIdx.x; unit < a.nunits; unit += gridDim.x) {
    const int rb = unit % a.nrb, sp = unit / a.nrb;
    const int m0 = rb * kRows;
    const int k_lo = static_cast<int>((static_cast<int64_t>(a.nsteps) * sp) / a.ksplit);
    const int k_hi = static_cast<int>((static_cast<int64_t>(a.nsteps) * (sp + 1)) / a.ksplit);
    const int c_lo = k_lo * kTileK;
    const int c_hi = min(a.M, k_hi * kTileK);
    const int nsub = (c_hi - c_lo + kSubCols - 1) / kSubCols;

    // sub-chunk c -> its stage (one commit group per call, empty past the end)
    auto issue = [&](int c) {
      if (c < nsub) {
        uint8_t* st = smem + ((g + c) % stages) * stage_bytes;
        const int col = c_lo + c * kSubCols + piece * kPer16;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int r = rg + 32 * i, row = m0 + r;
          const bool in = col < c_hi && row < a.B;
          cp_async16(st + swz(r, piece, kRows),
                     in ? static_cast<const void*>(x + static_cast<int64_t>(row) * a.ldx + col) : a.x, in ? 16 : 0);
        }
        for (int idx = tid; idx < rp * 16; idx += kWork) {
          const int j = idx >> 4, cc = idx & 15, colj = c_lo + c * kSubCols + cc * kPer16;
          const bool in = colj < c_hi;
          cp_async16(st + ld_off + swz(j, cc, rp),
                     in ? static_cast<const void*>(ld + static_cast<int64_t>(j) * a.M + colj) : a.ld, in ? 16 : 0);
        }
        if (tid < kSubCols) {   // the sub-chunk's scale values (any 4-byte alignment)
          const int cc = c_lo + c * kSubCols + tid;
          const bool in = cc < c_hi;
          cp_async4(st + sc_off + 4 * tid, in ? a.scale + cc : a.scale, in ? 4 : 0);
        }
      }
      cp_async_commit();
    };
    for (int c = 0; c < stages - 1; ++c) issue(c);
    for (int c = 0; c < nsub; ++c) {
      const uint32_t gc = g + c;
      const uint8_t* st = smem + (gc % stages) * stage_bytes;
      cp_async_wait_ring(stages);   // this thread's copies of sub-chunk c have landed
      fence_proxy_async_smem();     // ... and are visible to the tensor core
      __syncthreads();              // everyone's have; every thread is done with sub-chunk c - 1
      if (abort_sh) break;          // a bounded wait gave up (uniform after the barrier)
      if (rp > 0 && lane == 0 && warp < nacc) {
        // lane 0 of warps 0 .. nacc - 1 (one per SM sub-partition) each issue a
        // share of the sub-chunk's MMAs into an accumulator of their own
        tc_fence_after();
        const uint32_t xa = smem_u32(st), la = xa + ld_off;
        const uint32_t acc = tmem + acc_cols * warp;
        const int kk0 = warp * (kSub / 32) / nacc, kk1 = (warp + 1) * (kSub / 32) / nacc;
        for (int kk = kk0; kk < kk1; ++kk) {   // 32 bytes of K per MMA
          const uint32_t off = (kk >> 2) * kRows * kTileBytes + (kk & 3) * 32;
          const uint32_t offl = (kk >> 2) * rp * kTileBytes + (kk & 3) * 32;
          if constexpr (kEsz == 2)
            mma_f16(acc, smem_desc_sw128(xa + off), smem_desc_sw128(la + offl), idesc, (c > 0 || kk > kk0) ? 1u : 0u);
          else
            mma_tf32(acc, smem_desc_sw128(xa + off), smem_desc_sw128(la + offl), idesc, (c > 0 || kk > kk0) ? 1u : 0u);
        }
        mma_commit(&mma_bar[gc % stages]);
      }
      // refill the stage of sub-chunk c - 1 once its MMAs are done (each warp
      // waits for itself, then copies its share)
      if (rp > 0 && c > 0) mbar_wait_warp(&mma_bar[(gc - 1) % stages], ((gc - 1) / stages) & 1, a.status, &abort_sh);
      issue(c + stages - 1);
      {
        // max_k fl(colmax_k / scale_k): fl(a / c) is monotone in a, so the
        // column maximum of |x| is divided once per column
        uint32_t m = 0u;
#pragma unroll
        for (int i = 0; i < 16; ++i)
          m = abs_max_word<TIn>(m, ld_shared_u32(smem_u32(st + swz(rs + 8 * i, wi >> 2, kRows) + 4 * (wi & 3))));
        m = max_word<TIn>(m, __shfl_xor_sync(0xffffffffu, m, 4));
        m = max_word<TIn>(m, __shfl_xor_sync(0xffffffffu, m, 8));
        m = max_word<TIn>(m, __shfl_xor_sync(0xffffffffu, m, 16));
        // every lane of the word's group holds its maximum; row slice 0 (and 1
        // for the second bf16 lane) scales it
        const float* sc = reinterpret_cast<const float*>(st + sc_off);
        if constexpr (kEsz == 2) {
          if (rs < 2) {
            const int e = 2 * wi + rs;
            if (c_lo + c * kSubCols + e < c_hi) {
              const float v = __uint_as_float(rs == 0 ? m << 16 : m & 0xFFFF0000u);
              run = fmaxf(run, __fdiv_rn(v, sc[e]));
            }
          }
        } else {
          if (rs == 0 && c_lo + c * kSubCols + wi < c_hi)
            run = fmaxf(run, __fdiv_rn(__uint_as_float(m), sc[wi]));
        }
      }
    }
    // the unit's partial down tile: wait for its last MMAs, then TMEM -> ws_down
    if (rp > 0 && !abort_sh) {
      if (warp < 4) {
        const uint32_t gl = g + nsub - 1;
        const bool ok = mbar_wait_warp(&mma_bar[gl % stages], (gl / stages) & 1, a.status, &abort_sh);
        tc_fence_after();
        const int row = m0 + warp * 32 + lane;
        float* dst = a.ws_down + (static_cast<int64_t>(sp) * a.B + row) * rp;
        for (int c0 = 0; c0 < rp; c0 += 16) {
          // the accumulators summed in issuer order
          float sum[16];
          for (int q = 0; q < nacc; ++q) {
            uint32_t v[16];
            tmem_ld_32x32b_x16(tmem + (static_cast<uint32_t>(warp * 32) << 16) + acc_cols * q + c0, v);
            tmem_ld_wait_regs(v);
#pragma unroll
            for (int j = 0; j < 16; ++j) sum[j] = q == 0 ? __uint_as_float(v[j]) : sum[j] + __uint_as_float(v[j]);
          }
          if (ok && row < a.B) {
#pragma unroll
            for (int j = 0; j < 16; j += 4)
              *reinterpret_cast<float4*>(dst + c0 + j) = make_float4(sum[j], sum[j + 1], sum[j + 2], sum[j + 3]);
          }
        }
        tc_fence_before();
      }
    }
    g += nsub;
    __syncthreads();   // the drain is done before the next unit's first MMA; stages are free
    if (abort_sh) break;
  }
  cp_async_wait<0>();   // no copy is still on its way when the CTA ends
  // per-CTA maximum -> ws_max[blockIdx.x]
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) run = fmaxf(run, __shfl_xor_sync(0xffffffffu, run, o));
  if (lane == 0) red[warp] = run;
  __syncthreads();
  if (tid == 0) {
    float mx = red[0];
    for (int w = 1; w < kWorkWarps; ++w) mx = fmaxf(mx, red[w]);
    a.ws_max[blockIdx.x] = mx;
  }
  if (rp > 0 && warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, acc_cols * nacc);
  }
}

// ------------------------------------------------------------ codes kernel
template <typename TIn>
__global__ void __launch_bounds__(kWork, 1) act_codes_kernel(const ActArgs a) {
  constexpr int kTileK = kTileBytes / static_cast<int>(sizeof(TIn));
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ float red[kWorkWarps];
  float* rcp = reinterpret_cast<float*>(smem);   // the unit's reciprocals
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  auto unit_range = [&](int unit, int& m0, int& k_lo, int& n) {
    const int rb = unit % a.nrb, sp = unit / a.nrb;
    m0 = rb * kRows;
    k_lo = static_cast<int>((static_cast<int64_t>(a.nsteps) * sp) / a.ksplit);
    n = static_cast<int>((static_cast<int64_t>(a.nsteps) * (sp + 1)) / a.ksplit) - k_lo;
  };
  {
    float m = 0.0f;
    for (int i = tid; i < a.nparts; i += kWork) m = fmaxf(m, __ldcg(a.ws_max + i));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    __syncthreads();
    if (lane == 0) red[warp] = m;
    __syncthreads();
    m = red[0];
    for (int w = 1; w < kWorkWarps; ++w) m = fmaxf(m, red[w]);
    const bool nv = a.fmt_kind == SVDQ_KIND_NVFP4;
    const bool mx = a.fmt_kind == SVDQ_KIND_MXFP4;
    float s = 0.0f, u = 0.0f, gs_x = 1.0f;   // MXFP4: no global scale (1)
    if (nv) {
      gs_x = a.gs_given != nullptr ? __ldg(a.gs_given) : (m > 0.0f ? __fdiv_rn(2688.0f, m) : 1.0f);
    } else if (!mx) {
      s = __fdiv_rn(m, static_cast<float>(a.qmax));
      u = s > 0.0f ? __frcp_rn(s) : 0.0f;
    }
    if (blockIdx.x == 0 && tid == 0) *a.act_scale = nv || mx ? gs_x : s;
    const int kb = a.M / (mx ? 32 : 16);   // fp4 scale blocks per row
    const int64_t kbp = (kb + 3) / 4 * 4;

    for (int unit = blockIdx.x; unit < a.nunits; unit += gridDim.x) {
      int m0, k_lo, n;
      unit_range(unit, m0, k_lo, n);
      const int sp = unit / a.nrb;
      const int64_t col0 = static_cast<int64_t>(k_lo) * kTileK;
      __syncthreads();
      for (int j = tid; j < n * kTileK; j += kWork) {
        const int col = k_lo * kTileK + j;
        rcp[j] = col < a.M ? __frcp_rn(__ldg(a.scale + col)) : 0.0f;
      }
      __syncthreads();
      const int rows = min(kRows, a.B - m0);
      const int ncols = min(n * kTileK, a.M - k_lo * kTileK);   // a multiple of 32
      if (!nv && !mx) {
        // a warp writes 256 consecutive codes of a row (8 per lane, one 256-byte
        // store) for kR rows, whose loads are all issued first
        constexpr int kR = sizeof(TIn) == 2 ? 8 : 4;
        for (int c256 = 0; c256 < ncols; c256 += 256) {
          const int cl = c256 + 8 * lane;
          if (cl >= ncols) continue;
          float ck[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) ck[j] = __fmul_rn(rcp[cl + j], u);
          for (int r0 = warp * kR; r0 < rows; r0 += kWorkWarps * kR) {
            uint4 uv[kR][2];
#pragma unroll
            for (int i = 0; i < kR; ++i)
              if (r0 + i < rows) load8<TIn>(a.x, a.ldx, m0 + r0 + i, col0, cl, uv[i]);
#pragma unroll
            for (int i = 0; i < kR; ++i) {
              if (r0 + i < rows) {
                float v[8];
                unpack8<TIn>(uv[i], v);
                *reinterpret_cast<uint2*>(static_cast<int8_t*>(a.codes) + static_cast<int64_t>(m0 + r0 + i) * a.M +
                                          col0 + cl) =
                    int_codes8(v, ck, a.scale + col0 + cl, s, a.qmax);
              }
            }
          }
        }
      } else {
        // half a warp = 256 consecutive elements of one row (16 elements per
        // lane: one NVFP4 block, half an MXFP4 block whose other half is the
        // neighbouring lane's), kR rows per half warp with all loads issued first
        constexpr int kR = sizeof(TIn) == 2 ? 4 : 2;
        constexpr int kHalves = 2 * kWorkWarps;
        const int hw = 2 * warp + (lane >> 4);
        const int nch = (ncols + 255) / 256;
        for (int cc = 0; cc < nch; ++cc) {
          const int cl = cc * 256 + 16 * (lane & 15);
          if (cl >= ncols) continue;
          for (int r0 = hw; r0 < rows; r0 += kR * kHalves) {
            uint4 uv[kR][2][2];
#pragma unroll
            for (int i = 0; i < kR; ++i)
              if (r0 + kHalves * i < rows) {
                load8<TIn>(a.x, a.ldx, m0 + r0 + kHalves * i, col0, cl, uv[i][0]);
                load8<TIn>(a.x, a.ldx, m0 + r0 + kHalves * i, col0, cl + 8, uv[i][1]);
              }
#pragma unroll
            for (int i = 0; i < kR; ++i) {
              const int r = r0 + kHalves * i;
              if (r >= rows) continue;
              float xr[16], xs[16];   // the raw elements and their estimates fl(x r_k)
              unpack8<TIn>(uv[i][0], *reinterpret_cast<float(*)[8]>(xr));
              unpack8<TIn>(uv[i][1], *reinterpret_cast<float(*)[8]>(xr + 8));
#pragma unroll
              for (int j = 0; j < 16; ++j) xs[j] = __fmul_rn(xr[j], rcp[cl + j]);
              const float* sc16 = a.scale + col0 + cl;
              float amax = block_amax_exact<16>(xr, xs, sc16);
              const int64_t row = m0 + r;
              const int64_t col = col0 + cl;
              uint8_t sfb;
              float enc;
              if (mx) {
                // lanes 2i and 2i + 1 hold one 32-element block; both take the
                // same exits above (ncols is a multiple of 32), so the pair is
                // converged here
                amax = fmaxf(amax, __shfl_xor_sync(3u << (lane & 30), amax, 1));
                const int X = mx_block_exponent(amax);
                sfb = static_cast<uint8_t>(X + 127);
                enc = mx_inv_scale(X);
              } else {
                sfb = f32_to_ue4m3(__fmul_rn(__fdiv_rn(amax, 6.0f), gs_x));
                const float d = ue4m3_to_f32(sfb);
                enc = d > 0.0f ? __fdiv_rn(gs_x, d) : 0.0f;
              }
#pragma unroll
              for (int j = 0; j < 16; ++j) xs[j] = __fmul_rn(xs[j], enc);
              *reinterpret_cast<uint2*>(static_cast<uint8_t*>(a.codes) + row * (a.M / 2) + col / 2) =
                  make_uint2(e2m1x8_exact(xs, xr, enc, sc16), e2m1x8_exact(xs + 8, xr + 8, enc, sc16 + 8));
              if (!mx)
                a.sf[sf_swizzle_offset(row, col / 16, kbp)] = sfb;
              else if ((lane & 1) == 0)
                a.sf[sf_swizzle_offset(row, col / 32, kbp)] = sfb;
            }
          }
        }
      }
      // down = the K-split partials summed in split order, as bf16 hi | lo
      if (a.has_ld && a.down != nullptr) {
        const int r_lo = (kRows * sp) / a.ksplit, r_hi = (kRows * (sp + 1)) / a.ksplit;
        const float mult = nv ? (a.gs_w != nullptr ? __fmul_rn(gs_x, __ldg(a.gs_w)) : gs_x) : 1.0f;
        const int cnt = (r_hi - r_lo) * a.rank_pad;
        for (int i = tid; i < cnt; i += kWork) {
          const int rr = r_lo + i / a.rank_pad, j = i % a.rank_pad;
          const int row = m0 + rr;
          if (row >= a.B) continue;
          float acc = 0.0f;
          for (int z = 0; z < a.ksplit; ++z)
            acc += __ldcg(a.ws_down + (static_cast<int64_t>(z) * a.B + row) * a.rank_pad + j);
          acc = __fmul_rn(acc, mult);
          const __nv_bfloat16 hi = __float2bfloat16_rn(acc);
          const __nv_bfloat16 lo = __float2bfloat16_rn(acc - __bfloat162float(hi));
          a.down[static_cast<int64_t>(row) * 2 * a.rank_pad + j] = hi;
          a.down[static_cast<int64_t>(row) * 2 * a.rank_pad + a.rank_pad + j] = lo;
        }
      }
    }
    // fp4: zero the scale padding (rows up to a multiple of 128, columns up to 4)
    if (nv || mx) {
      const int64_t rows_p = (static_cast<int64_t>(a.B) + 127) / 128 * 128;
      const int64_t pad_cols = kbp - kb;
      const int64_t n_pad = (rows_p - a.B) * kbp + static_cast<int64_t>(a.B) * pad_cols;
      for (int64_t i = static_cast<int64_t>(blockIdx.x) * kWork + tid; i < n_pad;
           i += static_cast<int64_t>(gridDim.x) * kWork) {
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
}

template <typename TIn>
cudaError_t launch_stats(const ActArgs& a, int grid, size_t smem, cudaStream_t stream) {
  cudaError_t err = cudaFuncSetAttribute(act_stats_kernel<TIn>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
  if (err != cudaSuccess) return err;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kWork);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = a.chained ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, act_stats_kernel<TIn>, a);
}

template <typename TIn>
cudaError_t launch_codes(const ActArgs& a, size_t smem, cudaStream_t stream) {
  cudaError_t err = cudaFuncSetAttribute(act_codes_kernel<TIn>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
  if (err != cudaSuccess) return err;
  act_codes_kernel<TIn><<<a.nunits, kWork, smem, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace

void finish_act_plan(ActPlan& p) {
  if (p.small) {
    finish_act_plan_small(p);
    return;
  }
  p.nunits = p.nrb * p.ksplit;
  // stages: as many as fit, no more than the longest unit's sub-chunks + 1
  const int steps_max = (p.nsteps + p.ksplit - 1) / p.ksplit;
  const int sub_max = (steps_max * kTileBytes + kSub - 1) / kSub;
  const size_t sb = static_cast<size_t>(stats_stage_bytes(p.rank_pad));
  p.stages = static_cast<int>(std::min<size_t>(kMaxStages, (kStatsSmemBudget - 1024) / sb));
  p.stages = std::max(2, std::min(p.stages, sub_max + 1));
  p.smem = sb * p.stages + 1024;   // + alignment of the first stage to 1024 bytes
  // one CTA per SM (512 threads, most of the shared memory)
  p.grid = std::min(p.nunits, num_sms());
  p.nparts = p.grid;
}

ActPlan plan_act(int64_t B, int64_t M, int32_t rank_pad, svdq_dtype xdt, bool allow_small) {
  ActPlan p{};
  p.B = B;
  p.M = M;
  p.rank_pad = rank_pad;
  p.bf16 = xdt == SVDQ_BF16;
  if (allow_small && B <= kActSmallMaxB) {
    // short batch: one column chunk per SM
    p.small = 1;
    p.ksplit = num_sms();
    finish_act_plan_small(p);
    if (p.smem <= kActSmallSmemMax) return p;
    p = ActPlan{};
    p.B = B;
    p.M = M;
    p.rank_pad = rank_pad;
    p.bf16 = xdt == SVDQ_BF16;
  }
  p.tile_k = p.bf16 ? 64 : 32;
  p.nrb = static_cast<int>(ceil_div(B, kRows));
  p.nsteps = static_cast<int>(ceil_div(M, p.tile_k));
  // at most one unit per SM: split K until the units cover the SMs
  const int sms = num_sms();
  p.ksplit = std::max(1, std::min(p.nsteps, sms / std::max(p.nrb, 1)));
  finish_act_plan(p);
  return p;
}

size_t act_scratch_bytes(const ActPlan& p) {
  if (p.small)   // partial maxima, then the partial down tiles (act_small.cu)
    return static_cast<size_t>(round_up(static_cast<int64_t>(p.grid) * 4, 256)) +
           (p.rank_pad > 0 ? static_cast<size_t>(round_up(static_cast<int64_t>(p.grid) * p.B * p.rank_pad * 4, 256)) : 0) +
           256;
  size_t b = static_cast<size_t>(round_up(static_cast<int64_t>(std::max(p.grid, 1)) * 4, 256));
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
  if (p.small)
    return launch_act_small(p, x, xdt, ldx, scale, fmt, act_global_scale, w_global_scale, ld, codes, sf,
                            act_scale, down, scratch, stream, bad_args);
  const bool has_ld = ld != nullptr && p.rank_pad > 0 && down != nullptr;
  const int esz = xdt == SVDQ_BF16 ? 2 : 4;
  // 16-byte copies of x and ld rows
  if ((reinterpret_cast<uintptr_t>(x) & 15) != 0 || (ldx * esz) % 16 != 0 || (p.M * esz) % 16 != 0 ||
      (has_ld && (reinterpret_cast<uintptr_t>(ld) & 15) != 0)) {
    *bad_args = true;
    return cudaSuccess;
  }
  Carver cv(scratch, ~size_t(0));
  float* ws_max = static_cast<float*>(cv.take(static_cast<size_t>(std::max(p.grid, 1)) * 4));
  float* ws_down =
      has_ld ? static_cast<float*>(cv.take(static_cast<size_t>(p.ksplit) * p.B * p.rank_pad * 4))
             : nullptr;
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
  a.nparts = p.grid;
  a.fmt_kind = fmt.kind;
  a.qmax = fmt.kind == SVDQ_KIND_INT ? (1 << (fmt.bits - 1)) - 1 : 0;
  a.x = x;
  a.scale = scale;
  a.gs_given = fmt.kind == SVDQ_KIND_NVFP4 ? act_global_scale : nullptr;
  a.gs_w = fmt.kind == SVDQ_KIND_NVFP4 ? w_global_scale : nullptr;
  a.ld = has_ld ? ld : nullptr;
  a.ws_down = ws_down;
  a.ws_max = ws_max;
  a.codes = codes;
  a.sf = static_cast<uint8_t*>(sf);
  a.down = has_ld ? static_cast<__nv_bfloat16*>(down) : nullptr;
  a.act_scale = act_scale;
  a.status = device_status_word();
  // without the down factor the stages hold x alone (fewer bytes per stage)
  ActPlan q = p;
  if (!has_ld) {
    q.rank_pad = 0;
    finish_act_plan(q);
  }
  a.stages = q.stages;
  // as many MMA issuers (up to 4) as TMEM holds accumulators of rank_pad columns
  a.nacc = a.rank_pad > 0 ? static_cast<int>(std::min<uint32_t>(4u, 512u / tmem_cols_for(a.rank_pad))) : 1;
  a.chained = p.chained;
  // the codes kernel keeps only the unit's reciprocals in shared memory
  const int steps_max = (p.nsteps + p.ksplit - 1) / p.ksplit;
  const size_t smem2 = static_cast<size_t>(steps_max) * p.tile_k * sizeof(float) + 1024;
  cudaError_t err = xdt == SVDQ_BF16 ? launch_stats<__nv_bfloat16>(a, p.grid, q.smem, stream)
                                     : launch_stats<float>(a, p.grid, q.smem, stream);
  if (err != cudaSuccess) return err;
  return xdt == SVDQ_BF16 ? launch_codes<__nv_bfloat16>(a, smem2, stream) : launch_codes<float>(a, smem2, stream);
}

}  // namespace svdq
