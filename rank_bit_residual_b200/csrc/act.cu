// act.cu - the activation pass of the SVDQuant linear for batches of more
// than 128 rows: a maximum kernel and a quantise kernel.
//
// "SVDQuant Smoothing, Low-rank and Residual Quantization", Formula items 1
// and 3: X_hat = x / scale is quantised per tensor (INT grid, or NVFP4 blocks
// for the variant of "flashinfer.gemm.svdquant_linear" step 1, or MXFP4 blocks
// of 32 with power-of-two scales for the "mxfp4" per-block format of the
// SVDQuant parameter configuration guide), and the low-rank branch needs
// X_hat L1 = x ld^T (step 2 of that page) from the same read of x.
//
// The per-tensor scale needs the maximum of |X_hat| over the whole tensor
// before any code is written, so x is read twice, by two launches whose
// boundary is that grid-wide dependency:
//   max kernel       streams x once at the copy bandwidth (coalesced 16-byte
//                    loads, eight rows in flight per thread) and takes column
//                    maxima of |x|; since fl(a / c) is monotone in a, the
//                    tensor maximum of |X_hat| rounded to fp32 is
//                    max_k fl(colmax_k / scale_k) (IEEE quotients), one
//                    partial per CTA. It also clears the row-block counters
//                    of the quantise kernel. MXFP4, and NVFP4 with a given
//                    global scale, need no maximum: one block clears the
//                    counters and x is read once.
//   quantise kernel  work unit = 128 rows x a range of whole 256-byte row
//                    segments, streamed by TMA (one 16 KB box per 128 bytes of
//                    the 128 rows) through a ring of shared-memory stages; one
//                    thread issues the segment's tcgen05 MMAs of
//                    the down-projection (TMEM accumulator per unit) while
//                    all threads quantise the same segment from shared memory
//                    and store the codes (and block scales); at the unit's end
//                    the partial down tile goes to the workspace, and the last
//                    unit of a row block to finish sums the row block's
//                    partials in split order into bf16 hi | lo.
//
// Rounding: the stored scalars carry one fp32 rounding each (s = fl(m / qmax)
// with m the fp32 maximum above; the NVFP4 / MXFP4 block maxima and scales),
// and every code is the exactly rounded value of its real quotient. The
// quantise kernel estimates each quotient with multiplies by the reciprocals
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

constexpr int kWork = 512;                  // threads of the quantise kernel (one CTA per SM)
constexpr int kRows = 128;                  // rows per unit
constexpr int kTileBytes = 128;             // bytes of a row per column tile (64 bf16 / 32 fp32)
constexpr int kSub = 256;                   // bytes of a row per segment (two tiles)
constexpr int kMaxStages = 6;
constexpr int kMaxThreads = 256;            // threads of the maximum kernel
constexpr int kMaxSlab = 2048;              // bytes of a row per maximum-kernel CTA (16 per thread)
constexpr int kMaxCtasPerSm = 6;
constexpr int kFlatMinSegs = 8;             // segments per SM from which the flat partition pays

// Bytes of one quantise-kernel stage: x and ld as two 128-byte K blocks each; a
// multiple of 1024 so every block keeps the swizzle atom.
__host__ __device__ constexpr int quant_stage_bytes(int rank_pad) {
  return (2 * kRows * kTileBytes + 2 * rank_pad * kTileBytes + 1023) / 1024 * 1024;
}

// TMEM columns for a rank_pad-column fp32 accumulator (a power of two >= 32).
__host__ __device__ constexpr uint32_t tmem_cols_for(int rank_pad) {
  return rank_pad <= 32 ? 32u : rank_pad <= 64 ? 64u : rank_pad <= 128 ? 128u : 256u;
}
constexpr size_t kQuantSmemBudget = 220 * 1024;

struct ActArgs {
  int B, M;
  int64_t ldx;
  int nsteps;       // 256-byte segments of a row (the unit of the K split)
  int ksplit, nrb, nunits, rank_pad, has_ld, fmt_kind, qmax;
  int flat;         // 1: flat partition of the segments over the CTAs (else K split units)
  int nparts;       // partial maxima written by the maximum kernel (0: none needed)
  int max_rpc;      // maximum kernel: rows per CTA
  int max_nslabs;   // maximum kernel: column slabs of kMaxSlab bytes
  int stages;       // quantise kernel: shared-memory stages
  int nacc;         // quantise kernel: MMA issuers, each with its own TMEM accumulator
  int chained;      // maximum kernel: launched as a programmatic dependent of the previous kernel
  const void* x;
  const float* scale;
  const float* gs_given;
  const float* gs_w;
  const void* ld;   // [rank_pad][M], x's dtype
  float* ws_down;   // [ksplit][B][rank_pad]
  float* ws_max;    // [nparts]
  unsigned* ws_cnt; // [nrb] units of a row block done
  unsigned* zero_words;   // cleared by the maximum kernel for the GEMM that follows (nullable)
  int nzero;
  void* codes;
  uint8_t* sf;
  __nv_bfloat16* down;
  float* act_scale;
  unsigned* status;   // bounded waits record a timeout here
};

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
template <typename TIn>
__device__ __forceinline__ void abs_max16(uint32_t (&m)[4], const uint4 v) {
  m[0] = abs_max_word<TIn>(m[0], v.x);
  m[1] = abs_max_word<TIn>(m[1], v.y);
  m[2] = abs_max_word<TIn>(m[2], v.z);
  m[3] = abs_max_word<TIn>(m[3], v.w);
}

// A 16-byte read-only load that allocates no L1 line: the maximum kernel's
// stream of x is never re-read by the same SM, and without allocation the
// number of loads in flight is not bounded by the L1's capacity.
__device__ __forceinline__ uint4 ld_stream_v4(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// ------------------------------------------------------------ maximum kernel
// CTA = a slab of kMaxSlab bytes of every row in a range of rows; thread t
// reads the 16-byte piece t % 128 of rows r0 + t / 128, r0 + t / 128 + 2, ...
// (a warp reads 512 contiguous bytes of a row), eight loads in flight.
template <typename TIn>
__global__ void __launch_bounds__(kMaxThreads) act_max_kernel(const ActArgs a) {
  constexpr int kEsz = static_cast<int>(sizeof(TIn));
  constexpr int kPer16 = 16 / kEsz;
  __shared__ uint32_t xch[kMaxThreads / 2][4];
  __shared__ float red[kMaxThreads / 32];
  // chained after another linear: x is that linear's output
  if (a.chained) pdl_wait();
  // the quantise kernel may launch now and do its setup (it reads nothing of
  // this kernel's before its griddepcontrol.wait)
  pdl_trigger();
  const int tid = threadIdx.x;
  // block 0 clears the quantise kernel's row-block counters (and any words the
  // GEMM after this pass needs zeroed)
  if (blockIdx.x == 0) {
    for (int i = tid; i < a.nrb; i += kMaxThreads) a.ws_cnt[i] = 0u;
    for (int i = tid; i < a.nzero; i += kMaxThreads) a.zero_words[i] = 0u;
  }
  if (a.nparts == 0) return;
  const int slab = blockIdx.x % a.max_nslabs, rc = blockIdx.x / a.max_nslabs;
  const int col = slab * (kMaxSlab / kEsz) + (tid & 127) * kPer16;
  const int rsl = tid >> 7;
  const int r0 = rc * a.max_rpc, r1 = min(a.B, r0 + a.max_rpc);
  uint32_t m[4] = {0u, 0u, 0u, 0u};
  if (col < a.M && r0 + rsl < r1) {
    const int64_t step = 2 * a.ldx * kEsz / 16;   // two rows, in 16-byte units (ldx * esz % 16 == 0)
    const uint4* p = reinterpret_cast<const uint4*>(static_cast<const TIn*>(a.x) +
                                                    static_cast<int64_t>(r0 + rsl) * a.ldx + col);
    // eight loads issued before any is used, the last batch's past r1 skipped
    // (a zero word leaves the maximum unchanged)
    for (int r = r0 + rsl; r < r1; r += 16) {
      uint4 v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) v[u] = r + 2 * u < r1 ? ld_stream_v4(p + u * step) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
      for (int u = 0; u < 8; ++u) abs_max16<TIn>(m, v[u]);
      p += 8 * step;
    }
  }
  if (rsl == 1) {
#pragma unroll
    for (int j = 0; j < 4; ++j) xch[tid & 127][j] = m[j];
  }
  __syncthreads();
  float best = 0.0f;
  if (rsl == 0 && col < a.M) {
#pragma unroll
    for (int j = 0; j < 4; ++j) m[j] = max_word<TIn>(m[j], xch[tid][j]);
    float v[kPer16];
    unpack16<TIn>(make_uint4(m[0], m[1], m[2], m[3]), v);
#pragma unroll
    for (int e = 0; e < kPer16; ++e) best = fmaxf(best, __fdiv_rn(v[e], __ldg(a.scale + col + e)));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) best = fmaxf(best, __shfl_xor_sync(0xffffffffu, best, o));
  if ((tid & 31) == 0) red[tid >> 5] = best;
  __syncthreads();
  if (tid == 0) {
    float mx = red[0];
    for (int w = 1; w < kMaxThreads / 32; ++w) mx = fmaxf(mx, red[w]);
    a.ws_max[blockIdx.x] = mx;
  }
}

// ----------------------------------------------------------- quantise kernel
// A unit is streamed in segments of kSub bytes per row through a ring of
// `stages` shared-memory stages filled by TMA (stages - 1 segments in flight
// while one is consumed). A stage holds the x rows and the ld rows as two
// 128-byte-wide K blocks each, in the 128-byte-swizzled K-major layout the
// tensor core reads (16-byte chunk c of row r at chunk c ^ (r & 7) of the
// row's 128 bytes); rows past B and columns past M arrive as zeros.
//   copies      thread 0 loads the segment's four boxes (x and ld, two K
//               blocks each) once every thread is done with the stage's
//               previous segment and its MMAs have completed;
//   down tile   lane 0 of warps 0 .. nacc - 1 issue the segment's tcgen05 MMAs
//               (M = 128 rows, N = rank_pad, kind::f16 for bf16 x, kind::tf32
//               for fp32 x) into TMEM accumulators that live across the unit;
//               their commit frees the stage for the copies of a later segment;
//   codes       thread t takes E = 8 (INT) or 16 (fp4) consecutive elements
//               of a row (element group t % G, G = segment columns / E, rows
//               t / G + i * 512 / G), reads them from the stage and stores
//               their codes: a row's codes are written by consecutive threads.
// The per-column constants of the unit (c_k for INT, r_k for fp4) sit in
// shared memory after the stages.
template <typename TIn, bool kFp4>
__global__ void __launch_bounds__(kWork, 1) act_quant_kernel(const __grid_constant__ CUtensorMap tm_x,
                                                             const __grid_constant__ CUtensorMap tm_ld,
                                                             const ActArgs a) {
  constexpr int kEsz = static_cast<int>(sizeof(TIn));
  constexpr int kWorkWarps = kWork / 32;
  constexpr int kSubCols = kSub / kEsz;             // 128 bf16 or 64 fp32 columns
  constexpr int kPer16 = 16 / kEsz;                 // elements per 16-byte piece
  constexpr int kTileK = kTileBytes / kEsz;         // columns per K tile
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ float red[kWorkWarps];
  __shared__ __align__(8) uint64_t full_bar[kMaxStages];    // the stage's boxes have landed
  __shared__ __align__(8) uint64_t empty_bar[kMaxStages];   // every warp and every MMA is done with it
  __shared__ __align__(8) uint64_t unit_bar;                // the unit's MMAs are complete
  __shared__ uint32_t tmem_sh;
  __shared__ int abort_sh;
  __shared__ int last_sh;

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int rp = a.rank_pad;                        // 0 without the down factor
  const int stages = a.stages;
  const int stage_bytes = quant_stage_bytes(rp);
  const int ld_off = 2 * kRows * kTileBytes;        // the ld blocks follow the x blocks
  float* colv = reinterpret_cast<float*>(smem + static_cast<size_t>(stages) * stage_bytes);
  const uint32_t idesc = kEsz == 2 ? idesc_bf16(kRows, rp > 0 ? rp : 16) : idesc_tf32(kRows, rp > 0 ? rp : 16);
  const bool nv = a.fmt_kind == SVDQ_KIND_NVFP4;
  const bool mx = a.fmt_kind == SVDQ_KIND_MXFP4;

  const int nacc = a.nacc;
  const uint32_t acc_cols = tmem_cols_for(rp);
  if (tid == 0) {
    for (int s = 0; s < kMaxStages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], kWorkWarps + (rp > 0 ? nacc : 0));
    }
    mbar_init(&unit_bar, nacc);
    fence_mbar_init();
    abort_sh = 0;
    tma_prefetch_desc(&tm_x);
    if (rp > 0) tma_prefetch_desc(&tm_ld);
  }
  if (rp > 0 && warp == 0) {
    tmem_alloc(&tmem_sh, acc_cols * nacc);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();   // barriers initialised, TMEM allocated
  tc_fence_after();
  const uint32_t tmem = tmem_sh;

  // The kernel is launched as a programmatic dependent of the maximum kernel:
  // the setup above and the first piece's first copies of x and ld (which that
  // kernel does not write) overlap its tail; its partial maxima and counters,
  // and every output, are touched only after the wait in take_scale. The
  // per-tensor scale from the partial maxima (INT; NVFP4 without a given gs).
  float s = 0.0f, u = 0.0f, gs_x = 1.0f;   // MXFP4: no global scale (1)
  bool have_scale = false;
  auto take_scale = [&]() {
    pdl_wait();
    float m = 0.0f;
    for (int i = tid; i < a.nparts; i += kWork) m = fmaxf(m, __ldcg(a.ws_max + i));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) red[warp] = m;
    __syncthreads();
    m = red[0];
    for (int w = 1; w < kWorkWarps; ++w) m = fmaxf(m, red[w]);
    if (nv) {
      gs_x = a.gs_given != nullptr ? __ldg(a.gs_given) : (m > 0.0f ? __fdiv_rn(2688.0f, m) : 1.0f);
    } else if (!mx) {
      s = __fdiv_rn(m, static_cast<float>(a.qmax));
      u = s > 0.0f ? __frcp_rn(s) : 0.0f;
    }
    if (blockIdx.x == 0 && tid == 0) *a.act_scale = nv || mx ? gs_x : s;
    have_scale = true;
  };

  // element groups of the codes step: kE elements of a row per thread, the
  // threads of a row consecutive, kPasses rows per thread kRpp apart
  constexpr int kE = kFp4 ? 16 : 8;
  constexpr int kTpr = kSubCols / kE;                     // groups per row of a segment
  constexpr int kRpp = kWork / kTpr;                      // rows per pass
  constexpr int kPasses = kRows / kRpp > 0 ? kRows / kRpp : 1;
  const int grp = tid % kTpr, rr0 = tid / kTpr;
  const int64_t kb = a.M / (mx ? 32 : 16);                // fp4 scale blocks per row
  const int64_t kbp = (kb + 3) / 4 * 4;

  // 16-byte chunk c (0..15) of row r of a two-block region with `rows` rows
  auto swz = [](int r, int c, int rows) -> int {
    return (c >> 3) * rows * kTileBytes + r * kTileBytes + (((c & 7) ^ (r & 7)) << 4);
  };
  // the ring positions, advanced one segment at a time (no divisions): the
  // producer's (thread 0: next stage to fill and its use parity) and every
  // thread's (next stage to consume and its parity); a stage's first use is
  // the only one that does not wait for it to be released
  uint32_t p_seg = 0, p_stage = 0, p_par = 0;
  uint32_t c_stage = 0, c_par = 0;
  uint32_t unit_parity = 0;
  // Pieces of work: a row block and a range of its segments. Flat partition:
  // CTA i takes segments [W i / G, W (i + 1) / G) of all W = nrb * nsteps
  // segments in row-block-major order (every SM busy, at most one segment of
  // imbalance), which cuts a row block into the pieces of consecutive CTAs;
  // piece p of a row block writes partial slot p. Split partition: unit u =
  // (row block u % nrb, K range u / nrb of ksplit equal ranges), CTAs striding
  // over the units.
  const int64_t W = static_cast<int64_t>(a.nrb) * a.nsteps;
  const int G = static_cast<int>(gridDim.x);
  auto cta_of = [&](int64_t f) { return static_cast<int>(((f + 1) * G - 1) / W); };   // CTA holding segment f
  int64_t f = a.flat ? W * blockIdx.x / G : 0;
  const int64_t f_end = a.flat ? W * (blockIdx.x + 1) / G : 0;
  int unit = blockIdx.x;
  while (true) {
    int rb, sp, npieces, k_lo, k_hi;
    if (a.flat) {
      if (f >= f_end) break;
      rb = static_cast<int>(f / a.nsteps);
      k_lo = static_cast<int>(f - static_cast<int64_t>(rb) * a.nsteps);
      k_hi = static_cast<int>(min(static_cast<int64_t>(a.nsteps), k_lo + (f_end - f)));
      f += k_hi - k_lo;
      const int first = cta_of(static_cast<int64_t>(rb) * a.nsteps);
      sp = static_cast<int>(blockIdx.x) - first;
      npieces = cta_of(static_cast<int64_t>(rb) * a.nsteps + a.nsteps - 1) - first + 1;
    } else {
      if (unit >= a.nunits) break;
      rb = unit % a.nrb;
      sp = unit / a.nrb;
      npieces = a.ksplit;
      // whole segments per unit: no box reaches into another unit's columns
      k_lo = static_cast<int>((static_cast<int64_t>(a.nsteps) * sp) / a.ksplit);
      k_hi = static_cast<int>((static_cast<int64_t>(a.nsteps) * (sp + 1)) / a.ksplit);
      unit += G;
    }
    const int m0 = rb * kRows;
    const int c_lo = k_lo * kSubCols;
    const int c_hi = min(a.M, k_hi * kSubCols);
    const int nsub = k_hi - k_lo;
    const uint32_t seg_bytes = static_cast<uint32_t>(2 * kRows * kTileBytes + 2 * rp * kTileBytes);

    // segment c -> its stage (thread 0; nothing past the unit's end). A stage is
    // refilled once all 16 warps and the MMAs have released its previous
    // segment; only thread 0 waits for that, and only when it refills.
    auto issue = [&](int c) {
      if (tid == 0 && c < nsub) {
        const uint32_t s_ = p_stage;
        if (p_seg >= static_cast<uint32_t>(stages) && !mbar_wait(&empty_bar[s_], p_par ^ 1u, a.status, &abort_sh))
          return;   // a wait ran out: load nothing more
        ++p_seg;
        if (++p_stage == static_cast<uint32_t>(stages)) {
          p_stage = 0;
          p_par ^= 1u;
        }
        uint8_t* st = smem + s_ * stage_bytes;
        uint64_t* bar = &full_bar[s_];
        const int col = c_lo + c * kSubCols;
        mbar_arrive_expect_tx(bar, seg_bytes);
        tma_load_2d(st, &tm_x, bar, col, m0);
        tma_load_2d(st + kRows * kTileBytes, &tm_x, bar, col + kTileK, m0);
        if (rp > 0) {
          tma_load_2d(st + ld_off, &tm_ld, bar, col, 0);
          tma_load_2d(st + ld_off + rp * kTileBytes, &tm_ld, bar, col + kTileK, 0);
        }
      }
    };
    for (int c = 0; c < stages - 1; ++c) issue(c);
    if (!have_scale) take_scale();   // the first piece only (uniform over the CTA)
    // per-column constants of the unit: c_k = fl(fl(1 / scale_k) u) (INT) or
    // r_k = fl(1 / scale_k) (fp4)
    for (int j = tid; j < c_hi - c_lo; j += kWork) {
      const float r = __frcp_rn(__ldg(a.scale + c_lo + j));
      colv[j] = (nv || mx) ? r : __fmul_rn(r, u);
    }
    __syncthreads();   // the column constants are written
    for (int c = 0; c < nsub; ++c) {
      const uint32_t s_ = c_stage, par = c_par;
      if (++c_stage == static_cast<uint32_t>(stages)) {
        c_stage = 0;
        c_par ^= 1u;
      }
      const uint8_t* st = smem + s_ * stage_bytes;
      // thread 0 keeps stages - 1 segments in flight
      issue(c + stages - 1);
      // segment c has landed (every warp waits for itself)
      if (!mbar_wait_warp(&full_bar[s_], par, a.status, &abort_sh)) break;
      if (rp > 0 && lane == 0 && warp < nacc) {
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
        mma_commit(&empty_bar[s_]);
        if (c == nsub - 1) mma_commit(&unit_bar);
      }

      // ---- codes of segment c: the passes' loads first, then their arithmetic
      // (independent chains), then the stores of the rows below B
      const int cs = c * kSubCols + grp * kE;   // column of this thread's group, within the unit
      if (rr0 < kRows && c_lo + cs < c_hi) {
        const int64_t col = c_lo + cs;
        const uint32_t sbase = smem_u32(st);
        constexpr int kCh = kE / kPer16;         // 16-byte pieces per group
        const int ch = grp * kCh;
        float xv[kPasses][kE];
#pragma unroll
        for (int p = 0; p < kPasses; ++p)
#pragma unroll
          for (int h = 0; h < kCh; ++h)
            unpack16<TIn>(ld_shared_v4(sbase + swz(rr0 + p * kRpp, ch + h, kRows)), xv[p] + h * kPer16);
        float cv[kE];
#pragma unroll
        for (int j = 0; j < kE; ++j) cv[j] = colv[cs + j];
        if constexpr (!kFp4) {
          uint2 q[kPasses];
          int_codes8_rows<kPasses>(xv, cv, a.scale + col, s, a.qmax, q);
#pragma unroll
          for (int p = 0; p < kPasses; ++p) {
            const int64_t row = m0 + rr0 + p * kRpp;
            if (row < a.B) *reinterpret_cast<uint2*>(static_cast<int8_t*>(a.codes) + row * a.M + col) = q[p];
          }
        } else {
          const float* sc16 = a.scale + col;
#pragma unroll
          for (int p = 0; p < kPasses; ++p) {
            float xs[16];   // the estimates fl(x r_k) of the raw elements xv[p]
#pragma unroll
            for (int j = 0; j < 16; j += 2)
              upk2(fmul2_rn(pk2(xv[p][j], xv[p][j + 1]), pk2(cv[j], cv[j + 1])), xs[j], xs[j + 1]);
            float amax = block_amax_exact<16>(xv[p], xs, sc16);
            uint8_t sfb;
            float enc;
            if (mx) {
              // threads t and t ^ 1 hold the two halves of one 32-element block
              // (same row, same column block, same passes)
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
            for (int j = 0; j < 16; j += 2)
              upk2(fmul2_rn(pk2(xs[j], xs[j + 1]), pk2(enc, enc)), xs[j], xs[j + 1]);
            const uint2 q = make_uint2(e2m1x8_exact(xs, xv[p], enc, sc16), e2m1x8_exact(xs + 8, xv[p] + 8, enc, sc16 + 8));
            const int64_t row = m0 + rr0 + p * kRpp;
            if (row < a.B) {
              *reinterpret_cast<uint2*>(static_cast<uint8_t*>(a.codes) + row * (a.M / 2) + col / 2) = q;
              if (!mx)
                a.sf[sf_swizzle_offset(row, col / 16, kbp)] = sfb;
              else if ((lane & 1) == 0)
                a.sf[sf_swizzle_offset(row, col / 32, kbp)] = sfb;
            }
          }
        }
      }
      // this warp is done reading the stage
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty_bar[s_]);
    }
    // the unit's partial down tile: wait for its last MMAs, then TMEM -> ws_down;
    // the 16-column chunks go round the four warps of each TMEM lane quarter
    if (rp > 0) {
      if (!abort_sh) {
        const int quarter = warp & 3;
        const bool ok = mbar_wait_warp(&unit_bar, unit_parity, a.status, &abort_sh);
        tc_fence_after();
        const int row = m0 + quarter * 32 + lane;
        float* dst = a.ws_down + (static_cast<int64_t>(sp) * a.B + row) * rp;
        for (int c0 = 16 * (warp >> 2); c0 < rp; c0 += 16 * (kWorkWarps / 4)) {
          // the accumulators summed in issuer order
          float sum[16];
          for (int q = 0; q < nacc; ++q) {
            uint32_t v[16];
            tmem_ld_32x32b_x16(tmem + (static_cast<uint32_t>(quarter * 32) << 16) + acc_cols * q + c0, v);
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
        __threadfence();   // the partial is visible before the unit is counted
      }
      __syncthreads();
      if (tid == 0) last_sh = atomicAdd(a.ws_cnt + rb, 1u) == static_cast<unsigned>(npieces - 1);
      __syncthreads();
      if (last_sh) {
        // every unit of this row block is done: down = the partials summed in
        // split order, as bf16 hi | lo; four columns per thread, the loads of
        // three partials in flight at a time
        __threadfence();
        const float mult = nv ? (a.gs_w != nullptr ? __fmul_rn(gs_x, __ldg(a.gs_w)) : gs_x) : 1.0f;
        const int rows = min(kRows, a.B - m0);
        const int rp4 = rp / 4;
        const int64_t zs = static_cast<int64_t>(a.B) * rp4;   // float4s between partial tiles
        for (int i = tid; i < rows * rp4; i += kWork) {
          const int row = m0 + i / rp4, j = 4 * (i % rp4);
          const float4* src = reinterpret_cast<const float4*>(a.ws_down + static_cast<int64_t>(row) * rp + j);
          float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
          auto add = [&](const float4 v) {
            acc[0] += v.x;
            acc[1] += v.y;
            acc[2] += v.z;
            acc[3] += v.w;
          };
          int z = 0;
          for (; z + 3 <= npieces; z += 3) {
            const float4 v0 = __ldcg(src + z * zs), v1 = __ldcg(src + (z + 1) * zs), v2 = __ldcg(src + (z + 2) * zs);
            add(v0);
            add(v1);
            add(v2);
          }
          for (; z < npieces; ++z) add(__ldcg(src + z * zs));
          uint32_t hi[2], lo[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const float v0 = __fmul_rn(acc[2 * e], mult), v1 = __fmul_rn(acc[2 * e + 1], mult);
            const __nv_bfloat162 h = __floats2bfloat162_rn(v0, v1);
            const float2 hf = __bfloat1622float2(h);
            const __nv_bfloat162 l = __floats2bfloat162_rn(__fsub_rn(v0, hf.x), __fsub_rn(v1, hf.y));
            hi[e] = *reinterpret_cast<const uint32_t*>(&h);
            lo[e] = *reinterpret_cast<const uint32_t*>(&l);
          }
          __nv_bfloat16* drow = a.down + static_cast<int64_t>(row) * 2 * rp + j;   // 8-byte aligned
          *reinterpret_cast<uint2*>(drow) = make_uint2(hi[0], hi[1]);
          *reinterpret_cast<uint2*>(drow + rp) = make_uint2(lo[0], lo[1]);
        }
      }
    }
    unit_parity ^= 1u;
    __syncthreads();   // the drain is done and the column constants are free before the next unit
    if (abort_sh) break;
  }
  // no copy is still on its way when the CTA ends: the last segments' loads
  // were all waited for above, unless a wait ran out (then the status records it)
  if (!have_scale) take_scale();   // a CTA without pieces still waits (and CTA 0 writes the scale)
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
  if (rp > 0 && warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, acc_cols * nacc);
  }
}

template <typename TIn>
cudaError_t launch_max(const ActArgs& a, int grid, cudaStream_t stream) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kMaxThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = a.chained ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, act_max_kernel<TIn>, a);
}

template <typename TIn, bool kFp4>
cudaError_t launch_quant(const ActArgs& a, int grid, size_t smem, cudaStream_t stream) {
  constexpr int kEsz = static_cast<int>(sizeof(TIn));
  const CUtensorMapDataType dt = kEsz == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  CUtensorMap tx, tl;
  if (!make_tmap_2d(&tx, a.x, dt, kEsz, a.M, a.B, a.ldx, kTileBytes / kEsz, kRows, true))
    return cudaErrorInvalidValue;
  // without the down factor the ld map is never used: a valid stand-in (x) keeps the argument defined
  if (!make_tmap_2d(&tl, a.rank_pad > 0 ? a.ld : a.x, dt, kEsz, a.M, a.rank_pad > 0 ? a.rank_pad : a.B,
                    a.rank_pad > 0 ? a.M : a.ldx, kTileBytes / kEsz, a.rank_pad > 0 ? a.rank_pad : kRows, true))
    return cudaErrorInvalidValue;
  cudaError_t err = cudaFuncSetAttribute(act_quant_kernel<TIn, kFp4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
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
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, act_quant_kernel<TIn, kFp4>, tx, tl, a);
}

// Largest column count a unit may have: its per-column constants share the
// shared memory with two stages at least.
int max_unit_cols(int rank_pad) {
  const size_t two = 2 * static_cast<size_t>(quant_stage_bytes(rank_pad)) + 1024;
  return static_cast<int>((kQuantSmemBudget - two) / sizeof(float)) / 64 * 64;
}

}  // namespace

void finish_act_plan(ActPlan& p) {
  if (p.small) {
    finish_act_plan_small(p);
    return;
  }
  // pieces of at most max_unit_cols columns (the per-column constants live in
  // shared memory beside the stages)
  const int seg_cap = std::max(1, max_unit_cols(p.rank_pad) / p.tile_k);
  int steps_max;
  if (p.flat) {
    // every CTA a contiguous run of segments; as many CTAs as asked (the SMs),
    // more if a run would outgrow the shared memory
    const int64_t W = static_cast<int64_t>(p.nrb) * p.nsteps;
    const int64_t G = std::min(W, std::max<int64_t>(std::max(p.qgrid, 1), ceil_div(W, seg_cap)));
    p.grid = static_cast<int>(G);
    p.nunits = p.grid;
    // partial slots per row block: the most pieces a row block is cut into
    auto cta_of = [&](int64_t f) { return ((f + 1) * G - 1) / W; };
    int64_t maxp = 1;
    for (int64_t rb = 0; rb < p.nrb; ++rb)
      maxp = std::max(maxp, cta_of(rb * p.nsteps + p.nsteps - 1) - cta_of(rb * p.nsteps) + 1);
    p.ksplit = static_cast<int>(maxp);
    steps_max = static_cast<int>(std::min<int64_t>(p.nsteps, ceil_div(W, G)));
  } else {
    const int min_split = static_cast<int>(ceil_div(p.nsteps, seg_cap));
    p.ksplit = std::max(p.ksplit, std::min(p.nsteps, min_split));
    p.nunits = p.nrb * p.ksplit;
    steps_max = (p.nsteps + p.ksplit - 1) / p.ksplit;
    p.grid = std::min(p.nunits, num_sms());
  }
  const int unit_cols = steps_max * p.tile_k;
  const int sub_max = steps_max;
  const size_t sb = static_cast<size_t>(quant_stage_bytes(p.rank_pad));
  const size_t colv = static_cast<size_t>(unit_cols) * sizeof(float);
  p.stages = static_cast<int>(std::min<size_t>(kMaxStages, (kQuantSmemBudget - 1024 - colv) / sb));
  p.stages = std::max(2, std::min(p.stages, sub_max + 1));
  p.smem = sb * p.stages + colv + 1024;   // + alignment of the first stage to 1024 bytes
  // maximum kernel: slabs of kMaxSlab bytes x row ranges, about kMaxCtasPerSm CTAs per SM
  const int esz = p.bf16 ? 2 : 4;
  p.max_nslabs = static_cast<int>(ceil_div(p.M * esz, kMaxSlab));
  const int64_t target = static_cast<int64_t>(kMaxCtasPerSm) * num_sms();
  p.max_rpc = static_cast<int>(std::max<int64_t>(8, round_up(ceil_div(p.B * p.max_nslabs, target), 2)));
  p.nparts = static_cast<int>(p.max_nslabs * ceil_div(p.B, p.max_rpc));
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
  p.tile_k = p.bf16 ? kSub / 2 : kSub / 4;   // columns of a 256-byte segment
  p.nrb = static_cast<int>(ceil_div(B, kRows));
  p.nsteps = static_cast<int>(ceil_div(M, p.tile_k));
  // one quantise CTA per SM (most of the shared memory). With many segments per
  // SM they are spread flat (every SM busy; a CTA's run may be cut into two
  // pieces, each with its own pipeline start and drain); with few, a piece's
  // start and drain cost more than the SMs a K split leaves idle
  const int sms = num_sms();
  const int64_t W = static_cast<int64_t>(p.nrb) * p.nsteps;
  if (W >= static_cast<int64_t>(kFlatMinSegs) * sms) {
    p.flat = 1;
    p.qgrid = sms;
  } else {
    p.flat = 0;
    p.ksplit = std::max(1, std::min(p.nsteps, sms / std::max(p.nrb, 1)));
  }
  finish_act_plan(p);
  return p;
}

size_t act_scratch_bytes(const ActPlan& p) {
  if (p.small)   // partial maxima, then the partial down tiles (act_small.cu)
    return static_cast<size_t>(round_up(static_cast<int64_t>(p.grid) * 4, 256)) +
           (p.rank_pad > 0 ? static_cast<size_t>(round_up(static_cast<int64_t>(p.grid) * p.B * p.rank_pad * 4, 256)) : 0) +
           256;
  // partial maxima, row-block counters, partial down tiles
  size_t b = static_cast<size_t>(round_up(static_cast<int64_t>(std::max(p.nparts, 1)) * 4, 256)) +
             static_cast<size_t>(round_up(static_cast<int64_t>(p.nrb) * 4, 256));
  if (p.rank_pad > 0)
    b += static_cast<size_t>(round_up(static_cast<int64_t>(p.ksplit) * p.B * p.rank_pad * 4, 256));
  return b + 256;
}

cudaError_t launch_act(const ActPlan& p, const void* x, svdq_dtype xdt, int64_t ldx,
                       const float* scale, svdq_fmt fmt, const float* act_global_scale,
                       const float* w_global_scale, const void* ld, void* codes, void* sf,
                       float* act_scale, void* down, void* scratch, cudaStream_t stream,
                       bool* bad_args, unsigned* zero_words, int nzero) {
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
  // without the down factor the stages hold x alone (fewer bytes per stage,
  // the same split: the scratch layout does not change)
  ActPlan q = p;
  if (!has_ld) {
    q.rank_pad = 0;
    finish_act_plan(q);
  }
  Carver cv(scratch, ~size_t(0));
  float* ws_max = static_cast<float*>(cv.take(static_cast<size_t>(std::max(p.nparts, 1)) * 4));
  unsigned* ws_cnt = static_cast<unsigned*>(cv.take(static_cast<size_t>(p.nrb) * 4));
  float* ws_down =
      has_ld ? static_cast<float*>(cv.take(static_cast<size_t>(p.ksplit) * p.B * p.rank_pad * 4)) : nullptr;
  const bool need_max = fmt.kind == SVDQ_KIND_INT || (fmt.kind == SVDQ_KIND_NVFP4 && act_global_scale == nullptr);
  ActArgs a{};
  a.B = static_cast<int>(p.B);
  a.M = static_cast<int>(p.M);
  a.ldx = ldx;
  a.nsteps = p.nsteps;
  a.ksplit = p.ksplit;
  a.flat = p.flat;
  a.nrb = p.nrb;
  a.nunits = p.nunits;
  a.rank_pad = has_ld ? p.rank_pad : 0;
  a.has_ld = has_ld ? 1 : 0;
  a.nparts = need_max ? p.nparts : 0;
  a.max_rpc = p.max_rpc;
  a.max_nslabs = p.max_nslabs;
  a.fmt_kind = fmt.kind;
  a.qmax = fmt.kind == SVDQ_KIND_INT ? (1 << (fmt.bits - 1)) - 1 : 0;
  a.x = x;
  a.scale = scale;
  a.gs_given = fmt.kind == SVDQ_KIND_NVFP4 ? act_global_scale : nullptr;
  a.gs_w = fmt.kind == SVDQ_KIND_NVFP4 ? w_global_scale : nullptr;
  a.ld = has_ld ? ld : nullptr;
  a.ws_down = ws_down;
  a.ws_max = ws_max;
  a.ws_cnt = ws_cnt;
  a.codes = codes;
  a.sf = static_cast<uint8_t*>(sf);
  a.down = has_ld ? static_cast<__nv_bfloat16*>(down) : nullptr;
  a.act_scale = act_scale;
  a.status = device_status_word();
  a.stages = q.stages;
  // as many MMA issuers (up to 4) as TMEM holds accumulators of rank_pad columns
  a.nacc = a.rank_pad > 0 ? static_cast<int>(std::min<uint32_t>(4u, 512u / tmem_cols_for(a.rank_pad))) : 1;
  a.chained = p.chained;
  a.zero_words = zero_words;
  a.nzero = zero_words != nullptr ? nzero : 0;
  const int max_grid = need_max ? p.nparts : 1;
  cudaError_t err = xdt == SVDQ_BF16 ? launch_max<__nv_bfloat16>(a, max_grid, stream)
                                     : launch_max<float>(a, max_grid, stream);
  if (err != cudaSuccess) return err;
  const bool f4 = fmt.kind != SVDQ_KIND_INT;
  if (xdt == SVDQ_BF16)
    return f4 ? launch_quant<__nv_bfloat16, true>(a, p.grid, q.smem, stream)
              : launch_quant<__nv_bfloat16, false>(a, p.grid, q.smem, stream);
  return f4 ? launch_quant<float, true>(a, p.grid, q.smem, stream) : launch_quant<float, false>(a, p.grid, q.smem, stream);
}

}  // namespace svdq
