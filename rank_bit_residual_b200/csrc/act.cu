// act.cu - the activation pass of the SVDQuant linear, one cooperative kernel.
//
// "SVDQuant Smoothing, Low-rank and Residual Quantization", Formula items 1
// and 3: X_hat = x / scale is quantised per tensor (INT grid, or NVFP4 blocks
// for the variant of "flashinfer.gemm.svdquant_linear" step 1), and the
// low-rank branch needs X_hat L1 = x ld^T (step 2 of that page) from the same
// read of x.
//
// Work unit = 128 rows x a range of 128-byte K tiles. The kernel runs twice,
// and the boundary between the two launches is the grid-wide barrier the
// per-tensor scale needs (an in-kernel barrier would need its counter zeroed
// before every launch, a graph node that costs more than the barrier itself).
// Phase 1 streams the unit's x tiles in by TMA (128-byte swizzle), runs the
// down-projection on tcgen05 (bf16, or tf32 for fp32 x, accumulated in TMEM)
// and takes column maxima of |x| from the same shared-memory tiles; it writes
// a partial down tile and a partial maximum. Since fl(a r) is monotone in a,
// the tensor maximum of |X_hat| is max_k fl(colmax_k r_k). Phase 2 takes the
// per-tensor scale from the partial maxima, writes the codes from a second
// read of x (from L2 when x fits there) and sums the partial down tiles into
// bf16 hi | lo.
//
// fp32 evaluation order (the one the oracle's fp32 code mode repeats): the
// per-element divisions of the definition are multiplies by correctly rounded
// reciprocals, r_k = fl(1 / scale_k) once per column and u = fl(1 / s) once
// per tensor: X_hat = fl(x r_k), INT code = rint(fl(x c_k)) with the per-column
// constant c_k = fl(r_k u).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "encode.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace svdq {

namespace {

constexpr int kWorkWarps = 16;
constexpr int kWork = 32 * kWorkWarps;      // threads for column maxima, codes and down
constexpr int kThreads = kWork + 64;        // + a TMA warp and an MMA warp
constexpr int kTmaWarp = kWorkWarps;
constexpr int kMmaWarp = kWorkWarps + 1;
constexpr int kRows = 128;                  // rows per unit (MMA M)
constexpr int kTileBytes = kRows * 128;     // one 128 x 128-byte x tile
constexpr int kXRing = 4;                   // x tile buffers when the tiles are not held
constexpr int kLdRing = 6;                  // ld tile slots
constexpr int kMaxHold = 12;                // x tiles a unit may keep in shared memory
constexpr int kSmemBudget = 224 * 1024;

__host__ __device__ constexpr uint32_t pow2_cols(int n) {
  return n <= 32 ? 32u : n <= 64 ? 64u : n <= 128 ? 128u : 256u;
}

struct ActArgs {
  int B, M;
  int64_t ldx;
  int nsteps, ksplit, nrb, nunits, rank_pad, has_ld, xbuf, fmt_kind, qmax;
  int phase;        // 1: tiles, column maxima, partial down tiles; 2: codes and the down tile
  int nparts;       // partial maxima written by phase 1
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
  unsigned* status;
};

// Column maxima of |x| over a 128 x 128-byte swizzled tile (work threads only,
// t < kWork). Thread t owns the
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
  for (int i = 0; i < kRows / (kWork / 8); ++i) {
    const uint4 v = *reinterpret_cast<const uint4*>(tile + (rg + (kWork / 8) * i) * 128 + p * 16);
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
// Barrier among the work warps only (the TMA and MMA warps run their own loops).
__device__ __forceinline__ void work_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(kWork) : "memory");
}

// Eight consecutive elements of x (16 bytes of bf16, or 32 of fp32) from a held
// swizzled tile row or from global memory; cl: column within the unit, a
// multiple of 8.
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

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
// Waits until at most n of this thread's copy groups are still in flight.
__device__ __forceinline__ void cp_async_wait(int n) {
  switch (n) {
    case 0: asm volatile("cp.async.wait_group 0;" ::: "memory"); break;
    case 1: asm volatile("cp.async.wait_group 1;" ::: "memory"); break;
    case 2: asm volatile("cp.async.wait_group 2;" ::: "memory"); break;
    case 3: asm volatile("cp.async.wait_group 3;" ::: "memory"); break;
    case 4: asm volatile("cp.async.wait_group 4;" ::: "memory"); break;
    default: asm volatile("cp.async.wait_group 5;" ::: "memory"); break;
  }
}

// Warp roles: warps 0-15 ("work") take the column maxima in phase 1 and write
// the codes and the down factor in phase 2; warp 16 loads the x tiles by TMA
// (lane 0); warp 17 copies the ld tiles with cp.async (all lanes: a path apart
// from the TMA queue, so the small ld tiles never wait behind the x tiles) and
// issues the down-projection MMAs (lane 0). No block-wide barrier separates the
// K steps: the work warps follow the x tiles as they land, and the MMA chain
// runs on its own. The MMA warp issues one throwaway MMA first: the first
// tcgen05.mma a kernel issues takes microseconds longer than the ones after
// it, and this way that start-up overlaps the first loads.
template <typename TIn>
__global__ void __launch_bounds__(kThreads, 1)
    act_fused_kernel(const __grid_constant__ CUtensorMap tm_x, const ActArgs a) {
  constexpr int kTileK = 128 / static_cast<int>(sizeof(TIn));   // elements per 128-byte row
  constexpr int kPerChunk = 16 / static_cast<int>(sizeof(TIn)); // elements per 16 bytes
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t xfull[kMaxHold];
  __shared__ __align__(8) uint64_t xempty[kMaxHold];
  __shared__ __align__(8) uint64_t ld_free;
  __shared__ __align__(8) uint64_t mma_done;
  __shared__ __align__(8) uint64_t tmem_free;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;
  __shared__ float red[kWorkWarps];

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool producer = warp >= kWorkWarps;   // the TMA or the MMA warp
  const int ld_bytes = a.rank_pad * 128;
  uint8_t* xbuf = smem;                                               // a.xbuf tiles
  uint8_t* ldbuf = smem + static_cast<size_t>(a.xbuf) * kTileBytes;   // kLdRing ld tiles
  const bool mma_phase = a.phase == 1 && a.has_ld;   // the down-projection runs in phase 1
  float* rcp = reinterpret_cast<float*>(ldbuf + (mma_phase ? kLdRing * ld_bytes : 0));
  const uint32_t tcols = pow2_cols(a.rank_pad);
  unsigned* status = a.status;

  auto unit_range = [&](int unit, int& m0, int& k_lo, int& n) {
    const int rb = unit % a.nrb, sp = unit / a.nrb;
    m0 = rb * kRows;
    k_lo = static_cast<int>((static_cast<int64_t>(a.nsteps) * sp) / a.ksplit);
    n = static_cast<int>((static_cast<int64_t>(a.nsteps) * (sp + 1)) / a.ksplit) - k_lo;
  };

  if (tid == kWork) {
    for (int s = 0; s < kMaxHold; ++s) {
      mbar_init(&xfull[s], 1);
      mbar_init(&xempty[s], kWorkWarps + (a.has_ld ? 1 : 0));
    }
    mbar_init(&ld_free, 1);
    mbar_init(&mma_done, 1);
    mbar_init(&tmem_free, 4);
    fence_mbar_init();
    abort_sh = 0;
    tma_prefetch_desc(&tm_x);
  }
  if (warp == kMmaWarp && mma_phase) {
    tmem_alloc(&tmem_base_sh, tcols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = mma_phase ? tmem_base_sh : 0u;
  float run = 0.0f;
  bool ok = true;

  // ================================================================ phase 1
  if (a.phase == 1) {
  // x steps flow through the buffers as one ring over all of this CTA's units:
  // step G + i uses buffer (G + i) % xbuf in its use (G + i) / xbuf (counters
  // in registers: an indexed array would live in local memory)
  if (warp == kTmaWarp) {
    if (lane == 0) {
      uint32_t G = 0;   // x steps of the previous units
      bool pok = true;
      for (int unit = blockIdx.x; unit < a.nunits && pok; unit += gridDim.x) {
        int m0, k_lo, n;
        unit_range(unit, m0, k_lo, n);
        for (int i = 0; i < n && pok; ++i) {
          const uint32_t gs = G + i;
          const uint32_t b = gs % a.xbuf, use = gs / a.xbuf;
          if (use > 0)  // the previous tile in this buffer is fully read
            pok = mbar_wait(&xempty[b], (use - 1) & 1, status, &abort_sh);
          if (!pok) break;
          mbar_arrive_expect_tx(&xfull[b], kTileBytes);
          tma_load_2d(xbuf + static_cast<size_t>(b) * kTileBytes, &tm_x, &xfull[b], (k_lo + i) * kTileK, m0);
        }
        G += n;
      }
      if (!pok) {
        abort_sh = 1;
        // let loads already issued land before the block moves on (the loads
        // of the last xbuf steps of the ring, at most)
        for (uint32_t gs = G > static_cast<uint32_t>(a.xbuf) ? G - a.xbuf : 0u; gs < G; ++gs)
          mbar_wait(&xfull[gs % a.xbuf], (gs / a.xbuf) & 1, status, nullptr, 1000000ull);
      }
    }
  } else if (warp == kMmaWarp) {
    if (mma_phase) {
      uint32_t G = 0;        // x steps of the previous units
      uint32_t nbatch = 0;   // ld batches whose MMAs were committed to ld_free
      bool pok = true;
      // ld tiles of K tiles k_lo + j0 .. + cnt - 1 into slots 0 .. cnt - 1, one
      // copy group per lane; ld is [rank_pad, M] row-major, columns past M are
      // filled with zeros. The slots are free once the previous batch's MMAs
      // are done.
      auto copy_batch = [&](int k_lo, int j0, int cnt) {
        if (nbatch > 0) pok = mbar_wait_warp(&ld_free, (nbatch - 1) & 1, status, &abort_sh) && pok;
        const TIn* ld = static_cast<const TIn*>(a.ld);
        for (int t = 0; t < cnt; ++t) {
          uint8_t* dst = ldbuf + static_cast<size_t>(t) * ld_bytes;
          for (int c = lane; c < a.rank_pad * 8; c += 32) {
            const int r = c >> 3, cc = c & 7;
            const int col = (k_lo + j0 + t) * kTileK + cc * kPerChunk;
            const bool in = col < a.M;
            cp_async16(smem_u32(dst + r * 128 + ((cc ^ (r & 7)) << 4)),
                       in ? static_cast<const void*>(ld + static_cast<int64_t>(r) * a.M + col) : a.ld,
                       in ? 16u : 0u);
          }
        }
        cp_async_commit();
      };
      const uint32_t idesc = sizeof(TIn) == 2 ? idesc_bf16(128, a.rank_pad) : idesc_tf32(128, a.rank_pad);
      if (lane == 0) {
        // throwaway MMA (its result is overwritten by the first real one)
        const uint64_t ad = smem_desc_sw128(smem_u32(xbuf)), bd = smem_desc_sw128(smem_u32(ldbuf));
        if (sizeof(TIn) == 2)
          mma_f16(tmem, ad, bd, idesc, 0u);
        else
          mma_tf32(tmem, ad, bd, idesc, 0u);
      }
      __syncwarp();
      uint32_t ucount = 0;
      for (int unit = blockIdx.x; unit < a.nunits && pok; unit += gridDim.x, ++ucount) {
        int m0, k_lo, n;
        unit_range(unit, m0, k_lo, n);
        for (int j0 = 0; j0 < n && pok; j0 += kLdRing) {
          const int cnt = min(kLdRing, n - j0);
          copy_batch(k_lo, j0, cnt);
          if (lane == 0 && ucount > 0 && j0 == 0)  // the work warps have read the previous unit's accumulator
            pok = pok && mbar_wait(&tmem_free, (ucount - 1) & 1, status, &abort_sh);
          cp_async_wait(0);  // this lane's copies have landed
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            for (int t = 0; t < cnt && pok; ++t) {
              const int i = j0 + t;
              const uint32_t b = (G + i) % a.xbuf;
              pok = mbar_wait(&xfull[b], ((G + i) / a.xbuf) & 1, status, &abort_sh);
              if (!pok) break;
              tc_fence_after();
              const uint32_t a0 = smem_u32(xbuf + static_cast<size_t>(b) * kTileBytes);
              const uint32_t b0 = smem_u32(ldbuf + static_cast<size_t>(t) * ld_bytes);
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                const uint64_t ad = smem_desc_sw128(a0 + 32 * kk);
                const uint64_t bd = smem_desc_sw128(b0 + 32 * kk);
                if (sizeof(TIn) == 2)
                  mma_f16(tmem, ad, bd, idesc, (i > 0 || kk > 0) ? 1u : 0u);
                else
                  mma_tf32(tmem, ad, bd, idesc, (i > 0 || kk > 0) ? 1u : 0u);
              }
              mma_commit(&xempty[b]);
            }
            if (pok) mma_commit(&ld_free);
          }
          ++nbatch;
          pok = __shfl_sync(0xffffffffu, pok ? 1 : 0, 0) != 0;
        }
        if (lane == 0 && pok) mma_commit(&mma_done);
        G += n;
      }
      cp_async_wait(0);
      if (lane == 0 && !pok) abort_sh = 1;
    }
  } else {
    uint32_t G = 0;   // x steps of the previous units (the same ring as the producer's)
    uint32_t ucount = 0;
    for (int unit = blockIdx.x; unit < a.nunits; unit += gridDim.x, ++ucount) {
      int m0, k_lo, n;
      unit_range(unit, m0, k_lo, n);
      work_sync();  // the previous unit's reciprocals are no longer read
      for (int j = tid; j < n * kTileK; j += kWork) {
        const int col = k_lo * kTileK + j;
        rcp[j] = col < a.M ? __frcp_rn(__ldg(a.scale + col)) : 0.0f;
      }
      work_sync();
      for (int i = 0; i < n; ++i) {
        const uint32_t b = (G + i) % a.xbuf;
        ok = mbar_wait_warp(&xfull[b], ((G + i) / a.xbuf) & 1, status, &abort_sh) && ok;
        if (ok) run = tile_absmax<TIn>(xbuf + static_cast<size_t>(b) * kTileBytes, rcp + i * kTileK, run);
        __syncwarp();
        if (lane == 0) mbar_arrive(&xempty[b]);
      }
      if (mma_phase && warp < 4) {
        // drain the unit's accumulator into its partial before the next
        // unit's MMAs; TMEM lane = row, warps 0-3 cover the 128 lanes
        const bool fin = mbar_wait_warp(&mma_done, ucount & 1, status, &abort_sh) && ok;
        tc_fence_after();
        const int row = m0 + warp * 32 + lane;
        const int sp = unit / a.nrb;
        float* dst = a.ws_down + (static_cast<int64_t>(sp) * a.B + row) * a.rank_pad;
        for (int c0 = 0; c0 < a.rank_pad; c0 += 32) {
          uint32_t v[32];
          __syncwarp();
          tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(warp * 32) << 16) + c0, v);
          tmem_ld_wait_regs(v);
          if (fin && row < a.B) {
            const int cnt = min(32, a.rank_pad - c0);
            for (int j = 0; j < cnt; j += 4)
              *reinterpret_cast<float4*>(dst + c0 + j) =
                  make_float4(__uint_as_float(v[j]), __uint_as_float(v[j + 1]),
                              __uint_as_float(v[j + 2]), __uint_as_float(v[j + 3]));
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tmem_free);
        ok = ok && fin;
      }
      G += n;
    }
    // per-CTA maximum -> ws_max[blockIdx.x]
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) run = fmaxf(run, __shfl_xor_sync(0xffffffffu, run, o));
    if (lane == 0) red[warp] = run;
    work_sync();
    if (tid == 0) {
      float m = red[0];
      for (int w = 1; w < kWorkWarps; ++w) m = fmaxf(m, red[w]);
      a.ws_max[blockIdx.x] = ok ? m : 0.0f;
    }
  }
  }   // phase 1

  // ================================================================ phase 2
  if (a.phase == 2 && !producer) {
    float m = 0.0f;
    for (int i = tid; i < a.nparts; i += kWork) m = fmaxf(m, __ldcg(a.ws_max + i));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    work_sync();
    if (lane == 0) red[warp] = m;
    work_sync();
    m = red[0];
    for (int w = 1; w < kWorkWarps; ++w) m = fmaxf(m, red[w]);
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
      int m0, k_lo, n;
      unit_range(unit, m0, k_lo, n);
      const int sp = unit / a.nrb;
      const int64_t col0 = static_cast<int64_t>(k_lo) * kTileK;
      work_sync();
      for (int j = tid; j < n * kTileK; j += kWork) {
        const int col = k_lo * kTileK + j;
        rcp[j] = col < a.M ? __frcp_rn(__ldg(a.scale + col)) : 0.0f;
      }
      work_sync();
      const int rows = min(kRows, a.B - m0);
      const int ncols = min(n * kTileK, a.M - k_lo * kTileK);   // a multiple of 32
      if (!nv) {
        // a warp writes 256 consecutive codes of a row (8 per lane, one 256-byte
        // store), two rows (r, r + 16) at a time
        for (int c256 = 0; c256 < ncols; c256 += 256) {
          const int cl = c256 + 8 * lane;
          const bool live = cl < ncols;
          float ck[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) ck[j] = live ? __fmul_rn(rcp[cl + j], u) : 0.0f;
          for (int r = warp; r < rows; r += 2 * kWorkWarps) {
            const int r2 = r + kWorkWarps;
            const bool two = r2 < rows;
            uint4 ua[2], ub[2];
            if (live) {
              load8<TIn>(a.x, a.ldx, m0 + r, col0, cl, ua);
              if (two) load8<TIn>(a.x, a.ldx, m0 + r2, col0, cl, ub);
            }
            if (live) {
              float v[8];
              unpack8<TIn>(ua, v);
              *reinterpret_cast<uint2*>(static_cast<int8_t*>(a.codes) + static_cast<int64_t>(m0 + r) * a.M +
                                        col0 + cl) = int_codes8(v, ck);
              if (two) {
                unpack8<TIn>(ub, v);
                *reinterpret_cast<uint2*>(static_cast<int8_t*>(a.codes) +
                                          static_cast<int64_t>(m0 + r2) * a.M + col0 + cl) = int_codes8(v, ck);
              }
            }
          }
        }
      } else {
        // half a warp = 256 consecutive elements of one row (one 16-element block per lane)
        const int nch = (ncols + 255) / 256;
        const int items = nch * rows;
        for (int base = 2 * warp; base < items; base += 2 * kWorkWarps) {
          const int it = base + (lane >> 4);
          if (it >= items) continue;
          const int cc = it / rows, r = it - cc * rows;
          const int cl = cc * 256 + 16 * (lane & 15);
          if (cl >= ncols) continue;
          float xs[16];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            uint4 uu[2];
            float v8[8];
            load8<TIn>(a.x, a.ldx, m0 + r, col0, cl + 8 * h, uu);
            unpack8<TIn>(uu, v8);
#pragma unroll
            for (int j = 0; j < 8; ++j) xs[8 * h + j] = v8[j];
          }
          float amax = 0.0f;
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            xs[j] = __fmul_rn(xs[j], rcp[cl + j]);
            amax = fmaxf(amax, fabsf(xs[j]));
          }
          const uint8_t sfb = f32_to_ue4m3(__fmul_rn(__fdiv_rn(amax, 6.0f), gs_x));
          const float d = ue4m3_to_f32(sfb);
          const float enc = d > 0.0f ? __fdiv_rn(gs_x, d) : 0.0f;
#pragma unroll
          for (int j = 0; j < 16; ++j) xs[j] = __fmul_rn(xs[j], enc);
          const int64_t row = m0 + r;
          const int64_t col = col0 + cl;
          *reinterpret_cast<uint2*>(static_cast<uint8_t*>(a.codes) + row * (a.M / 2) + col / 2) =
              make_uint2(f32x8_to_e2m1(xs), f32x8_to_e2m1(xs + 8));
          a.sf[sf_swizzle_offset(row, col / 16, kbp)] = sfb;
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
    // NVFP4: zero the scale padding (rows up to a multiple of 128, columns up to 4)
    if (nv) {
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

  __syncthreads();
  if (mma_phase && warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, tcols);
  }
}

size_t smem_for(const ActPlan& p, int xbuf) {
  const int ld_bytes = p.rank_pad * 128;
  const int steps_max = (p.nsteps + p.ksplit - 1) / p.ksplit;
  return static_cast<size_t>(xbuf) * kTileBytes + (p.rank_pad > 0 ? kLdRing * ld_bytes : 0) +
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
  if (p.small) {
    finish_act_plan_small(p);
    return;
  }
  p.nunits = p.nrb * p.ksplit;
  const int steps_max = (p.nsteps + p.ksplit - 1) / p.ksplit;
  // all of a unit's x tiles in flight at once when they fit (a deep TMA queue),
  // else a ring of kXRing tiles
  p.xbuf = kXRing;
  if (steps_max <= kMaxHold && smem_for(p, steps_max) <= static_cast<size_t>(kSmemBudget)) p.xbuf = steps_max;
  p.smem = smem_for(p, p.xbuf);
  p.grid = std::min(p.nunits, num_sms() * resident_per_sm(p.smem, p.bf16));
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
  Carver cv(scratch, ~size_t(0));
  float* ws_max = static_cast<float*>(cv.take(static_cast<size_t>(std::max(p.grid, 1)) * 4));
  float* ws_down =
      has_ld ? static_cast<float*>(cv.take(static_cast<size_t>(p.ksplit) * p.B * p.rank_pad * 4))
             : nullptr;
  const int esz = xdt == SVDQ_BF16 ? 2 : 4;
  const CUtensorMapDataType cdt =
      xdt == SVDQ_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  CUtensorMap tm_x;
  if (!make_tmap_2d(&tm_x, x, cdt, esz, p.M, p.B, ldx, p.tile_k, kRows, true) ||
      (has_ld && (reinterpret_cast<uintptr_t>(ld) & 15) != 0)) {
    *bad_args = true;
    return cudaSuccess;
  }
  cudaError_t err;
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
  a.xbuf = p.xbuf;
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
  // without the down factor the launch needs no ld ring (plan keeps its grid)
  ActPlan q = p;
  if (!has_ld) q.rank_pad = 0;
  const size_t smem1 = smem_for(q, p.xbuf);
  // phase 2 keeps only the unit's reciprocals in shared memory
  const int steps_max = (p.nsteps + p.ksplit - 1) / p.ksplit;
  const size_t smem2 = static_cast<size_t>(steps_max) * p.tile_k * sizeof(float) + 1024;
  ActArgs a2 = a;
  a.phase = 1;
  a2.phase = 2;
  a2.xbuf = 0;
  if (xdt == SVDQ_BF16) {
    err = cudaFuncSetAttribute(act_fused_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(std::max(smem1, smem2)));
    if (err != cudaSuccess) return err;
    act_fused_kernel<__nv_bfloat16><<<p.grid, kThreads, smem1, stream>>>(tm_x, a);
    err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    act_fused_kernel<__nv_bfloat16><<<p.nunits, kThreads, smem2, stream>>>(tm_x, a2);
  } else {
    err = cudaFuncSetAttribute(act_fused_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(std::max(smem1, smem2)));
    if (err != cudaSuccess) return err;
    act_fused_kernel<float><<<p.grid, kThreads, smem1, stream>>>(tm_x, a);
    err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    act_fused_kernel<float><<<p.nunits, kThreads, smem2, stream>>>(tm_x, a2);
  }
  return cudaGetLastError();
}

}  // namespace svdq
