// gemm_skinny.cu - the residual GEMM with the low-rank epilogue for short
// batches (B <= 128 rows), where the weight stream from HBM is the cost.
//
// "SVDQuant Smoothing, Low-rank and Residual Quantization", Formula item 3:
//   Y = (X_hat L1) L2 + Q(X_hat) Q(R)
// from prepared operands (step 3 of "flashinfer.gemm.svdquant_linear": the
// residual GEMM with the low-rank up-projection and bias in its epilogue).
//
// Orientation: the weight rows are the MMA's M side (128 per tile) and the
// batch is its N side (Bp = B rounded up to 16), so a batch of one wastes no
// tensor-core rows:  D[n, b] = sum_k W[n, k] X[b, k].
// Each 128-row weight tile is one cluster of S CTAs that split K; every CTA
// sees only 1/S of the tile's weights, so all SMs stream weights at once.
// The partial tiles are combined through distributed shared memory: each CTA
// stores its partial of the output columns owned by CTA p straight into p's
// shared memory, and p sums the S partials in rank order (a fixed order) and
// writes Y.
//
// Weights are loaded before griddepcontrol.wait: launched with programmatic
// serialization right after the activation pass, the weight stream overlaps
// that kernel; only the activation-side loads and the epilogue wait for it.
//
// Formats:
//   INT, int8 codes     A tiles come by TMA (128-byte swizzle)       kind::i8
//   INT, packed 4-bit   64-byte packed rows by TMA, widened to int8 in shared
//                       memory by the epilogue warps                 kind::i8
//   NVFP4               e2m1 tiles by TMA, ue4m3 scales by bulk copy
//                       then tcgen05.cp to TMEM                      kind::mxf4nvf4
//   MXFP4               the same with E8M0 scales per 32 elements    kind::mxf4
// Low-rank branch: lu (weight side) x down hi|lo (batch side), kind::f16, in
// 64-wide K boxes spread over the cluster's CTAs; INT keeps it in its own fp32
// accumulator, fp4 adds it to the residual accumulator (down is pre-scaled
// by gs_x gs_w, which MXFP4 does not have: 1).
//
// Warps: 0 weight loads, 1 activation loads, 2 TMEM + MMA issue,
//        3-6 widening of packed codes, then the epilogue (TMEM lane quarter w % 4).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "encode.cuh"
#include "gemm_common.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace svdq {

namespace {

constexpr int kTileN = 128;
constexpr int kThreads = 224;
constexpr int kWarpW = 0, kWarpX = 1, kWarpMma = 2, kWarpEpi0 = 3;
constexpr int kMaxRing = 8;
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kLrCol = 128;                      // INT: low-rank fp32 accumulator
constexpr uint32_t kSfaCol = 128, kSfbCol = 144;      // fp4: scale factors (4 columns per 128x4 atom)
constexpr int kATile = 16384;                         // 128 rows x 128 bytes
constexpr int kPSlot = 8192;                          // 128 rows x 64 packed bytes
constexpr int kSfBytes = 2048;                        // up to 4 scale atoms of 512 bytes
constexpr size_t kSmemBudget = 200 * 1024;
constexpr size_t kMinSmem = 120 * 1024;

enum SkinnyFmt { kFmtInt8 = 0, kFmtInt4 = 1, kFmtNvfp4 = 2, kFmtMxfp4 = 3 };

constexpr bool fmt_is_f4(int f) { return f == kFmtNvfp4 || f == kFmtMxfp4; }
// 128x4 scale atoms per 128-row tile and 256-element K step: four scales per
// row cover 64 elements of NVFP4 (16-element blocks), 128 of MXFP4
constexpr int sf_atoms_per_step(int f) { return f == kFmtNvfp4 ? 4 : (f == kFmtMxfp4 ? 2 : 0); }

struct SkinnyArgs {
  int B, Bp, N, M, S, kst, lr_boxes, sh;
  int dr, dp, a_slot, b_slot;   // ring depth (both operands), packed-weight ring depth
  int katoms;
  const float* s_x;
  const float* s_w;
  const __nv_bfloat16* bias;
  void* y;
  int64_t ldy;
  int vec_ok;
  const uint8_t* sfw;   // fp4 weight scales, 128x4 layout
  const uint8_t* sfx;   // fp4 activation scales, 128x4 layout
  unsigned* status;
};

// Dequantisation factor of the residual accumulator (s_x s_w for INT,
// 1 / (gs_x gs_w) for fp4, 1 for MXFP4; unused for the raw int32 product).
template <int kFmt, int kOut>
__device__ __forceinline__ float skinny_alpha(const SkinnyArgs& a) {
  if (kOut == kOutI32) return 0.0f;
  if (fmt_is_f4(kFmt)) return __fdiv_rn(1.0f, __fmul_rn(__ldg(a.s_x), __ldg(a.s_w)));
  return __ldg(a.s_x) * __ldg(a.s_w);
}

template <int kFmt, int kOut>
__global__ void __launch_bounds__(kThreads, 1)
    skinny_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_x,
                  const __grid_constant__ CUtensorMap tm_lu, const __grid_constant__ CUtensorMap tm_dn,
                  const SkinnyArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // one ring for both operands: full[s] completes when the weight side (TMA, or
  // the four widening warps) and the activation side have both landed; one
  // MMA commit per step frees both halves of the slot (empty[s])
  __shared__ __align__(8) uint64_t full[kMaxRing];
  __shared__ __align__(8) uint64_t empty[kMaxRing];
  __shared__ __align__(8) uint64_t full_p[kMaxRing];
  __shared__ __align__(8) uint64_t empty_p[kMaxRing];
  __shared__ __align__(8) uint64_t tmem_full;
  __shared__ __align__(8) uint64_t mma_done;
  __shared__ __align__(8) uint64_t recv_bar;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  // a chained linear's activation pass queued after this kernel may start its
  // weight-side setup now (it reads this kernel's output only after griddepcontrol.wait)
  pdl_trigger();
  uint8_t* ring_a = smem;
  uint8_t* ring_b = ring_a + static_cast<size_t>(a.dr) * a.a_slot;
  uint8_t* ring_p = ring_b + static_cast<size_t>(a.dr) * a.b_slot;
  uint32_t* recv_base = reinterpret_cast<uint32_t*>(smem);   // partials: reuse the rings once every MMA is done

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = a.S;
  const int rank = static_cast<int>(cluster_ctarank());
  const int n0 = blockIdx.y * kTileN;
  const int k_lo = (a.kst * rank) / S, k_hi = (a.kst * (rank + 1)) / S;
  const int nres = k_hi - k_lo;
  const int nlr = a.lr_boxes > rank ? (a.lr_boxes - rank + S - 1) / S : 0;  // boxes rank, rank + S, ...
  const int nsteps = nlr + nres;
  unsigned* status = a.status;
  constexpr uint32_t kFullACount = kFmt == kFmtInt4 ? 4u : 1u;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kMaxRing; ++s) {
      mbar_init(&full[s], kFullACount + 1);
      mbar_init(&empty[s], 1);
      mbar_init(&full_p[s], 1);
      mbar_init(&empty_p[s], 4);
    }
    mbar_init(&tmem_full, 1);
    mbar_init(&mma_done, 1);
    mbar_init(&recv_bar, 1);
    fence_mbar_init();
    // the shares the other S - 1 CTAs will copy here
    mbar_arrive_expect_tx(&recv_bar, static_cast<uint32_t>((S - 1) * a.B * a.sh * 4));
    abort_sh = 0;
    tma_prefetch_desc(&tm_w);
    tma_prefetch_desc(&tm_x);
    if (a.lr_boxes) {
      tma_prefetch_desc(&tm_lu);
      tma_prefetch_desc(&tm_dn);
    }
  }
  if (warp == kWarpMma) {
    tmem_alloc(&tmem_base_sh, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;

  if (warp == kWarpW) {
    // ---------------------------------------------------- weight producer
    if (lane == 0) {
      bool ok = true;
      int ia = 0, ip = 0;   // A-ring loads (lu boxes, direct weight tiles) and packed loads issued
      // low-rank step i (< nlr): the lu box rank + i S into A slot i % da
      auto load_lu = [&](int i) {
        const int s = i % a.dr;
        if (i >= a.dr) ok = ok && mbar_wait(&empty[s], ((i / a.dr) - 1) & 1, status, &abort_sh);
        if (!ok) return;
        mbar_arrive_expect_tx(&full[s], kATile);
        for (uint32_t c = 1; c < kFullACount; ++c) mbar_arrive(&full[s]);
        tma_load_2d(ring_a + static_cast<size_t>(s) * a.a_slot, &tm_lu, &full[s], 64 * (rank + i * S), n0);
        ++ia;
      };
      if constexpr (kFmt == kFmtInt4) {
        // packed residual step r into P slot r % dp; the first dp go out before
        // anything can block
        auto load_p = [&](int r) {
          const int s = r % a.dp;
          if (r >= a.dp) ok = ok && mbar_wait(&empty_p[s], ((r / a.dp) - 1) & 1, status, &abort_sh);
          if (!ok) return;
          mbar_arrive_expect_tx(&full_p[s], kPSlot);
          tma_load_2d(ring_p + static_cast<size_t>(s) * kPSlot, &tm_w, &full_p[s], 64 * (k_lo + r), n0);
          ++ip;
        };
        int r = 0;
        for (; r < min(a.dp, nres) && ok; ++r) load_p(r);
        for (int i = 0; i < nlr && ok; ++i) load_lu(i);
        for (; r < nres && ok; ++r) load_p(r);
      } else {
        for (int i = 0; i < nsteps && ok; ++i) {
          if (i < nlr) {
            load_lu(i);
            continue;
          }
          const int s = i % a.dr, k = k_lo + (i - nlr);
          if (i >= a.dr) ok = ok && mbar_wait(&empty[s], ((i / a.dr) - 1) & 1, status, &abort_sh);
          if (!ok) break;
          uint8_t* dst = ring_a + static_cast<size_t>(s) * a.a_slot;
          if constexpr (fmt_is_f4(kFmt)) {
            constexpr int kAt = sf_atoms_per_step(kFmt);
            const int na = min(kAt, a.katoms - kAt * k);
            mbar_arrive_expect_tx(&full[s], kATile + na * 512);
            tma_load_2d(dst, &tm_w, &full[s], 128 * k, n0);
            bulk_load(dst + kATile, a.sfw + (static_cast<int64_t>(n0 / 128) * a.katoms + kAt * k) * 512, na * 512,
                      &full[s]);
          } else {
            mbar_arrive_expect_tx(&full[s], kATile);
            tma_load_2d(dst, &tm_w, &full[s], 128 * k, n0);
          }
          ++ia;
        }
      }
      if (!ok) {
        // the MMAs will not consume what is in flight: let it land before the
        // block can exit (on the normal path every load was consumed)
        abort_sh = 1;
        if (kFmt != kFmtInt4)
          for (int q = max(0, ia - a.dr); q < ia; ++q)
            mbar_wait(&full[q % a.dr], (q / a.dr) & 1, status, nullptr, 1000000ull);
        for (int q = max(0, ip - a.dp); q < ip; ++q)
          mbar_wait(&full_p[q % a.dp], (q / a.dp) & 1, status, nullptr, 1000000ull);
      }
    }
  } else if (warp == kWarpX) {
    // ------------------------------------------------ activation producer
    if (lane == 0) {
      pdl_wait();   // codes, scales and down come from the activation pass
      bool ok = true;
      int ib = 0;   // loads issued
      const int xbytes = a.Bp * 128;
      for (int i = 0; i < nsteps && ok; ++i, ++ib) {
        const int s = i % a.dr;
        if (i >= a.dr) ok = mbar_wait(&empty[s], ((i / a.dr) - 1) & 1, status, &abort_sh);
        if (!ok) break;
        uint8_t* dst = ring_b + static_cast<size_t>(s) * a.b_slot;
        if (i < nlr) {
          mbar_arrive_expect_tx(&full[s], xbytes);
          tma_load_2d(dst, &tm_dn, &full[s], 64 * (rank + i * S), 0);
        } else {
          const int k = k_lo + (i - nlr);
          if constexpr (fmt_is_f4(kFmt)) {
            constexpr int kAt = sf_atoms_per_step(kFmt);
            const int na = min(kAt, a.katoms - kAt * k);
            mbar_arrive_expect_tx(&full[s], xbytes + na * 512);
            tma_load_2d(dst, &tm_x, &full[s], 128 * k, 0);
            bulk_load(dst + xbytes, a.sfx + static_cast<int64_t>(kAt * k) * 512, na * 512, &full[s]);
          } else {
            mbar_arrive_expect_tx(&full[s], xbytes);
            tma_load_2d(dst, &tm_x, &full[s], 128 * k, 0);
          }
        }
      }
      if (!ok) {
        abort_sh = 1;
        for (int q = max(0, ib - a.dr); q < ib; ++q)
          mbar_wait(&full[q % a.dr], (q / a.dr) & 1, status, nullptr, 1000000ull);
      }
    }
  } else if (warp == kWarpMma) {
    // ---------------------------------------------------------------- MMA
    if (lane == 0) {
      const uint32_t id_i8 = idesc_i8(kTileN, a.Bp);
      const uint32_t id_bf = idesc_bf16(kTileN, a.Bp);
      const uint32_t id_f4 = idesc_nvf4(kTileN, a.Bp);
      const uint32_t id_mx0 = idesc_mxf4(kTileN, a.Bp, 0), id_mx1 = idesc_mxf4(kTileN, a.Bp, 2);
      const int kmma = (a.M + 63) / 64;   // fp4 K = 64 MMAs of the residual
      const uint32_t lr_acc = fmt_is_f4(kFmt) ? tmem : tmem + kLrCol;
      {
        // throwaway MMA: the first tcgen05.mma of a kernel completes microseconds
        // after the rest; issued now it overlaps the first loads (the first real
        // MMA overwrites its accumulator)
        const uint64_t d0 = smem_desc_sw128(smem_u32(smem));
        if constexpr (kFmt == kFmtNvfp4)
          mma_nvf4(tmem, d0, d0, id_f4, 0u, tmem + kSfaCol, tmem + kSfbCol);
        else if constexpr (kFmt == kFmtMxfp4)
          mma_mxf4(tmem, d0, d0, id_mx0, 0u, tmem + kSfaCol, tmem + kSfbCol);
        else
          mma_i8(tmem, d0, d0, id_i8, 0u);
      }
      bool ok = true;
      for (int i = 0; i < nsteps && ok; ++i) {
        const int sa = i % a.dr, sb = sa;
        ok = mbar_wait(&full[sa], (i / a.dr) & 1, status, &abort_sh);
        if (!ok) break;
        tc_fence_after();
        const uint32_t a0 = smem_u32(ring_a + static_cast<size_t>(sa) * a.a_slot);
        const uint32_t b0 = smem_u32(ring_b + static_cast<size_t>(sb) * a.b_slot);
        if (i < nlr) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_f16(lr_acc, smem_desc_sw128(a0 + 32 * kk), smem_desc_sw128(b0 + 32 * kk), id_bf,
                    (i > 0 || kk > 0) ? 1u : 0u);
        } else {
          const int r = i - nlr;
          if constexpr (fmt_is_f4(kFmt)) {
            constexpr int kAt = sf_atoms_per_step(kFmt);
            const int k = k_lo + r;
            const int na = min(kAt, a.katoms - kAt * k);
            const uint32_t sfa_s = a0 + kATile;
            const uint32_t sfb_s = b0 + a.Bp * 128;
            // tcgen05.cp and tcgen05.mma from one thread execute in order, so
            // the scale columns can be refilled every step
            for (int kk = 0; kk < na; ++kk) {
              tmem_cp_32x128b_warpx4(tmem + kSfaCol + 4 * kk, smem_desc_plain(sfa_s + 512 * kk));
              tmem_cp_32x128b_warpx4(tmem + kSfbCol + 4 * kk, smem_desc_plain(sfb_s + 512 * kk));
            }
            if constexpr (kFmt == kFmtNvfp4) {
              for (int kk = 0; kk < na; ++kk)
                mma_nvf4(tmem, smem_desc_sw128(a0 + 32 * kk), smem_desc_sw128(b0 + 32 * kk), id_f4,
                         (i > 0 || kk > 0) ? 1u : 0u, tmem + kSfaCol + 4 * kk, tmem + kSfbCol + 4 * kk);
            } else {
              // MMA kk: atom kk / 2, scale bytes 2 (kk % 2) and up of each row's four
              const int nm = min(4, kmma - 4 * k);
              for (int kk = 0; kk < nm; ++kk)
                mma_mxf4(tmem, smem_desc_sw128(a0 + 32 * kk), smem_desc_sw128(b0 + 32 * kk), ((kk & 1) ? id_mx1 : id_mx0),
                         (i > 0 || kk > 0) ? 1u : 0u, sf_taddr(tmem + kSfaCol + 4 * (kk >> 1), kk),
                         sf_taddr(tmem + kSfbCol + 4 * (kk >> 1), kk));
            }
          } else {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_i8(tmem, smem_desc_sw128(a0 + 32 * kk), smem_desc_sw128(b0 + 32 * kk), id_i8,
                     (r > 0 || kk > 0) ? 1u : 0u);
          }
        }
        mma_commit(&empty[sa]);
      }
      if (ok) mma_commit(&tmem_full);
      if (!ok) abort_sh = 1;
      // every MMA issued so far has completed before TMEM can be released
      mma_commit(&mma_done);
      mbar_wait(&mma_done, 0, status, nullptr);
    }
  } else {
    // ------------------------------------------- widening of packed codes
    if constexpr (kFmt == kFmtInt4) {
      const int t = (warp - kWarpEpi0) * 32 + lane;   // 0..127
      bool ok = true;
      for (int r = 0; r < nres && ok; ++r) {
        const int ps = r % a.dp, i = nlr + r, as = i % a.dr;
        ok = mbar_wait_warp(&full_p[ps], (r / a.dp) & 1, status, &abort_sh);
        if (ok && i >= a.dr) ok = mbar_wait_warp(&empty[as], ((i / a.dr) - 1) & 1, status, &abort_sh);
        if (!ok) break;
        const uint8_t* src = ring_p + static_cast<size_t>(ps) * kPSlot;
        uint8_t* dst = ring_a + static_cast<size_t>(as) * a.a_slot;
#pragma unroll
        for (int it = 0; it < 4; ++it) {
          const int idx = t + 128 * it;            // 16-byte piece of the packed tile
          const int row = idx >> 2, q = idx & 3;   // row, quarter of its 64 bytes
          const uint4 v = ld_shared_v4(smem_u32(src + row * 64 + q * 16));
          uint32_t o[8];
          widen_int4(v, o);
          uint8_t* drow = dst + row * 128;
          st_shared_v4(smem_u32(drow + (((2 * q) ^ (row & 7)) << 4)), make_uint4(o[0], o[1], o[2], o[3]));
          st_shared_v4(smem_u32(drow + (((2 * q + 1) ^ (row & 7)) << 4)), make_uint4(o[4], o[5], o[6], o[7]));
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&full[as]);
          mbar_arrive(&empty_p[ps]);
        }
      }
    }
  }

  // ------------------------------------------------------------ epilogue
  // Partials of the whole tile are staged per owner in this CTA's shared memory
  // (stg[p][b][nl], p the CTA that owns weight rows [p sh, p sh + sh)), then
  // one bulk copy per owner moves each share into recv[rank] of that owner,
  // completing on the owner's recv_bar; the owner sums recv[c] (stg[rank] for
  // its own) in rank order. Both buffers reuse the operand rings, whose last
  // reads are the MMAs: staging waits for this CTA's accumulator, the copies
  // for the cluster barrier that follows every CTA's staging.
  const bool epi = warp >= kWarpEpi0;
  const int slot_words = a.B * a.sh;
  uint32_t* stg = recv_base;
  uint32_t* recv = recv_base + static_cast<size_t>(S) * slot_words;
  float alpha = 0.0f;
  if (epi) {
    const bool fin = mbar_wait_warp(&tmem_full, 0, status, &abort_sh);
    tc_fence_after();
    pdl_wait();   // the activation scale comes from the activation pass
    alpha = skinny_alpha<kFmt, kOut>(a);
    if (fin) {
      const int q = warp & 3;
      const int nloc = q * 32 + lane;                 // weight row within the tile
      const int p = nloc / a.sh, nl = nloc - p * a.sh;
      // shared-window stores (the pointer's origin is not visible to the compiler)
      const uint32_t dst_s = smem_u32(stg + static_cast<size_t>(p) * slot_words + nl);
      const uint32_t lane_addr = tmem + (static_cast<uint32_t>(q * 32) << 16);
      const bool lr_here = !fmt_is_f4(kFmt) && kOut != kOutI32 && nlr > 0;
      for (int c0 = 0; c0 < a.B; c0 += 32) {
        uint32_t acc[32], up[32];
        __syncwarp();
        if (c0 + 16 < a.Bp) {   // 32 columns are allocated to the accumulator
          tmem_ld_32x32b_x32(lane_addr + c0, acc);
          if (lr_here) tmem_ld_32x32b_x32(lane_addr + kLrCol + c0, up);
        } else {
          tmem_ld_32x32b_x16(lane_addr + c0, *reinterpret_cast<uint32_t(*)[16]>(acc));
          if (lr_here) tmem_ld_32x32b_x16(lane_addr + kLrCol + c0, *reinterpret_cast<uint32_t(*)[16]>(up));
        }
        tmem_ld_wait_regs(acc);
        if (lr_here) tmem_ld_wait_regs(up);
        const int cnt = min(32, a.B - c0);
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          if (j >= cnt) break;
          uint32_t v = acc[j];
          if (!fmt_is_f4(kFmt) && kOut != kOutI32) {
            float f = alpha * static_cast<float>(static_cast<int32_t>(acc[j]));
            if (lr_here) f += __uint_as_float(up[j]);
            v = __float_as_uint(f);
          }
          st_shared_u32(dst_s + static_cast<uint32_t>((c0 + j) * a.sh) * 4u, v);
        }
      }
    }
    fence_proxy_async_smem();   // the staged partials are read by the bulk copies
  }
  tc_fence_before();
  __syncwarp();
  cluster_sync();
  if (threadIdx.x == kWarpEpi0 * 32) {
    const uint32_t bytes = static_cast<uint32_t>(slot_words) * 4u;
    for (int p = 0; p < S; ++p) {
      if (p == rank) continue;
      bulk_copy_to_cluster(mapa_shared(smem_u32(recv + static_cast<size_t>(rank) * slot_words), p),
                           smem_u32(stg + static_cast<size_t>(p) * slot_words), bytes,
                           mapa_shared(smem_u32(&recv_bar), p));
    }
  }
  const bool got = mbar_wait(&recv_bar, 0, status, &abort_sh);

  // ------------------------------------- sum of the partials, bias, store
  {
    const int cnt = min(a.sh, kTileN - rank * a.sh);      // weight rows this CTA owns
    const int nq = cnt / 4;
    const int nbase = n0 + rank * a.sh;
    pdl_wait();   // returns at once: the epilogue warps waited before the barriers
    const float alpha_f4 = fmt_is_f4(kFmt) ? skinny_alpha<kFmt, kOut>(a) : 1.0f;
    for (int it = threadIdx.x; it < a.B * nq; it += kThreads) {
      const int b = it / nq, nl = (it - b * nq) * 4;
      const int n = nbase + nl;
      if (n >= a.N || !got) continue;
      if constexpr (kOut == kOutI32) {
        int4 s = make_int4(0, 0, 0, 0);
        for (int c = 0; c < S; ++c) {
          const uint32_t* src = (c == rank ? stg + static_cast<size_t>(c) * slot_words : recv + static_cast<size_t>(c) * slot_words);
          const uint4 v = ld_shared_v4(smem_u32(src + b * a.sh + nl));
          s.x += static_cast<int>(v.x); s.y += static_cast<int>(v.y); s.z += static_cast<int>(v.z); s.w += static_cast<int>(v.w);
        }
        int32_t* dst = static_cast<int32_t*>(a.y) + static_cast<int64_t>(b) * a.ldy + n;
        if (a.vec_ok) {
          *reinterpret_cast<int4*>(dst) = s;
        } else {
          dst[0] = s.x; dst[1] = s.y; dst[2] = s.z; dst[3] = s.w;
        }
      } else {
        float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int c = 0; c < S; ++c) {
          const uint32_t* src = (c == rank ? stg + static_cast<size_t>(c) * slot_words : recv + static_cast<size_t>(c) * slot_words);
          const uint4 v = ld_shared_v4(smem_u32(src + b * a.sh + nl));
          s.x += __uint_as_float(v.x); s.y += __uint_as_float(v.y); s.z += __uint_as_float(v.z); s.w += __uint_as_float(v.w);
        }
        float o[4] = {s.x, s.y, s.z, s.w};
        if (fmt_is_f4(kFmt)) {
#pragma unroll
          for (int j = 0; j < 4; ++j) o[j] *= alpha_f4;
        }
        if (a.bias != nullptr) {
          const uint2 bb = *reinterpret_cast<const uint2*>(a.bias + n);
          o[0] += __uint_as_float(bb.x << 16);
          o[1] += __uint_as_float(bb.x & 0xFFFF0000u);
          o[2] += __uint_as_float(bb.y << 16);
          o[3] += __uint_as_float(bb.y & 0xFFFF0000u);
        }
        if constexpr (kOut == kOutF32) {
          float* dst = static_cast<float*>(a.y) + static_cast<int64_t>(b) * a.ldy + n;
          if (a.vec_ok) {
            *reinterpret_cast<float4*>(dst) = make_float4(o[0], o[1], o[2], o[3]);
          } else {
            dst[0] = o[0]; dst[1] = o[1]; dst[2] = o[2]; dst[3] = o[3];
          }
        } else {
          uint16_t* dst = static_cast<uint16_t*>(a.y) + static_cast<int64_t>(b) * a.ldy + n;
          const uint32_t p0 = pack_bf16x2(o[0], o[1]), p1 = pack_bf16x2(o[2], o[3]);
          if (a.vec_ok) {
            *reinterpret_cast<uint2*>(dst) = make_uint2(p0, p1);
          } else {
            dst[0] = static_cast<uint16_t>(p0 & 0xFFFFu); dst[1] = static_cast<uint16_t>(p0 >> 16);
            dst[2] = static_cast<uint16_t>(p1 & 0xFFFFu); dst[3] = static_cast<uint16_t>(p1 >> 16);
          }
        }
      }
    }
  }

  // every owner has received its shares (so every copy out of this CTA's
  // shared memory is done) before any CTA of the cluster exits
  __syncwarp();
  cluster_sync();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ------------------------------------------------------------------ GEMV
// Batches of at most kGemvMaxB rows with INT weights. The tensor-core path
// above issues one MMA per 32 bytes of K per 128 weight rows whatever the
// batch, and for one or two rows that issue rate, not HBM, sets its time; here
// the int32 dot products run on the integer units (dp4a) instead. (dp4a runs
// at a fraction of the FP32 rate on this part: measured per decode step, one
// row 13.1 us here against 15.4 us on the tensor cores, two rows 14.5 us, four
// 17.5 us, eight 24.1 us.) Each CTA
// owns rows_per_cta consecutive weight rows: it copies them (and their lu rows)
// into shared memory before griddepcontrol.wait, so the whole weight stream
// overlaps the activation pass; after the wait it copies the activation codes
// and down hi | lo, and each warp forms the B dot products of its rows (lanes
// split K), then Y = alpha acc + down . lu + bias.
constexpr int kGemvMaxB = 2;   // past two rows the dp4a rate makes the tensor-core path faster
constexpr int kGemvThreads = 256;
constexpr int kGemvWarps = kGemvThreads / 32;
constexpr size_t kGemvSmemMax = 200 * 1024;

struct GemvArgs {
  int B, N, M, rp, rows_per_cta, row_bytes;
  const uint8_t* w;             // packed [N, M/2] or int8 [N, M]
  const int8_t* act;            // [B, M]
  const __nv_bfloat16* down2;   // [B, 2 rp]
  const __nv_bfloat16* lu;      // [N, 2 rp]
  const float* s_x;
  const float* s_w;
  const __nv_bfloat16* bias;
  void* y;
  int64_t ldy;
};

__host__ __device__ constexpr size_t gemv_smem(int rows, int row_bytes, int B, int M, int rp) {
  return static_cast<size_t>(rows) * row_bytes + static_cast<size_t>(rows) * 4 * rp +
         static_cast<size_t>(B) * M + static_cast<size_t>(B) * 4 * rp + 64;
}

template <bool kPacked, int kOut>
__global__ void __launch_bounds__(kGemvThreads, 1) gemv_kernel(const GemvArgs g) {
  extern __shared__ __align__(16) uint8_t gsm[];
  // a chained linear's activation pass queued after this kernel may start its
  // weight-side setup now (it reads this kernel's output only after griddepcontrol.wait)
  pdl_trigger();
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n0 = blockIdx.x * g.rows_per_cta;
  const int rows = min(g.rows_per_cta, g.N - n0);
  const int lrw = 2 * g.rp * 2;   // bytes of a lu / down2 row
  uint8_t* ws = gsm;                                                  // [rows_per_cta][row_bytes]
  uint8_t* lus = ws + static_cast<size_t>(g.rows_per_cta) * g.row_bytes;       // [rows_per_cta][4 rp]
  uint8_t* acts = lus + static_cast<size_t>(g.rows_per_cta) * lrw;              // [B][M]
  uint8_t* dns = acts + static_cast<size_t>(g.B) * g.M;                         // [B][4 rp]
  // weight side, independent of the activation pass
  {
    const int per_row = g.row_bytes / 16, total = rows * per_row;
    for (int i = tid; i < total; i += kGemvThreads) {
      const int r = i / per_row, c = i - r * per_row;
      cp_async16(ws + static_cast<size_t>(r) * g.row_bytes + 16 * c,
                 g.w + static_cast<int64_t>(n0 + r) * g.row_bytes + 16 * c, 16);
    }
    const int lper = lrw / 16, ltot = (kOut == kOutI32 ? 0 : rows * lper);
    for (int i = tid; i < ltot; i += kGemvThreads) {
      const int r = i / lper, c = i - r * lper;
      cp_async16(lus + r * lrw + 16 * c, reinterpret_cast<const uint8_t*>(g.lu) + static_cast<int64_t>(n0 + r) * lrw + 16 * c,
                 16);
    }
    cp_async_commit();
  }
  pdl_wait();   // codes, down and s_x come from the activation pass
  {
    const int per_row = g.M / 16, total = g.B * per_row;
    for (int i = tid; i < total; i += kGemvThreads)
      cp_async16(acts + 16 * i, reinterpret_cast<const uint8_t*>(g.act) + 16 * i, 16);
    const int dtot = (kOut == kOutI32 ? 0 : g.B * lrw / 16);
    for (int i = tid; i < dtot; i += kGemvThreads)
      cp_async16(dns + 16 * i, reinterpret_cast<const uint8_t*>(g.down2) + 16 * i, 16);
    cp_async_commit();
  }
  const float alpha = kOut == kOutI32 ? 0.0f : __ldg(g.s_x) * __ldg(g.s_w);
  cp_async_wait<0>();
  __syncthreads();

  // one 16-byte weight chunk per lane and step (32 packed codes, K = 32, or 16
  // int8 codes) for kRB rows at once, so each activation chunk read from shared
  // memory serves kRB rows
  constexpr int kK = kPacked ? 32 : 16;
  constexpr int kRB = 4;
  const int nchunks = g.row_bytes / 16;
  for (int r0 = warp * kRB; r0 < rows; r0 += kGemvWarps * kRB) {
    int acc[kRB][kGemvMaxB];
#pragma unroll
    for (int i = 0; i < kRB; ++i)
#pragma unroll
      for (int b = 0; b < kGemvMaxB; ++b) acc[i][b] = 0;
    for (int j = lane; j < nchunks; j += 32) {
      uint32_t w8[kRB][kK / 4];
#pragma unroll
      for (int i = 0; i < kRB; ++i) {
        const int r = min(r0 + i, rows - 1);   // rows past the end repeat the last (not stored)
        const uint4 wv = ld_shared_v4(smem_u32(ws + static_cast<size_t>(r) * g.row_bytes + 16 * j));
        if constexpr (kPacked) {
          widen_int4(wv, *reinterpret_cast<uint32_t(*)[8]>(w8[i]));
        } else {
          w8[i][0] = wv.x; w8[i][1] = wv.y; w8[i][2] = wv.z; w8[i][3] = wv.w;
        }
      }
#pragma unroll
      for (int b = 0; b < kGemvMaxB; ++b) {
        if (b >= g.B) break;
        const uint32_t abase = smem_u32(acts + static_cast<size_t>(b) * g.M + kK * j);
#pragma unroll
        for (int h = 0; h < kK / 16; ++h) {
          const uint4 av = ld_shared_v4(abase + 16 * h);
#pragma unroll
          for (int i = 0; i < kRB; ++i) {
            acc[i][b] = __dp4a(static_cast<int>(w8[i][4 * h + 0]), static_cast<int>(av.x), acc[i][b]);
            acc[i][b] = __dp4a(static_cast<int>(w8[i][4 * h + 1]), static_cast<int>(av.y), acc[i][b]);
            acc[i][b] = __dp4a(static_cast<int>(w8[i][4 * h + 2]), static_cast<int>(av.z), acc[i][b]);
            acc[i][b] = __dp4a(static_cast<int>(w8[i][4 * h + 3]), static_cast<int>(av.w), acc[i][b]);
          }
        }
      }
    }
#pragma unroll
    for (int i = 0; i < kRB; ++i) {
      const int r = r0 + i;
      if (r >= rows) break;
      // every lane ends up with every batch row's sum; lane b keeps row b's
      int mine = 0;
#pragma unroll
      for (int b = 0; b < kGemvMaxB; ++b) {
        if (b >= g.B) break;
        int v = acc[i][b];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == b) mine = v;
      }
      const int n = n0 + r;
      if (lane < g.B) {
        const int b = lane;
        if constexpr (kOut == kOutI32) {
          static_cast<int32_t*>(g.y)[static_cast<int64_t>(b) * g.ldy + n] = mine;
        } else {
          // the up-projection: down hi | lo against lu (both halves of lu hold L2)
          float up = 0.0f;
          const __nv_bfloat16* dr = reinterpret_cast<const __nv_bfloat16*>(dns + b * lrw);
          const __nv_bfloat16* lr = reinterpret_cast<const __nv_bfloat16*>(lus + r * lrw);
          for (int q = 0; q < 2 * g.rp; ++q) up = fmaf(__bfloat162float(dr[q]), __bfloat162float(lr[q]), up);
          float v = alpha * static_cast<float>(mine) + up;
          if (g.bias != nullptr) v += __bfloat162float(g.bias[n]);
          if constexpr (kOut == kOutF32)
            static_cast<float*>(g.y)[static_cast<int64_t>(b) * g.ldy + n] = v;
          else
            static_cast<__nv_bfloat16*>(g.y)[static_cast<int64_t>(b) * g.ldy + n] = __float2bfloat16_rn(v);
        }
      }
    }
  }
}

template <bool kPacked, int kOut>
cudaError_t launch_gemv_one(const GemvArgs& g, int grid, size_t smem, bool pdl, cudaStream_t st) {
  auto kern = gemv_kernel<kPacked, kOut>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (err != cudaSuccess) return err;
  err = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
  if (err != cudaSuccess) return err;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kGemvThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, g);
}

// The GEMV path when it applies (INT weights, B <= kGemvMaxB, everything in
// shared memory); false (nothing launched) otherwise.
bool launch_gemv(int out, const GemmArgs& ga, const void* act_codes, const void* down2, const svdq_weight* w,
                 bool pdl, cudaStream_t stream, cudaError_t* err) {
  const int64_t M = w->M, N = w->N, B = ga.B;
  if (B < 1 || B > kGemvMaxB) return false;
  const bool packed = w->fmt.bits <= 4 && w->codes4 != nullptr;
  const int row_bytes = static_cast<int>(packed ? M / 2 : M);
  const int rp = (out != kOutI32 && down2 != nullptr) ? w->rank_pad : 0;
  const int rows = static_cast<int>(round_up(ceil_div(N, num_sms()), kGemvWarps));
  const size_t smem = gemv_smem(rows, row_bytes, static_cast<int>(B), static_cast<int>(M), rp);
  if (smem > kGemvSmemMax) return false;
  for (const void* q : {static_cast<const void*>(packed ? w->codes4 : w->codes), act_codes, down2,
                        static_cast<const void*>(w->lu)})
    if (q != nullptr && (reinterpret_cast<uintptr_t>(q) & 15) != 0) return false;
  GemvArgs g{};
  g.B = static_cast<int>(B);
  g.N = static_cast<int>(N);
  g.M = static_cast<int>(M);
  g.rp = rp;
  g.rows_per_cta = rows;
  g.row_bytes = row_bytes;
  g.w = static_cast<const uint8_t*>(packed ? w->codes4 : w->codes);
  g.act = static_cast<const int8_t*>(act_codes);
  g.down2 = static_cast<const __nv_bfloat16*>(down2);
  g.lu = static_cast<const __nv_bfloat16*>(w->lu);
  g.s_x = ga.s_x;
  g.s_w = ga.s_w;
  g.bias = ga.bias;
  g.y = ga.y;
  g.ldy = ga.ldy;
  const int grid = static_cast<int>(ceil_div(N, rows));
#define SVDQ_GEMV(P, O) *err = launch_gemv_one<P, O>(g, grid, smem, pdl, stream)
  if (packed) {
    if (out == kOutI32) SVDQ_GEMV(true, kOutI32);
    else if (out == kOutF32) SVDQ_GEMV(true, kOutF32);
    else SVDQ_GEMV(true, kOutBF16);
  } else {
    if (out == kOutI32) SVDQ_GEMV(false, kOutI32);
    else if (out == kOutF32) SVDQ_GEMV(false, kOutF32);
    else SVDQ_GEMV(false, kOutBF16);
  }
#undef SVDQ_GEMV
  return true;
}

struct SkinnyPlan {
  int S, sh, dr, dp, a_slot, b_slot;
  size_t smem;
};

SkinnyPlan plan_skinny(int kFmt, int Bp, int64_t N, int kst, int lr_boxes) {
  SkinnyPlan p{};
  const int64_t tiles = ceil_div(N, kTileN);
  const int sms = num_sms();
  int S = 1;
  for (int s = std::min(8, kst); s >= 1; --s)
    if (tiles * s <= sms) {
      S = s;
      break;
    }
  p.S = S;
  p.sh = static_cast<int>(round_up(ceil_div(kTileN, S), 4));
  p.a_slot = kATile + sf_atoms_per_step(kFmt) * 512;
  p.b_slot = Bp * 128 + sf_atoms_per_step(kFmt) * 512;
  const int nres_max = static_cast<int>(ceil_div(kst, S));
  const int nsteps_max = nres_max + static_cast<int>(ceil_div(lr_boxes, S));
  p.dp = kFmt == kFmtInt4 ? std::min(nres_max, kMaxRing) : 0;
  p.dr = std::min(nsteps_max, kMaxRing);
  auto total = [&]() {
    return static_cast<size_t>(p.dr) * (p.a_slot + p.b_slot) + static_cast<size_t>(p.dp) * kPSlot;
  };
  while (total() > kSmemBudget) {
    if (p.dp > 4) --p.dp;
    else if (p.dr > 2) --p.dr;
    else if (p.dp > 2) --p.dp;
    else break;
  }
  const size_t recv = 2 * static_cast<size_t>(S) * Bp * p.sh * 4;   // staged and received partials
  // more than half an SM's shared memory: one CTA of this kernel per SM, so
  // the TMEM allocation never waits on another cluster's CTA
  p.smem = std::max({total(), recv, kMinSmem}) + 1024;
  return p;
}

template <int kFmt, int kOut>
cudaError_t launch_one(const CUtensorMap& w, const CUtensorMap& x, const CUtensorMap& lu, const CUtensorMap& dn,
                       const SkinnyArgs& args, int tiles, size_t smem, bool pdl, cudaStream_t st) {
  auto kern = skinny_kernel<kFmt, kOut>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (err != cudaSuccess) return err;
  // same (largest) shared-memory configuration as the activation pass, so CTAs
  // of the two kernels can share an SM under a dependent launch
  err = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
  if (err != cudaSuccess) return err;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(args.S), static_cast<unsigned>(tiles));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(args.S);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, kern, w, x, lu, dn, args);
}

}  // namespace

// Host side: tensor maps and launch. kind: GemmKind; out: GemmOut.
bool launch_gemm_skinny(int kind, int out, const GemmArgs& g, const void* act_codes, const uint8_t* act_sf,
                        const void* down2, const svdq_weight* w, bool pdl, cudaStream_t stream,
                        cudaError_t* err) {
  *err = cudaSuccess;
  const int64_t M = w->M, N = w->N, B = g.B;
  if (B <= 0 || B > 128) return false;
  if (kind == kKindInt && launch_gemv(out, g, act_codes, down2, w, pdl, stream, err)) return true;
  const int Bp = static_cast<int>(std::max<int64_t>(16, round_up(B, 16)));
  const bool packed = kind == kKindInt && w->fmt.bits <= 4 && w->codes4 != nullptr;
  const int fmt = kind == kKindNvfp4 ? kFmtNvfp4 : kind == kKindMxfp4 ? kFmtMxfp4 : (packed ? kFmtInt4 : kFmtInt8);
  const int kst = static_cast<int>(kind != kKindInt ? ceil_div(M, 256) : ceil_div(M, 128));
  const int rp = w->rank_pad;
  const bool has_lr = out != kOutI32 && rp > 0 && down2 != nullptr;
  const int lr_boxes = has_lr ? static_cast<int>(ceil_div(2 * rp, 64)) : 0;
  const SkinnyPlan p = plan_skinny(fmt, Bp, N, kst, lr_boxes);

  CUtensorMap tm_w, tm_x, tm_lu, tm_dn;
  bool ok;
  if (fmt == kFmtInt4)
    ok = make_tmap_2d(&tm_w, w->codes4, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, M / 2, N, M / 2, 64, kTileN, false);
  else if (fmt_is_f4(fmt))
    ok = make_tmap_2d(&tm_w, w->codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, M / 2, N, M / 2, 128, kTileN, true);
  else
    ok = make_tmap_2d(&tm_w, w->codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, M, N, M, 128, kTileN, true);
  const int64_t xrow = kind != kKindInt ? M / 2 : M;
  ok = ok && make_tmap_2d(&tm_x, act_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, xrow, B, xrow, 128, Bp, true);
  if (ok && has_lr) {
    ok = make_tmap_2d(&tm_lu, w->lu, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, 2 * rp, N, 2 * rp, 64, kTileN, true) &&
         make_tmap_2d(&tm_dn, down2, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, 2 * rp, B, 2 * rp, 64, Bp, true);
  } else {
    tm_lu = tm_w;
    tm_dn = tm_x;
  }
  if (!ok) return false;

  SkinnyArgs a{};
  a.B = static_cast<int>(B);
  a.Bp = Bp;
  a.N = static_cast<int>(N);
  a.M = static_cast<int>(M);
  a.S = p.S;
  a.kst = kst;
  a.lr_boxes = lr_boxes;
  a.sh = p.sh;
  a.dr = p.dr;
  a.dp = p.dp;
  a.a_slot = p.a_slot;
  a.b_slot = p.b_slot;
  a.katoms = g.katoms;
  a.s_x = g.s_x;
  a.s_w = g.s_w;
  a.bias = g.bias;
  a.y = g.y;
  a.ldy = g.ldy;
  a.vec_ok = g.vec_ok;
  a.sfw = static_cast<const uint8_t*>(w->sf);
  a.sfx = act_sf;
  a.status = g.status;
  const int tiles = static_cast<int>(ceil_div(N, kTileN));
#define SVDQ_SKINNY(F, O) *err = launch_one<F, O>(tm_w, tm_x, tm_lu, tm_dn, a, tiles, p.smem, pdl, stream)
  if (out == kOutI32) {
    if (fmt == kFmtInt4) SVDQ_SKINNY(kFmtInt4, kOutI32);
    else if (fmt == kFmtInt8) SVDQ_SKINNY(kFmtInt8, kOutI32);
    else return false;
  } else if (out == kOutF32) {
    if (fmt == kFmtInt4) SVDQ_SKINNY(kFmtInt4, kOutF32);
    else if (fmt == kFmtInt8) SVDQ_SKINNY(kFmtInt8, kOutF32);
    else if (fmt == kFmtMxfp4) SVDQ_SKINNY(kFmtMxfp4, kOutF32);
    else SVDQ_SKINNY(kFmtNvfp4, kOutF32);
  } else {
    if (fmt == kFmtInt4) SVDQ_SKINNY(kFmtInt4, kOutBF16);
    else if (fmt == kFmtInt8) SVDQ_SKINNY(kFmtInt8, kOutBF16);
    else if (fmt == kFmtMxfp4) SVDQ_SKINNY(kFmtMxfp4, kOutBF16);
    else SVDQ_SKINNY(kFmtNvfp4, kOutBF16);
  }
#undef SVDQ_SKINNY
  return true;
}

}  // namespace svdq
