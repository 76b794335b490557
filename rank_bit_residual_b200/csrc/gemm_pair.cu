// gemm_pair.cu - the residual GEMM on CTA pairs (tcgen05 cta_group::2).
//
// Same operator as gemm.cu ("SVDQuant Smoothing, Low-rank and Residual
// Quantization", Formula item 3; step 3 of "flashinfer.gemm.svdquant_linear"):
// Y = alpha * Q(X_hat) Q(R) + down . lu^T [+ bias], INT (kind::i8), NVFP4
// (kind::mxf4nvf4 with ue4m3 scales per 16 elements) or MXFP4 (kind::mxf4 with
// E8M0 scales per 32 elements).
//
// A cluster of two CTAs computes one 256 x 256 output tile: CTA r holds rows
// [128 r, 128 r + 128) of the A tile and rows [128 r, 128 r + 128) of the B
// tile in its shared memory, and its TMEM receives its 128 rows of the
// accumulator for all 256 columns. One thread of the even CTA issues every MMA
// for the pair. Each CTA loads its own halves by TMA and signals the even CTA's
// barrier; the MMA commits signal the barriers of both CTAs; each CTA's
// epilogue drains its own TMEM and reports back to the even CTA. Per SM this
// halves the B-operand traffic of the one-CTA kernel and, for NVFP4, the scale
// copies per multiply-accumulate.
//
// Warps: 0 TMA producer, 1 MMA (even CTA), 2-9 epilogue (two warps per TMEM
// lane quarter, each for 128 of the 256 columns). The epilogue runs in two
// passes so that the global stores overlap the next tile's MMAs:
//   pass 1  alpha * acc (+ up) + bias, rounded to the output type, written back
//           into TMEM columns the next tile's residual MMAs do not touch; then
//           the accumulator columns are released (acc_empty);
//   pass 2  those columns -> Y; then (INT) the low-rank columns are released
//           (lr_empty).
// Each tile runs its residual K steps first and its low-rank K steps last, so
// the next tile's MMAs need the low-rank columns only at the end of its chain.
// TMEM columns (512):
//   INT    [0, 256) int32 residual | [256, 512) fp32 up-projection, which
//          pass 1 overwrites in place with the combined result
//   fp4    [0, 256) fp32 (both branches) | [256, 304) block scales |
//          [384, 512) bf16 result of pass 1 (fp32 output: one direct pass)
// fp4: each CTA's TMEM holds the scales of its 128 A rows (4 columns per
// 128 x 4 scale atom) and of all 256 B rows (8 columns), copied from its own
// shared memory by the pair-wide tcgen05.cp the even CTA issues. An atom holds
// four scales per row: one K = 64 MMA's worth for NVFP4 (16-element blocks),
// two MMAs' for MXFP4 (32-element blocks; the MMA's scale-factor id picks the
// byte pair), so a 256-element stage copies 4 atoms per row tile for NVFP4 and
// 2 for MXFP4.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "gemm_common.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace svdq {

namespace {

constexpr int kEpiWarps = 8;
constexpr int kPairThreads = 64 + 32 * kEpiWarps;
constexpr int kHalf = 128;                        // rows of A and of B per CTA
constexpr int kTileN = 256;
constexpr int kABytes = kHalf * 128;
constexpr int kBBytes = kHalf * 128;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSfaCol = 256;
constexpr uint32_t kSfbCol = 272;
constexpr uint32_t kNvOutCol = 384;               // fp4 bf16 pass-1 result

template <int kKind>
struct PairCfg {
  static constexpr bool kF4 = kKind != kKindInt;
  // INT: two 128-byte K blocks per stage (8 MMAs per barrier wait and commit)
  static constexpr int kKb = kF4 ? 1 : 2;
  // scale atoms per 128-row tile and stage (256 elements of K)
  static constexpr int kSfAtoms = kKind == kKindNvfp4 ? 4 : (kKind == kKindMxfp4 ? 2 : 0);
  static constexpr int kSfaBytes = kSfAtoms * 512;       // this CTA's A rows
  static constexpr int kSfbBytes = 2 * kSfAtoms * 512;   // both B row tiles
  static constexpr int kStages = kKind == kKindNvfp4 ? 5 : (kKind == kKindMxfp4 ? 6 : 3);
  static constexpr int kStageBytes = kKb * (kABytes + kBBytes) + kSfaBytes + kSfbBytes;
};

// Whether the epilogue's stores overlap the next tile's MMAs.
template <int kKind, int kOut>
struct TwoPass {
  static constexpr bool value = kOut == kOutBF16 || (kKind == kKindInt && kOut == kOutF32);
};

__device__ __forceinline__ unsigned ld_acquire_gpu_u32(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// One round's work of a pair: tile t, residual K steps [j0, j1); role 0 = the
// whole tile, 1 = owner of a split tile (slice 0: adds the other slices'
// partials), 2 = a later slice (writes its partial); q = index of the split tile,
// sl = slice. Only roles 0 and 1 run the low-rank steps and write Y.
struct PairItem {
  int t, j0, j1, role, q, sl;
};

template <int kKind, int kOut>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kPairThreads, 1)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                     const __grid_constant__ CUtensorMap tm_da, const __grid_constant__ CUtensorMap tm_lu,
                     const __grid_constant__ CUtensorMap tm_sfa, const __grid_constant__ CUtensorMap tm_sfb,
                     const GemmArgs args) {
  constexpr int kStages = PairCfg<kKind>::kStages;
  constexpr int kStageBytes = PairCfg<kKind>::kStageBytes;
  constexpr bool kF4 = PairCfg<kKind>::kF4;
  constexpr int kSfAtoms = PairCfg<kKind>::kSfAtoms;
  constexpr int kSfaBytes = PairCfg<kKind>::kSfaBytes;
  constexpr int kSfbBytes = PairCfg<kKind>::kSfbBytes;
  constexpr bool kTwoPass = TwoPass<kKind, kOut>::value;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[kStages];
  __shared__ __align__(8) uint64_t empty_bar[kStages];
  __shared__ __align__(8) uint64_t tmem_full_bar;
  __shared__ __align__(8) uint64_t acc_empty_bar;
  __shared__ __align__(8) uint64_t lr_empty_bar;
  __shared__ __align__(8) uint64_t exit_bar;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  // a chained linear's activation pass queued after this kernel may start its
  // weight-side setup now (it reads this kernel's output only after griddepcontrol.wait)
  pdl_trigger();
  const int B = args.B, N = args.N, M = args.M, lr_steps = args.lr_steps;
  unsigned* status = args.status;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair = blockIdx.x >> 1;
  const int npairs = gridDim.x >> 1;
  const int tiles_m = (B + 2 * kHalf - 1) / (2 * kHalf);
  const int tiles_n = (N + kTileN - 1) / kTileN;
  const int total = tiles_m * tiles_n;
  constexpr int kKb = PairCfg<kKind>::kKb;
  constexpr int kStageK = kF4 ? 256 : 128 * kKb;   // K elements per stage
  const int ksteps = (M + kStageK - 1) / kStageK;
  // Work items of this pair, one per round: the tiles pair, pair + npairs, ...
  // With a split (nsplit > 1) the tiles of the last, partial round are cut
  // along K into nsplit slices run by different pairs: slice 0 (the owner)
  // also runs the low-rank steps and, in its epilogue, adds the other slices'
  // raw partial accumulators (written to the workspace) in slice order.
  const int rounds_full = total / npairs, trem = total - rounds_full * npairs;
  const int nrounds = rounds_full + (trem > 0 ? 1 : 0);
  const int nsplit = args.nsplit;
  auto item = [&](int r, PairItem& it) -> bool {
    it.j0 = 0;
    it.j1 = ksteps;
    it.role = 0;
    it.q = 0;
    it.sl = 0;
    if (r < rounds_full) {
      it.t = pair + r * npairs;
      return true;
    }
    if (r >= nrounds) return false;
    if (nsplit <= 1) {
      it.t = rounds_full * npairs + pair;
      return pair < trem;
    }
    if (pair >= trem * nsplit) return false;
    it.q = pair % trem;
    it.sl = pair / trem;
    it.t = rounds_full * npairs + it.q;
    it.j0 = (ksteps * it.sl) / nsplit;
    it.j1 = (ksteps * (it.sl + 1)) / nsplit;
    it.role = it.sl == 0 ? 1 : 2;
    return true;
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    mbar_init(&tmem_full_bar, 1);
    mbar_init(&acc_empty_bar, 2 * kEpiWarps);   // the epilogue warps of both CTAs
    mbar_init(&lr_empty_bar, 2 * kEpiWarps);
    mbar_init(&exit_bar, 1);                    // the peer's arrival at teardown
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
    tmem_alloc_pair(&tmem_base_sh, kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();  // both CTAs: barriers initialised, TMEM allocated
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      PairItem wi;
      for (int r = 0; ok && item(r, wi); ++r) {
        const int t = wi.t;
        const int m0 = (t % tiles_m) * 2 * kHalf + static_cast<int>(rank) * kHalf;
        const int nt = (t / tiles_m) * kTileN;
        const int n0 = nt + static_cast<int>(rank) * kHalf;
        const int nres = wi.j1 - wi.j0;
        const int nsteps_it = nres + (wi.role != 2 ? lr_steps : 0);
        for (int jj = 0; jj < nsteps_it && ok; ++jj, ++it) {
          const int j = wi.j0 + jj;   // residual K step
          const int s = it % kStages;
          const uint32_t ph = (it / kStages) & 1;
          ok = mbar_wait(&empty_bar[s], ph ^ 1, status, &abort_sh);
          if (!ok) break;
          uint8_t* st = smem + s * kStageBytes;
          const uint32_t fb = mapa_shared(smem_u32(&full_bar[s]), 0);
          if (jj >= nres) {
            const int l = jj - nres;
            if (rank == 0) mbar_arrive_expect_tx(&full_bar[s], 2 * (kABytes + kBBytes));
            tma_load_2d_pair(st, &tm_da, fb, 64 * l, m0);
            tma_load_2d_pair(st + kABytes, &tm_lu, fb, 64 * l, n0);
          } else if constexpr (kF4) {
            if (rank == 0)
              mbar_arrive_expect_tx(&full_bar[s], 2 * (kABytes + kBBytes + kSfaBytes + kSfbBytes));
            tma_load_2d_pair(st, &tm_a, fb, 128 * j, m0);
            tma_load_2d_pair(st + kABytes, &tm_b, fb, 128 * j, n0);
            // scale atoms: rows of 256 bytes, two rows per 512-byte atom
            uint8_t* sfa_s = st + kABytes + kBBytes;
            uint8_t* sfb_s = sfa_s + kSfaBytes;
            const int a0 = kSfAtoms * j;
            tma_load_2d_pair(sfa_s, &tm_sfa, fb, 0, 2 * ((m0 / 128) * args.katoms + a0));
            for (int rt = 0; rt < 2; ++rt)
              tma_load_2d_pair(sfb_s + rt * kSfaBytes, &tm_sfb, fb, 0, 2 * ((nt / 128 + rt) * args.katoms + a0));
          } else {
            // A blocks then B blocks, 128 bytes of K each
            if (rank == 0) mbar_arrive_expect_tx(&full_bar[s], 2 * kKb * (kABytes + kBBytes));
            for (int kb = 0; kb < kKb; ++kb) {
              tma_load_2d_pair(st + kb * kABytes, &tm_a, fb, kStageK * j + 128 * kb, m0);
              tma_load_2d_pair(st + kKb * kABytes + kb * kBBytes, &tm_b, fb, kStageK * j + 128 * kb, n0);
            }
          }
        }
      }
      // wait for the MMA's release of the last stages, so no commit arrival
      // is still on its way to this CTA's barriers when it exits
      if (ok) {
        const uint32_t first = it > static_cast<uint32_t>(kStages) ? it - kStages : 0u;
        for (uint32_t i = first; i < it; ++i)
          mbar_wait(&empty_bar[i % kStages], (i / kStages) & 1, status, nullptr);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------- MMA (even CTA only)
    if (lane == 0 && rank == 0) {
      const uint32_t id_i8 = idesc_i8(2 * kHalf, kTileN);
      const uint32_t id_bf = idesc_bf16(2 * kHalf, kTileN);
      const uint32_t id_f4 = idesc_nvf4(2 * kHalf, kTileN);
      const uint32_t id_mx0 = idesc_mxf4(2 * kHalf, kTileN, 0), id_mx1 = idesc_mxf4(2 * kHalf, kTileN, 2);
      const int kmma = (M + 63) / 64;   // fp4 K = 64 MMAs of the residual
      const uint32_t lr_acc = kF4 ? tmem : tmem + 256;
      {
        // throwaway MMA: the first tcgen05.mma of a kernel takes microseconds
        // longer than the rest; issued now, that start-up overlaps the first
        // loads (the first real MMA of the tile overwrites the accumulator)
        const uint64_t d0 = smem_desc_sw128(smem_u32(smem));
        if constexpr (kKind == kKindNvfp4)
          mma_nvf4_pair(tmem, d0, d0, id_f4, 0u, tmem + kSfaCol, tmem + kSfbCol);
        else if constexpr (kKind == kKindMxfp4)
          mma_mxf4_pair(tmem, d0, d0, id_mx0, 0u, tmem + kSfaCol, tmem + kSfbCol);
        else
          mma_i8_pair(tmem, d0, d0, id_i8, 0u);
      }
      uint32_t it = 0, lt = 0;
      bool ok = true;
      PairItem wi;
      for (int r = 0; ok && item(r, wi); ++r, ++lt) {
        ok = mbar_wait(&acc_empty_bar, (lt & 1) ^ 1, status, &abort_sh);
        if (!ok) break;
        tc_fence_after();
        const int nres = wi.j1 - wi.j0;
        const bool lr_here = wi.role != 2 && lr_steps > 0;
        const int nsteps_it = nres + (lr_here ? lr_steps : 0);
        for (int jj = 0; jj < nsteps_it; ++jj, ++it) {
          const int j = wi.j0 + jj;   // residual K step
          if (kKind == kKindInt && jj == nres) {
            // the low-rank columns: the previous tile's stores are done
            ok = mbar_wait(&lr_empty_bar, (lt & 1) ^ 1, status, &abort_sh);
            if (!ok) break;
            tc_fence_after();
          }
          const int s = it % kStages;
          const uint32_t ph = (it / kStages) & 1;
          ok = mbar_wait(&full_bar[s], ph, status, &abort_sh);
          if (!ok) break;
          tc_fence_after();
          const uint32_t a0 = smem_u32(smem + s * kStageBytes);
          const uint32_t b0 = a0 + kABytes;
          if (jj >= nres) {
            const int l = jj - nres;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_f16_pair(lr_acc, smem_desc_sw128(a0 + 32 * kk), smem_desc_sw128(b0 + 32 * kk), id_bf,
                           (kF4 || l > 0 || kk > 0) ? 1u : 0u);
          } else if constexpr (kF4) {
            const int na = min(kSfAtoms, args.katoms - kSfAtoms * j);
            const uint32_t sfa_s = b0 + kBBytes;
            const uint32_t sfb_s = sfa_s + kSfaBytes;
            for (int kk = 0; kk < na; ++kk) {
              tmem_cp_32x128b_warpx4_pair(tmem + kSfaCol + 4 * kk, smem_desc_plain(sfa_s + 512 * kk));
              for (int rt = 0; rt < 2; ++rt)
                tmem_cp_32x128b_warpx4_pair(tmem + kSfbCol + 8 * kk + 4 * rt,
                                            smem_desc_plain(sfb_s + kSfaBytes * rt + 512 * kk));
            }
            if constexpr (kKind == kKindNvfp4) {
              for (int kk = 0; kk < na; ++kk)
                mma_nvf4_pair(tmem, smem_desc_sw128(a0 + 32 * kk), smem_desc_sw128(b0 + 32 * kk), id_f4,
                              (jj > 0 || kk > 0) ? 1u : 0u, tmem + kSfaCol + 4 * kk, tmem + kSfbCol + 8 * kk);
            } else {
              // MMA kk: atom kk / 2, scale bytes 2 (kk % 2) and up of each row's four
              const int nm = min(4, kmma - 4 * j);
              for (int kk = 0; kk < nm; ++kk)
                mma_mxf4_pair(tmem, smem_desc_sw128(a0 + 32 * kk), smem_desc_sw128(b0 + 32 * kk), ((kk & 1) ? id_mx1 : id_mx0),
                              (jj > 0 || kk > 0) ? 1u : 0u, sf_taddr(tmem + kSfaCol + 4 * (kk >> 1), kk),
                              sf_taddr(tmem + kSfbCol + 8 * (kk >> 1), kk));
            }
          } else {
            const uint32_t bb = a0 + kKb * kABytes;
#pragma unroll
            for (int kk = 0; kk < 4 * kKb; ++kk)
              mma_i8_pair(tmem, smem_desc_sw128(a0 + (kk >> 2) * kABytes + 32 * (kk & 3)),
                          smem_desc_sw128(bb + (kk >> 2) * kBBytes + 32 * (kk & 3)), id_i8,
                          (jj > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit_pair(&empty_bar[s], 0x3);
        }
        if (!ok) break;
        if (kKind == kKindInt && !lr_here) {
          // keep the low-rank barrier's phases in step with the tiles
          ok = mbar_wait(&lr_empty_bar, (lt & 1) ^ 1, status, &abort_sh);
          if (!ok) break;
        }
        mma_commit_pair(&tmem_full_bar, 0x3);
      }
      // both epilogues have released the last tile: no arrival from the odd
      // CTA is still on its way when this CTA leaves
      if (ok && lt > 0) {
        mbar_wait(&acc_empty_bar, (lt - 1) & 1, status, &abort_sh);
        if (kKind == kKindInt) mbar_wait(&lr_empty_bar, (lt - 1) & 1, status, &abort_sh);
      }
    }
  } else {
    // ----------------------------------------------------------- epilogue
    const int q = warp & 3;                         // TMEM lane quarter
    const int h = (warp - 2) >> 2;                  // column half of the tile
    const int r_in = q * 32 + lane;
    const float alpha = epilogue_alpha<kKind, kOut>(args);
    const bool sep_lr = kKind == kKindInt && kOut != kOutI32 && lr_steps > 0;
    const uint32_t acc_empty_even = mapa_shared(smem_u32(&acc_empty_bar), 0);
    const uint32_t lr_empty_even = mapa_shared(smem_u32(&lr_empty_bar), 0);
    auto release = [&](uint32_t even_addr, uint64_t* local) {
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (rank == 0)
          mbar_arrive(local);
        else
          mbar_arrive_remote(even_addr);
      }
    };
    uint32_t lt = 0;
    PairItem wi;
    for (int r = 0; item(r, wi); ++r, ++lt) {
      const int t = wi.t;
      if (!mbar_wait_warp(&tmem_full_bar, lt & 1, status, &abort_sh)) break;
      tc_fence_after();
      const int row = (t % tiles_m) * 2 * kHalf + static_cast<int>(rank) * kHalf + r_in;
      const int nt = (t / tiles_m) * kTileN;
      const uint32_t lane_addr = tmem + (static_cast<uint32_t>(q * 32) << 16);
      if constexpr (kTwoPass) {
        // the warp's four accumulator chunks go to registers first, so the
        // accumulator is handed back to the next tile's MMAs before any
        // arithmetic; the result of chunk c then goes to dst(c): INT in place
        // over its own low-rank columns, fp4 (bf16) to the free columns
        // from 384
        auto dst = [](int c) -> uint32_t {
          return kKind == kKindInt ? 256u + 32u * c : kNvOutCol + 16u * c;
        };
        uint32_t accs[4][32];
        __syncwarp();
#pragma unroll
        for (int i = 0; i < 4; ++i) tmem_ld_32x32b_x32(lane_addr + 32u * (4 * h + i), accs[i]);
#pragma unroll
        for (int i = 0; i < 4; ++i) tmem_ld_wait_regs(accs[i]);
        release(acc_empty_even, &acc_empty_bar);
        if (wi.role != 0) {
          // split tile: the partial of slice sl, laid out [tile q][slice - 1]
          // [CTA rank][column half h][16-byte piece][row], so that each warp
          // access covers 32 consecutive rows' pieces (512 contiguous bytes)
          const size_t per_slice = static_cast<size_t>(2) * kHalf * kTileN / 4;   // in 16-byte pieces
          auto part_row = [&](int sl) {
            return reinterpret_cast<uint4*>(args.split_part) +
                   (static_cast<size_t>(wi.q) * (nsplit - 1) + (sl - 1)) * per_slice +
                   (static_cast<size_t>(rank) * 2 + h) * 32 * kHalf + r_in;
          };
          if (wi.role == 2) {
            // a later slice: the raw accumulator to the workspace, then count
            // this warp's part in; nothing of Y
            uint4* dst4 = part_row(wi.sl);
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
              for (int e = 0; e < 8; ++e)
                __stcg(dst4 + (8 * i + e) * kHalf, make_uint4(accs[i][4 * e], accs[i][4 * e + 1], accs[i][4 * e + 2],
                                                    accs[i][4 * e + 3]));
            __threadfence();
            __syncwarp();
            if (lane == 0) atomicAdd(args.split_cnt + wi.q, 1u);
            if (kKind == kKindInt) release(lr_empty_even, &lr_empty_bar);
            continue;
          }
          // the owner: wait (bounded) until every warp of the other slices'
          // CTAs has written its part, then add the partials in slice order
          const unsigned target = static_cast<unsigned>(2 * kEpiWarps * (nsplit - 1));
          int got = 1;
          if (lane == 0) {
            const unsigned long long t0 = globaltimer_ns();
            while (ld_acquire_gpu_u32(args.split_cnt + wi.q) < target) {
              if (globaltimer_ns() - t0 > kWaitLimitNs) {
                record_status(status, kStatusTimeout);
                got = 0;
                break;
              }
            }
          }
          got = __shfl_sync(0xffffffffu, got, 0);
          __syncwarp();
          if (got) {
            for (int sl = 1; sl < nsplit; ++sl) {
              const uint4* src4 = part_row(sl);
#pragma unroll
              for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                  const uint4 v = __ldcg(src4 + (8 * i + e) * kHalf);
                  const uint32_t pv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                  for (int u = 0; u < 4; ++u) {
                    uint32_t& a = accs[i][4 * e + u];
                    if constexpr (kKind == kKindInt)
                      a = static_cast<uint32_t>(static_cast<int32_t>(a) + static_cast<int32_t>(pv[u]));
                    else
                      a = __float_as_uint(__uint_as_float(a) + __uint_as_float(pv[u]));
                  }
                }
            }
          }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int c = 4 * h + i;
          const int n = nt + 32 * c;
          if (n < N)
            epilogue_combine_regs<kKind, kOut>(args, lane_addr, n, accs[i], 256u + 32u * c, dst(c), alpha, sep_lr);
        }
        tmem_st_wait();
        for (int c = 4 * h; c < 4 * h + 4; ++c) {
          const int n = nt + 32 * c;
          if (n < N) epilogue_store<kOut>(args, lane_addr, row, n, dst(c));
        }
        if (kKind == kKindInt) release(lr_empty_even, &lr_empty_bar);
      } else {
        for (int c = 4 * h; c < 4 * h + 4; ++c)
          epilogue_chunk_direct<kKind, kOut>(args, lane_addr, row, nt + 32 * c, 32u * c, alpha, sep_lr);
        release(acc_empty_even, &acc_empty_bar);
        if (kKind == kKindInt) release(lr_empty_even, &lr_empty_bar);
      }
    }
  }

  // teardown: each CTA tells the other it is done and waits (bounded) to hear
  // the same, so neither releases TMEM or shared memory the other still uses
  __syncthreads();
  if (threadIdx.x == 0) {
    mbar_arrive_remote(mapa_shared(smem_u32(&exit_bar), rank ^ 1u));
    mbar_wait(&exit_bar, 0, status, nullptr);
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, kTmemCols);
  }
}

// The K split of the last round: with P CTA pairs and T tiles, R = T / P full
// rounds leave T mod P tiles for a last round in which most pairs would idle;
// each of those tiles is cut into s slices (s (T mod P) <= P), so s (T mod P)
// pairs share the last round. (A grid of fewer tiles than pairs is one such
// round.) The split saves (1 - 1/s) of a tile's K steps and costs the owner an
// exposed epilogue (about 7 K steps' time) and the reading of s - 1 partial
// tiles (about 2.4 K steps' time each, measured at K = 12288): s maximises the
// saving net of that cost, and no split is taken when it is not positive.
int pick_nsplit(int64_t ksteps, int64_t smax) {
  int best = 1;
  double best_net = 0.0;
  for (int64_t s = 2; s <= std::min<int64_t>(smax, 8); ++s) {
    const double net = (1.0 - 1.0 / static_cast<double>(s)) * static_cast<double>(ksteps) - 7.0 -
                       2.4 * static_cast<double>(s - 1);
    if (net > best_net) {
      best_net = net;
      best = static_cast<int>(s);
    }
  }
  return best;
}

struct PairSplit {
  int pairs, trem, nsplit;
};
PairSplit pair_split(int64_t B, int64_t M, int64_t N) {
  const int64_t tiles = ceil_div(B, 2 * kHalf) * ceil_div(N, kTileN);
  const int64_t P = std::max(1, num_sms() / 2);
  const int64_t ksteps = ceil_div(M, 256);
  PairSplit ps{static_cast<int>(std::min(tiles, P)), 0, 1};
  const int64_t trem = tiles >= P ? tiles % P : tiles;
  if (trem == 0) return ps;
  const int64_t s = pick_nsplit(ksteps, std::min<int64_t>(P / trem, ksteps));
  if (s < 2) return ps;
  ps.trem = static_cast<int>(trem);
  ps.nsplit = static_cast<int>(s);
  if (tiles < P) ps.pairs = static_cast<int>(trem * s);
  return ps;
}

template <int kKind, int kOut>
cudaError_t launch_pair_one(const CUtensorMap* maps, const GemmArgs& args, int grid, cudaStream_t st) {
  const size_t smem = static_cast<size_t>(PairCfg<kKind>::kStages) * PairCfg<kKind>::kStageBytes + 1024;
  cudaError_t err = cudaFuncSetAttribute(gemm_pair_kernel<kKind, kOut>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
  if (err != cudaSuccess) return err;
  gemm_pair_kernel<kKind, kOut><<<grid, kPairThreads, smem, st>>>(maps[0], maps[1], maps[2], maps[3],
                                                                    maps[4], maps[5], args);
  return cudaGetLastError();
}

}  // namespace

// Builds the pair kernel's tensor maps and launches it; returns false (and
// launches nothing) if a map cannot be encoded.
size_t pair_split_counter_offset(int64_t B, int64_t M, int64_t N) {
  const PairSplit ps = pair_split(B, M, N);
  return ps.nsplit < 2 ? 0 : static_cast<size_t>(ps.trem) * (ps.nsplit - 1) * 2 * kHalf * kTileN * 4;
}

int pair_split_counters(int64_t B, int64_t M, int64_t N) {
  const PairSplit ps = pair_split(B, M, N);
  return ps.nsplit < 2 ? 0 : ps.trem;
}

size_t pair_split_bytes(int64_t B, int64_t M, int64_t N) {
  const PairSplit ps = pair_split(B, M, N);
  if (ps.nsplit < 2) return 0;
  return pair_split_counter_offset(B, M, N) + static_cast<size_t>(round_up(static_cast<int64_t>(ps.trem) * 4, 256));
}

bool launch_gemm_pair(int kind, int out, const GemmArgs& args_in, const void* act_codes,
                      const void* down2, const svdq_weight* w, void* split_ws, cudaStream_t stream,
                      cudaError_t* err) {
  *err = cudaSuccess;
  GemmArgs args = args_in;
  const int64_t M = args.M, N = args.N, B = args.B;
  const int rp = w->rank_pad;
  const int64_t row_bytes = kind != kKindInt ? M / 2 : M;
  CUtensorMap maps[6];
  bool ok =
      make_tmap_2d(&maps[0], act_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, row_bytes, B, row_bytes, 128, kHalf, true) &&
      make_tmap_2d(&maps[1], w->codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, row_bytes, N, row_bytes, 128, kHalf, true);
  if (ok && args.lr_steps) {
    ok = make_tmap_2d(&maps[2], down2, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, 2 * rp, B, 2 * rp, 64, kHalf, true) &&
         make_tmap_2d(&maps[3], w->lu, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, 2 * rp, N, 2 * rp, 64, kHalf, true);
  } else {
    maps[2] = maps[0];
    maps[3] = maps[1];
  }
  if (ok && kind != kKindInt) {
    // one box = the scale atoms of one stage (two 256-byte rows per atom)
    const int box = kind == kKindMxfp4 ? 2 * PairCfg<kKindMxfp4>::kSfAtoms : 2 * PairCfg<kKindNvfp4>::kSfAtoms;
    const int64_t rows_a = ceil_div(B, 128) * args.katoms * 2;
    const int64_t rows_b = ceil_div(N, 128) * args.katoms * 2;
    ok = make_tmap_2d(&maps[4], args.sfa, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, 256, rows_a, 256, 256, box, false) &&
         make_tmap_2d(&maps[5], args.sfb, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, 256, rows_b, 256, 256, box, false);
  } else {
    maps[4] = maps[0];
    maps[5] = maps[1];
  }
  if (!ok) return false;
  // the split needs the workspace and the two-pass epilogue; it is taken for INT
  // only, whose int32 sums are exact in any order (a split fp4 tile would round
  // its fp32 sums differently from the same tile unsplit, so the fp32 and bf16
  // outputs of one call, or the workspace and the staged entry points, could
  // differ in the last bit)
  PairSplit ps = pair_split(B, M, N);
  const bool splittable = kind == kKindInt && (out == kOutBF16 || out == kOutF32);
  if (split_ws == nullptr || !splittable || (reinterpret_cast<uintptr_t>(split_ws) & 15) != 0) {
    const int64_t tiles = ceil_div(B, 2 * kHalf) * ceil_div(N, kTileN);
    ps = PairSplit{static_cast<int>(std::min<int64_t>(tiles, std::max(1, num_sms() / 2))), 0, 1};
  }
  args.nsplit = ps.nsplit;
  if (ps.nsplit > 1) {
    args.split_part = static_cast<uint32_t*>(split_ws);
    // the counters must be zero at the launch (the activation pass clears them)
    args.split_cnt = reinterpret_cast<unsigned*>(static_cast<uint8_t*>(split_ws) + pair_split_counter_offset(B, M, N));
  }
  const int grid = 2 * ps.pairs;
  if (kind == kKindInt) {
    if (out == kOutI32) *err = launch_pair_one<kKindInt, kOutI32>(maps, args, grid, stream);
    else if (out == kOutF32) *err = launch_pair_one<kKindInt, kOutF32>(maps, args, grid, stream);
    else *err = launch_pair_one<kKindInt, kOutBF16>(maps, args, grid, stream);
  } else if (kind == kKindMxfp4) {
    if (out == kOutF32) *err = launch_pair_one<kKindMxfp4, kOutF32>(maps, args, grid, stream);
    else *err = launch_pair_one<kKindMxfp4, kOutBF16>(maps, args, grid, stream);
  } else {
    if (out == kOutF32) *err = launch_pair_one<kKindNvfp4, kOutF32>(maps, args, grid, stream);
    else *err = launch_pair_one<kKindNvfp4, kOutBF16>(maps, args, grid, stream);
  }
  return true;
}

}  // namespace svdq
