// decode.cu - the whole SVDQuant linear for up to 16 rows of x with INT
// weights, in one launch.
//
// "SVDQuant Smoothing, Low-rank and Residual Quantization", Formula items 1-3:
// Y = x ld^T lu^T + s_x s_w (Q(X_hat) . Q(R)), X_hat = x / scale, per-tensor
// INT grid. With a few rows the activation pass is a few thousand elements
// and the cost of the step is launches and the dependencies between them, not
// the weight stream. So one kernel does everything. The grid is clusters of 8
// CTAs (no more clusters than fit on the GPU at once); each CTA owns a run of
// weight rows and, inside its cluster, one eighth of K (its share):
//   1. warp 0 issues bulk copies at entry: the CTA's weight rows (packed 4-bit
//      or int8 codes) and lu rows, its share of x and of every ld row. (A
//      dependent launch issues the weight side first and waits for the kernel
//      before it only then.)
//   2. each CTA takes the maximum of |X_hat| over its share; after a cluster
//      barrier every CTA combines the 8 partial maxima (the same per-tensor
//      scale everywhere). The partial down-projection x ld^T of the share
//      (warp MMAs, fp32 accumulate) runs while the barrier completes.
//   3. each CTA writes the codes of its share (exact rounding as in
//      encode.cuh) into the shared memory of all 8 CTAs of its cluster; after
//      a second barrier every CTA holds the codes of all of x and sums the 8
//      partial down tiles in rank order.
//   4. the int32 dot products of the weight rows with the codes run on warp
//      MMAs (m16n8k32, s8; 16 weight rows by 8 batch rows per tile, warps
//      splitting K), the partials are summed in a fixed order, and one thread
//      per output forms Y = s_x s_w acc + down . lu + bias.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>

#include "encode.cuh"
#include "gemm_common.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace svdq {

namespace {

constexpr int kDecThreads = 512;
constexpr int kDecWarps = kDecThreads / 32;
constexpr int kDecCluster = 8;
constexpr int kDecMaxB = 16;
constexpr size_t kDecSmemMax = 220 * 1024;
constexpr int kMaxDevs = 64;
std::atomic<int> g_max_clusters[kMaxDevs];

struct DecodeArgs {
  int B, N, M, rp, rows_per_cta, row_bytes, qmax, chained;
  int kslice;        // columns of a share (a multiple of 16)
  int sstride;       // bytes between rows of the x and ld shares
  int wstride;       // bytes between weight rows
  int astride;       // bytes between rows of the codes
  int lstride;       // bytes between lu rows (4 rank_pad: one bulk copy)
  int mtiles, ksub;  // 16-row weight tiles; warps splitting K per tile
  int64_t ldx, ldy;
  const void* x;
  const float* scale;
  const uint8_t* w;             // packed [N, M/2] or int8 [N, M]
  const void* ld;               // [rp, M], x's dtype
  const __nv_bfloat16* lu;      // [N, 2 rp]; the first rp columns are L2^T
  const float* s_w;
  const __nv_bfloat16* bias;
  void* y;
  unsigned* status;
};

// Shared memory: the partial dot products (red) reuse the x and ld shares,
// which are dead by then.
struct DecodeLayout {
  size_t ws, lus, xs, lds, red, rk, acts, part, down, total;
};

__host__ __device__ inline DecodeLayout decode_layout(const DecodeArgs& g) {
  DecodeLayout L{};
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o = (o + bytes + 15) / 16 * 16;
    return at;
  };
  L.ws = take(static_cast<size_t>(g.rows_per_cta) * g.wstride);
  L.lus = take(static_cast<size_t>(g.rows_per_cta) * g.lstride);   // whole lu rows (both copies of L2^T)
  const size_t shares = static_cast<size_t>(g.B + g.rp) * g.sstride;
  const size_t red = static_cast<size_t>(g.mtiles) * g.ksub * 16 * 16 * 4;
  const size_t region = take(shares > red ? shares : red);
  L.xs = region;
  L.lds = region + static_cast<size_t>(g.B) * g.sstride;
  L.red = region;
  L.rk = take(static_cast<size_t>(g.kslice) * 4);
  L.acts = take(static_cast<size_t>(g.B) * g.astride);
  L.part = take(static_cast<size_t>(g.B) * g.rp * 4);
  L.down = take(static_cast<size_t>(g.B) * (g.rp + 1) * 4);   // rows rp + 1 apart: no bank conflicts
  L.total = o;
  return L;
}

template <typename TIn>
__device__ __forceinline__ float to_f(const uint8_t* base, int idx) {
  if constexpr (sizeof(TIn) == 2)
    return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(base)[idx]);
  else
    return reinterpret_cast<const float*>(base)[idx];
}

__device__ __forceinline__ void st_cluster_v2(uint32_t cluster_addr, uint2 v) {
  asm volatile("st.shared::cluster.v2.u32 [%0], {%1, %2};" ::"r"(cluster_addr), "r"(v.x), "r"(v.y) : "memory");
}

__device__ __forceinline__ uint2 ld_shared_v2(uint32_t saddr) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(saddr) : "memory");
  return v;
}

// The two halves of a whole-cluster barrier, so that independent work can run
// between a CTA's arrival and its wait.
__device__ __forceinline__ void cluster_arrive() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// D += A B for one 16 x 8 int32 tile, A 16 x 32 s8 (row), B 32 x 8 s8 (col),
// fragments as the PTX ISA gives them for mma.sync m16n8k32.
__device__ __forceinline__ void mma_s8_16832(int (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// Eight 4-bit two's-complement codes (element i in bits 4i..4i+3) as eight
// int8: elements 0-3 in lo, 4-7 in hi.
__device__ __forceinline__ void widen8(uint32_t w, uint32_t& lo, uint32_t& hi) {
  uint32_t e = w & 0x0F0F0F0Fu;           // elements 0, 2, 4, 6
  uint32_t o = (w >> 4) & 0x0F0F0F0Fu;    // elements 1, 3, 5, 7
  e |= (e & 0x08080808u) * 0x1Eu;         // sign-extend each nibble to its byte
  o |= (o & 0x08080808u) * 0x1Eu;
  lo = __byte_perm(e, o, 0x5140);
  hi = __byte_perm(e, o, 0x7362);
}

template <typename TIn, bool kPacked, int kOut, int kNT>
__global__ void __launch_bounds__(kDecThreads, 1) decode_kernel(const DecodeArgs g) {
  constexpr int kEsz = static_cast<int>(sizeof(TIn));
  extern __shared__ __align__(16) uint8_t dsm[];
  __shared__ float red_max[kDecWarps];
  __shared__ float pmax;
  __shared__ __align__(8) uint64_t bar[2];   // 0: the x and ld shares, 1: weight and lu rows
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gq = lane >> 2, tq = lane & 3;   // MMA fragment coordinates
  const int crank = static_cast<int>(cluster_ctarank());
  const int n0 = blockIdx.x * g.rows_per_cta;
  const int rows = max(0, min(g.rows_per_cta, g.N - n0));
  const int B = g.B;
  const DecodeLayout L = decode_layout(g);
  uint8_t* ws = dsm + L.ws;
  uint8_t* lus = dsm + L.lus;
  uint8_t* xs = dsm + L.xs;
  uint8_t* lds = dsm + L.lds;
  int* red = reinterpret_cast<int*>(dsm + L.red);
  float* rk = reinterpret_cast<float*>(dsm + L.rk);
  uint8_t* acts = dsm + L.acts;
  float* part = reinterpret_cast<float*>(dsm + L.part);
  float* down = reinterpret_cast<float*>(dsm + L.down);
  const int k0 = min(g.M, crank * g.kslice), k1 = min(g.M, k0 + g.kslice);
  const int kn = k1 - k0;   // columns of this CTA's share (a multiple of 16, may be 0)
  if (tid == 0) {
    mbar_init(&bar[0], 1);
    mbar_init(&bar[1], 1);
    fence_mbar_init();
  }
  __syncthreads();
  // a chained linear queued after this kernel may start its weight-side setup
  // now (it reads this kernel's output only after griddepcontrol.wait)
  pdl_trigger();

  // ---- 1. warp 0 issues every copy as a bulk copy (one per weight row, to
  // padded rows)
  if (warp == 0) {
    auto issue_x = [&]() {
      const uint32_t share = static_cast<uint32_t>(kn) * kEsz;
      if (lane == 0) mbar_arrive_expect_tx(&bar[0], static_cast<uint32_t>(B + g.rp) * share);
      __syncwarp();
      if (share > 0) {
        for (int b = lane; b < B; b += 32)
          bulk_load(xs + static_cast<size_t>(b) * g.sstride,
                    static_cast<const uint8_t*>(g.x) + (static_cast<int64_t>(b) * g.ldx + k0) * kEsz, share, &bar[0]);
        for (int j = lane; j < g.rp; j += 32)
          bulk_load(lds + static_cast<size_t>(j) * g.sstride,
                    static_cast<const uint8_t*>(g.ld) + (static_cast<int64_t>(j) * g.M + k0) * kEsz, share, &bar[0]);
      }
    };
    auto issue_w = [&]() {
      const uint32_t ltot = static_cast<uint32_t>(rows) * static_cast<uint32_t>(g.rp) * 4u;
      if (lane == 0) mbar_arrive_expect_tx(&bar[1], static_cast<uint32_t>(rows * g.row_bytes) + ltot);
      __syncwarp();
      for (int r = lane; r < rows; r += 32)
        bulk_load(ws + static_cast<size_t>(r) * g.wstride, g.w + static_cast<int64_t>(n0 + r) * g.row_bytes,
                  static_cast<uint32_t>(g.row_bytes), &bar[1]);
      if (ltot > 0 && lane == 31)
        bulk_load(lus, reinterpret_cast<const uint8_t*>(g.lu) + static_cast<int64_t>(n0) * g.rp * 4, ltot, &bar[1]);
    };
    // a chained launch (x is the previous linear's output) starts the weight
    // side before it waits for that kernel; otherwise x goes first (the
    // weights issued only after x has landed arrive during the later phases
    // and slow them more than they delay x when issued together)
    if (g.chained) {
      issue_w();
      pdl_wait();
      issue_x();
    } else {
      issue_x();
      issue_w();
    }
  }
  // reciprocals of the share's smoothing scales (the estimates of the codes)
  for (int c = tid; c < kn; c += kDecThreads) rk[c] = __frcp_rn(__ldg(g.scale + k0 + c));
  // a wait that gives up records the timeout in g.status; the kernel then runs
  // to the end (every CTA must reach every cluster barrier)
  mbar_wait_warp(&bar[0], 0, g.status, nullptr);

  // ---- 2. maximum of |X_hat| over the share (IEEE quotients of the column maxima)
  float m = 0.0f;
  for (int c = tid; c < kn; c += kDecThreads) {
    float cm = 0.0f;
    for (int b = 0; b < B; ++b) cm = fmaxf(cm, fabsf(to_f<TIn>(xs + static_cast<size_t>(b) * g.sstride, c)));
    m = fmaxf(m, __fdiv_rn(cm, __ldg(g.scale + k0 + c)));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (lane == 0) red_max[warp] = m;
  __syncthreads();
  if (tid == 0) {
    float mm = red_max[0];
    for (int w = 1; w < kDecWarps; ++w) mm = fmaxf(mm, red_max[w]);
    pmax = mm;
  }
  cluster_arrive();   // #1: this CTA's partial maximum is written
  // the share's partial down tile, while the barrier completes: warp w takes
  // 8-column tiles w, w + 16, ... of the rank_pad columns (rows of x past B are 0)
  {
    const uint32_t xa = smem_u32(xs), la = smem_u32(lds);
    for (int nt = warp; nt < g.rp / 8; nt += kDecWarps) {
      // four accumulators over alternating K steps (independent MMA chains),
      // added in a fixed order at the end
      float dd[4][4] = {};
      const uint32_t lrow = la + static_cast<uint32_t>((nt * 8 + gq) * g.sstride);
      const uint32_t xr0 = xa + static_cast<uint32_t>(gq * g.sstride);
      const uint32_t xr1 = xa + static_cast<uint32_t>((gq + 8) * g.sstride);
      const bool r0 = gq < B, r1 = gq + 8 < B;
      if constexpr (kEsz == 2) {
        for (int k4 = 0; k4 < kn; k4 += 64) {
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int kk = k4 + 16 * u;
            if (kk >= kn) break;
            const uint32_t o0 = static_cast<uint32_t>(kk + 2 * tq) * 2, o1 = o0 + 16;
            uint32_t a[4], b[2];
            a[0] = r0 ? ld_shared_u32(xr0 + o0) : 0u;
            a[1] = r1 ? ld_shared_u32(xr1 + o0) : 0u;
            a[2] = r0 ? ld_shared_u32(xr0 + o1) : 0u;
            a[3] = r1 ? ld_shared_u32(xr1 + o1) : 0u;
            b[0] = ld_shared_u32(lrow + o0);
            b[1] = ld_shared_u32(lrow + o1);
            mma_bf16_16816(dd[u], a, b);
          }
        }
      } else {
        for (int k4 = 0; k4 < kn; k4 += 32) {
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int kk = k4 + 8 * u;
            if (kk >= kn) break;
            const uint32_t o0 = static_cast<uint32_t>(kk + tq) * 4, o1 = o0 + 16;
            uint32_t a[4], b[2];
            a[0] = r0 ? to_tf32(ld_shared_u32(xr0 + o0)) : 0u;
            a[1] = r1 ? to_tf32(ld_shared_u32(xr1 + o0)) : 0u;
            a[2] = r0 ? to_tf32(ld_shared_u32(xr0 + o1)) : 0u;
            a[3] = r1 ? to_tf32(ld_shared_u32(xr1 + o1)) : 0u;
            b[0] = to_tf32(ld_shared_u32(lrow + o0));
            b[1] = to_tf32(ld_shared_u32(lrow + o1));
            mma_tf32_1688(dd[u], a, b);
          }
        }
      }
      float d[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) d[e] = (dd[0][e] + dd[1][e]) + (dd[2][e] + dd[3][e]);
      const int j = nt * 8 + 2 * tq;
      if (r0) {
        part[gq * g.rp + j] = d[0];
        part[gq * g.rp + j + 1] = d[1];
      }
      if (r1) {
        part[(gq + 8) * g.rp + j] = d[2];
        part[(gq + 8) * g.rp + j + 1] = d[3];
      }
    }
  }
  cluster_wait();   // #1: every CTA's partial maximum is written
  // the per-tensor scale from the 8 partial maxima (lanes 0-7 of each warp)
  {
    float pm = lane < kDecCluster ? ld_cluster_f32(mapa_shared(smem_u32(&pmax), lane)) : 0.0f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) pm = fmaxf(pm, __shfl_xor_sync(0xffffffffu, pm, o));
    m = pm;
  }
  const float s = __fdiv_rn(m, static_cast<float>(g.qmax));
  const float u = s > 0.0f ? __frcp_rn(s) : 0.0f;

  // ---- 3. codes of this share, 8 columns per item, into every CTA of the cluster
  {
    const int n8 = kn / 8;
    for (int i = tid; i < B * n8; i += kDecThreads) {
      const int b = i / n8, cl = (i - b * n8) * 8;   // column within the share
      const uint8_t* xr = xs + static_cast<size_t>(b) * g.sstride;
      float v[8], ck[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        v[j] = to_f<TIn>(xr, cl + j);
        ck[j] = __fmul_rn(rk[cl + j], u);
      }
      const uint2 q = int_codes8(v, ck, g.scale + k0 + cl, s, g.qmax);
      const uint32_t at = smem_u32(acts + static_cast<size_t>(b) * g.astride + k0 + cl);
#pragma unroll
      for (int r = 0; r < kDecCluster; ++r) st_cluster_v2(mapa_shared(at, r), q);
    }
  }
  cluster_arrive();   // #2: this CTA's codes and partial down tile are written
  mbar_wait_warp(&bar[1], 0, g.status, nullptr);   // the weight and lu rows
  cluster_wait();     // #2: every CTA holds all codes and its partial down tile

  // ---- 4. dot products on warp MMAs. Inside each 32-code K step, fragment
  // slot 4t + i (i < 4) holds code 8t + i and slot 16 + 4t + i holds code
  // 8t + 4 + i, for the weights and the codes alike: a permutation of K, so the
  // sums are unchanged, and each lane reads 8 consecutive codes.
  if (rows > 0) {
    const int nk = g.M / 32;
    for (int task = warp; task < g.mtiles * g.ksub; task += kDecWarps) {
      const int mt = task / g.ksub, kp = task - mt * g.ksub;
      const int ks0 = (nk * kp) / g.ksub, ks1 = (nk * (kp + 1)) / g.ksub;
      // rows past the end repeat the last (their sums are not used)
      const int ra = min(mt * 16 + gq, rows - 1), rb = min(mt * 16 + gq + 8, rows - 1);
      const uint32_t wa = smem_u32(ws + static_cast<size_t>(ra) * g.wstride);
      const uint32_t wb = smem_u32(ws + static_cast<size_t>(rb) * g.wstride);
      // two accumulators per batch tile over alternating K steps (independent
      // MMA chains; int32 sums, exact in any order)
      int acc[2][kNT][4] = {};
      for (int k2 = ks0; k2 < ks1; k2 += 2) {
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int ks = k2 + u;
          if (ks >= ks1) break;
          uint32_t a[4];
          if constexpr (kPacked) {
            widen8(ld_shared_u32(wa + ks * 16 + 4 * tq), a[0], a[2]);
            widen8(ld_shared_u32(wb + ks * 16 + 4 * tq), a[1], a[3]);
          } else {
            const uint2 va = ld_shared_v2(wa + ks * 32 + 8 * tq), vb = ld_shared_v2(wb + ks * 32 + 8 * tq);
            a[0] = va.x;
            a[2] = va.y;
            a[1] = vb.x;
            a[3] = vb.y;
          }
#pragma unroll
          for (int t = 0; t < kNT; ++t) {
            const int col = t * 8 + gq;   // batch row
            uint32_t bf[2] = {0u, 0u};
            if (col < B) {
              const uint2 vb = ld_shared_v2(smem_u32(acts + static_cast<size_t>(col) * g.astride + ks * 32 + 8 * tq));
              bf[0] = vb.x;
              bf[1] = vb.y;
            }
            mma_s8_16832(acc[u][t], a, bf);
          }
        }
      }
      int* rt = red + task * 256;   // [16 weight rows][16 batch rows]
#pragma unroll
      for (int t = 0; t < kNT; ++t) {
        const int c = t * 8 + 2 * tq;
        rt[gq * 16 + c] = acc[0][t][0] + acc[1][t][0];
        rt[gq * 16 + c + 1] = acc[0][t][1] + acc[1][t][1];
        rt[(gq + 8) * 16 + c] = acc[0][t][2] + acc[1][t][2];
        rt[(gq + 8) * 16 + c + 1] = acc[0][t][3] + acc[1][t][3];
      }
    }
  }
  // the down-projection: the 8 partial tiles of the cluster in rank order
  const int nout = B * g.rp;
  for (int o = tid; o < nout; o += kDecThreads) {
    float sum = 0.0f;
    for (int r = 0; r < kDecCluster; ++r) sum += ld_cluster_f32(mapa_shared(smem_u32(part + o), r));
    const int b = o / g.rp;
    down[b * (g.rp + 1) + (o - b * g.rp)] = sum;
  }
  cluster_arrive();   // #3: this CTA reads no other CTA's memory from here on
  __syncthreads();    // the partial dot products and the down sums

  // ---- epilogue: one thread per output, consecutive threads along the batch
  // (then n); each lane starts the up-projection at its own column, so the lu
  // rows and the down sums are read (nearly) without bank conflicts
  const float alpha = s * __ldg(g.s_w);
  const int q0 = g.rp > 0 ? lane % g.rp : 0;
  for (int o = tid; o < B * rows; o += kDecThreads) {
    const int r = o / B, b = o - r * B;
    const int mt = r >> 4, rr = r & 15;
    int isum = 0;
    for (int kp = 0; kp < g.ksub; ++kp) isum += red[(mt * g.ksub + kp) * 256 + rr * 16 + b];
    const __nv_bfloat16* lr = reinterpret_cast<const __nv_bfloat16*>(lus + static_cast<size_t>(r) * g.lstride);
    const float* dn = down + b * (g.rp + 1);
    float up = 0.0f;
    for (int i = 0, q = q0; i < g.rp; ++i, q = q + 1 < g.rp ? q + 1 : 0)
      up = fmaf(dn[q], __bfloat162float(lr[q]), up);
    const int n = n0 + r;
    float yv = alpha * static_cast<float>(isum) + up;
    if (g.bias != nullptr) yv += __bfloat162float(g.bias[n]);
    if constexpr (kOut == kOutF32)
      static_cast<float*>(g.y)[static_cast<int64_t>(b) * g.ldy + n] = yv;
    else
      static_cast<__nv_bfloat16*>(g.y)[static_cast<int64_t>(b) * g.ldy + n] = __float2bfloat16_rn(yv);
  }
  cluster_wait();   // #3: no CTA leaves while another may still read its partial down tile
}

template <typename TIn, bool kPacked, int kOut, int kNT>
cudaError_t launch_decode_one(const DecodeArgs& g, int grid, size_t smem, bool pdl, cudaStream_t st) {
  auto kern = decode_kernel<TIn, kPacked, kOut, kNT>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (err != cudaSuccess) return err;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kDecThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kDecCluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, kern, g);
}

// Clusters of 8 CTAs (one per SM, most of the shared memory) that can be
// resident at once on this device: the grid never exceeds them, since a
// cluster started late would double the kernel's time. Queried once per device.
int max_decode_clusters() {
  int d = 0;
  if (cudaGetDevice(&d) != cudaSuccess || d < 0 || d >= kMaxDevs) d = 0;
  int n = g_max_clusters[d].load(std::memory_order_relaxed);
  if (n > 0) return n;
  auto kern = decode_kernel<__nv_bfloat16, true, kOutBF16, 2>;
  n = 0;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kDecSmemMax)) ==
      cudaSuccess) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(static_cast<unsigned>(kDecCluster));
    cfg.blockDim = dim3(kDecThreads);
    cfg.dynamicSmemBytes = kDecSmemMax;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kDecCluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) n = 0;
  }
  (void)cudaGetLastError();
  if (n <= 0) n = num_sms() / (2 * kDecCluster);   // conservative: half the SMs
  g_max_clusters[d].store(n, std::memory_order_relaxed);
  return n;
}

}  // namespace

bool launch_decode(const svdq_weight* w, const void* x, svdq_dtype xdt, int64_t B, int64_t ldx, const void* bias,
                   void* y, svdq_dtype ydt, int64_t ldy, bool chained, cudaStream_t st, cudaError_t* err) {
  *err = cudaSuccess;
  if (w->fmt.kind != SVDQ_KIND_INT || B < 1 || B > kDecMaxB) return false;
  const int64_t M = w->M, N = w->N;
  const int esz = xdt == SVDQ_BF16 ? 2 : 4;
  const int rp = w->rank > 0 ? w->rank_pad : 0;
  const void* ld = xdt == SVDQ_BF16 ? w->ld : w->ld32;
  if (rp > 0 && ld == nullptr) return false;
  const bool packed = w->fmt.bits <= 4 && w->codes4 != nullptr;
  for (const void* q : {static_cast<const void*>(packed ? w->codes4 : w->codes), x, ld,
                        static_cast<const void*>(w->lu), bias})
    if (q != nullptr && (reinterpret_cast<uintptr_t>(q) & 15) != 0) return false;
  if ((ldx * esz) % 16 != 0) return false;
  DecodeArgs g{};
  g.B = static_cast<int>(B);
  g.N = static_cast<int>(N);
  g.M = static_cast<int>(M);
  g.rp = rp;
  g.row_bytes = static_cast<int>(packed ? M / 2 : M);
  // weight rows per CTA: a multiple of 8, over no more CTAs than fit at once
  const int64_t ctas = std::min<int64_t>(static_cast<int64_t>(max_decode_clusters()) * kDecCluster, num_sms());
  g.rows_per_cta = static_cast<int>(round_up(ceil_div(N, ctas), 8));
  const int grid = static_cast<int>(round_up(ceil_div(N, g.rows_per_cta), kDecCluster));
  g.qmax = (1 << (w->fmt.bits - 1)) - 1;
  g.chained = chained ? 1 : 0;
  // each CTA's share of K: a multiple of 16 columns (whole MMA steps, whole
  // 16-byte pieces); with M a multiple of 32 every share is
  g.kslice = static_cast<int>(round_up(ceil_div(M, kDecCluster), 16));
  // row pitches padded so each MMA fragment load falls on distinct banks:
  // 16 bytes past a multiple of 128 for 4-byte loads, 32 for 8-byte loads
  g.sstride = g.kslice * esz + 16;
  g.wstride = g.row_bytes + (packed ? 16 : 32);
  g.astride = static_cast<int>(M) + 32;
  g.lstride = rp * 4;
  g.mtiles = static_cast<int>(ceil_div(g.rows_per_cta, 16));
  g.ksub = std::max(1, kDecWarps / g.mtiles);
  const DecodeLayout L = decode_layout(g);
  if (L.total > kDecSmemMax) return false;
  g.ldx = ldx;
  g.ldy = ldy;
  g.x = x;
  g.scale = w->scale;
  g.w = static_cast<const uint8_t*>(packed ? w->codes4 : w->codes);
  g.ld = rp > 0 ? ld : nullptr;
  g.lu = static_cast<const __nv_bfloat16*>(w->lu);
  g.s_w = w->w_scale;
  g.bias = static_cast<const __nv_bfloat16*>(bias);
  g.y = y;
  g.status = device_status_word();
  const bool two = B > 8;
#define SVDQ_DEC(T, P, O)                                                   \
  *err = two ? launch_decode_one<T, P, O, 2>(g, grid, L.total, chained, st) \
             : launch_decode_one<T, P, O, 1>(g, grid, L.total, chained, st)
  if (xdt == SVDQ_BF16) {
    if (packed) {
      if (ydt == SVDQ_F32) SVDQ_DEC(__nv_bfloat16, true, kOutF32); else SVDQ_DEC(__nv_bfloat16, true, kOutBF16);
    } else {
      if (ydt == SVDQ_F32) SVDQ_DEC(__nv_bfloat16, false, kOutF32); else SVDQ_DEC(__nv_bfloat16, false, kOutBF16);
    }
  } else {
    if (packed) {
      if (ydt == SVDQ_F32) SVDQ_DEC(float, true, kOutF32); else SVDQ_DEC(float, true, kOutBF16);
    } else {
      if (ydt == SVDQ_F32) SVDQ_DEC(float, false, kOutF32); else SVDQ_DEC(float, false, kOutBF16);
    }
  }
#undef SVDQ_DEC
  return true;
}

}  // namespace svdq
