// prepare.cu - the one-time weight split of the SVDQuant linear, on the GPU.
//
// "SVDQuant Smoothing, Low-rank and Residual Quantization", Formula items 1-2:
// ws = scale[:, None] * W, left @ right a best rank-r approximation of ws by
// truncated SVD, residual = ws - left @ right; the offline transforms of
// "flashinfer.gemm.svdquant_linear" fold the smoothing into the down factor.
//
// The truncated SVD is computed by randomized subspace iteration (Halko,
// Martinsson & Tropp, "Finding structure with randomness", SIAM Review 2011,
// Algorithms 4.4 and 5.1):
//   Omega ~ N(0,1)^{N x l}, l = min(r + p, M, N)   (Philox4x32-10 + Box-Muller)
//   Q = orth(ws Omega);  q times: Q' = orth(ws^T Q), Q = orth(ws Q')
//   Bt = ws^T Q = Qb Rb (thin QR)  =>  Q^T ws = Rb^T Qb^T
//   Rb^T = Ur S Vr^T (one-sided Jacobi, Hestenes 1958)  =>  ws ~ (Q Ur) S (Qb Vr)^T
// orth() is a Householder QR (Golub & Van Loan, Alg. 5.2.1 and the backward
// accumulation of Q, Sec. 5.1.6), run by one cooperative kernel whose CTAs each
// keep a slice of rows in shared memory and meet at bounded grid barriers for
// the two reductions of every column.
// The factors are rounded to bf16 (1/scale folded into ld), the residual is
// formed against the rounded factors, then quantised (quant.cu).
#include <cooperative_groups.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <vector>

#include "internal.h"
#include "ptx.cuh"

namespace svdq {

namespace {

constexpr int kDefaultOversample = 16;
constexpr int kDefaultPowerIters = 4;
constexpr int kQrThreads = 512;
constexpr int kMaxL = 288;

// ---------------------------------------------------------------- smoothing
template <typename TW>
__global__ void __launch_bounds__(256) smooth_weight_kernel(const TW* __restrict__ W, int64_t ldW,
                                                            const float* __restrict__ scale,
                                                            int64_t M, int64_t N,
                                                            float* __restrict__ ws,
                                                            unsigned* status) {
  const int64_t total = M * N;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t m = i / N, n = i - m * N;
    const float s = __ldg(scale + m);
    if (n == 0 && !(s > 0.0f && s <= 3.402823466e38f)) record_status(status, kStatusEinval);
    float w;
    if constexpr (sizeof(TW) == 2)
      w = __bfloat162float(W[m * ldW + n]);
    else
      w = W[m * ldW + n];
    ws[i] = __fmul_rn(s, w);
  }
}

// ------------------------------------------------------- Gaussian test matrix
// Philox4x32-10 (Salmon, Moraes, Dror & Shaw, SC'11): 10 rounds of the
// multiply-xor bijection keyed by the seed, counter = block index of 4 outputs.
__device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint2 k) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    const uint32_t hi0 = __umulhi(0xD2511F53u, c.x), lo0 = 0xD2511F53u * c.x;
    const uint32_t hi1 = __umulhi(0xCD9E8D57u, c.z), lo1 = 0xCD9E8D57u * c.z;
    c = make_uint4(hi1 ^ c.y ^ k.x, lo1, hi0 ^ c.w ^ k.y, lo0);
    k.x += 0x9E3779B9u;
    k.y += 0xBB67AE85u;
  }
  return c;
}

__global__ void __launch_bounds__(256) gaussian_kernel(float* __restrict__ out, int64_t count,
                                                       uint64_t seed) {
  const int64_t blocks = (count + 3) / 4;
  const uint2 key = make_uint2(static_cast<uint32_t>(seed), static_cast<uint32_t>(seed >> 32));
  for (int64_t b = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; b < blocks;
       b += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const uint4 r = philox4x32_10(
        make_uint4(static_cast<uint32_t>(b), static_cast<uint32_t>(b >> 32), 0x5356u, 0x44u), key);
    // Box-Muller: u1 in (0, 1], u2 in [0, 1)
    const float u1 = (static_cast<float>(r.x) + 1.0f) * 2.3283064365386963e-10f;
    const float u2 = static_cast<float>(r.y) * 2.3283064365386963e-10f;
    const float u3 = (static_cast<float>(r.z) + 1.0f) * 2.3283064365386963e-10f;
    const float u4 = static_cast<float>(r.w) * 2.3283064365386963e-10f;
    const float ra = sqrtf(-2.0f * logf(fminf(u1, 1.0f)));
    const float rb = sqrtf(-2.0f * logf(fminf(u3, 1.0f)));
    float s1, c1, s2, c2;
    sincospif(2.0f * u2, &s1, &c1);
    sincospif(2.0f * u4, &s2, &c2);
    const float z[4] = {ra * c1, ra * s1, rb * c2, rb * s2};
#pragma unroll
    for (int j = 0; j < 4; ++j)
      if (4 * b + j < count) out[4 * b + j] = z[j];
  }
}

// ------------------------------------------------- tall GEMMs on tcgen05
// Cpart[z] = A[P, Kz] . Bt[L, Kz]^T over the z-th range of K blocks, fp32
// operands read by the tensor core as tf32 (kind::tf32, fp32 accumulation in
// TMEM). Both operands are K-major (row-major with K contiguous): A is [P, K]
// with leading dimension lda, Bt is [L, K] with leading dimension ldb. A CTA
// owns 128 rows of P and all L <= 512 columns (two MMAs per K step when
// L > 256); thread 0 issues the TMA loads (128-byte swizzled boxes of 32 fp32
// along K), thread 32 the MMAs, and the four warps drain TMEM (lane = row).
constexpr int kTgThreads = 128;
constexpr int kTgStages = 4;

struct TgArgs {
  int P, L, Lpad, nkb, ksplit, ptiles, nboxb;
  float* part;       // [ksplit][P][L]
  unsigned* status;
};

__host__ __device__ constexpr int tg_stage_bytes(int Lpad) { return 128 * 128 + Lpad * 128; }

__global__ void __launch_bounds__(kTgThreads, 1)
    tf32_gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                     const TgArgs g) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full[kTgStages], empty[kTgStages], done;
  __shared__ uint32_t tmem_sh;
  __shared__ int abort_sh;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int stage_bytes = tg_stage_bytes(g.Lpad);
  const int ptile = blockIdx.x % g.ptiles, z = blockIdx.x / g.ptiles;
  const int p0 = ptile * 128;
  const int kb_lo = static_cast<int>((static_cast<int64_t>(g.nkb) * z) / g.ksplit);
  const int kb_hi = static_cast<int>((static_cast<int64_t>(g.nkb) * (z + 1)) / g.ksplit);
  const int n = kb_hi - kb_lo;   // >= 1: ksplit <= nkb
  const int n0 = min(g.Lpad, 256), n1 = g.Lpad - n0;
  const uint32_t cols = g.Lpad <= 32 ? 32u : g.Lpad <= 64 ? 64u : g.Lpad <= 128 ? 128u : g.Lpad <= 256 ? 256u : 512u;
  if (tid == 0) {
    for (int s = 0; s < kTgStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(&done, 1);
    fence_mbar_init();
    abort_sh = 0;
  }
  if (warp == 0) {
    tmem_alloc(&tmem_sh, cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_sh;
  const uint32_t bytes = static_cast<uint32_t>(stage_bytes);
  const int boxb = g.Lpad / g.nboxb;
  if (tid == 0) {
    tma_prefetch_desc(&tm_a);
    tma_prefetch_desc(&tm_b);
    for (int i = 0; i < n; ++i) {
      const int s = i % kTgStages;
      if (i >= kTgStages && !mbar_wait(&empty[s], ((i / kTgStages) - 1) & 1, g.status, &abort_sh)) break;
      uint8_t* st = smem + static_cast<size_t>(s) * stage_bytes;
      mbar_arrive_expect_tx(&full[s], bytes);
      const int kc = (kb_lo + i) * 32;
      tma_load_2d(st, &tm_a, &full[s], kc, p0);
      for (int b = 0; b < g.nboxb; ++b)
        tma_load_2d(st + 128 * 128 + b * boxb * 128, &tm_b, &full[s], kc, b * boxb);
    }
  } else if (tid == 32) {
    const uint32_t id0 = idesc_tf32(128, n0), id1 = idesc_tf32(128, n1 > 0 ? n1 : 16);
    bool ok = true;
    for (int i = 0; i < n && ok; ++i) {
      const int s = i % kTgStages;
      ok = mbar_wait(&full[s], (i / kTgStages) & 1, g.status, &abort_sh);
      if (!ok) break;
      tc_fence_after();
      const uint32_t sa = smem_u32(smem + static_cast<size_t>(s) * stage_bytes);
      const uint32_t sb = sa + 128 * 128;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {   // 8 fp32 (32 bytes) of K per MMA
        const uint32_t acc = (i > 0 || kk > 0) ? 1u : 0u;
        mma_tf32(tmem, smem_desc_sw128(sa + kk * 32), smem_desc_sw128(sb + kk * 32), id0, acc);
        if (n1 > 0)
          mma_tf32(tmem + 256, smem_desc_sw128(sa + kk * 32), smem_desc_sw128(sb + 256 * 128 + kk * 32), id1, acc);
      }
      mma_commit(&empty[s]);
    }
    mma_commit(&done);
  }
  __syncwarp();
  const bool ok = mbar_wait_warp(&done, 0, g.status, &abort_sh);
  tc_fence_after();
  const int row = p0 + warp * 32 + lane;
  float* dst = g.part + (static_cast<int64_t>(z) * g.P + row) * g.L;
  for (int c0 = 0; c0 < g.Lpad; c0 += 16) {
    uint32_t v[16];
    tmem_ld_32x32b_x16(tmem + (static_cast<uint32_t>(warp * 32) << 16) + c0, v);
    tmem_ld_wait_regs(v);
    if (ok && row < g.P) {
#pragma unroll
      for (int j = 0; j < 16; ++j)
        if (c0 + j < g.L) dst[c0 + j] = __uint_as_float(v[j]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, cols);
  }
}

__global__ void __launch_bounds__(256) to_f32_kernel(const double* __restrict__ in, int64_t count,
                                                     float* __restrict__ out) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < count;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    out[i] = static_cast<float>(in[i]);
}

__global__ void __launch_bounds__(256) sum_parts_kernel(const float* __restrict__ parts, int nz,
                                                        int64_t count, float* __restrict__ C) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < count;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    float s = 0.0f;
    for (int z = 0; z < nz; ++z) s += parts[static_cast<int64_t>(z) * count + i];
    C[i] = s;
  }
}

__device__ __forceinline__ float block_sum(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  float t = 0.0f;
  for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) t += red[w];
  return t;
}

// Householder QR of A[m, l] (row-major, ld = l) in place: on exit A holds the
// explicit thin Q and, if Rout != nullptr, Rout[l, l] the upper-triangular R.
// CTA g owns rows [g * rpc, (g + 1) * rpc); its rows of the factored matrix
// (R above the diagonal, Householder vectors below) stay in shared memory.
// part: [2][G][lpad] floats of partial sums.
__global__ void __launch_bounds__(kQrThreads, 1)
    householder_qr_kernel(float* __restrict__ A, int m, int l, int rpc, float* __restrict__ Rout,
                          float* __restrict__ part, int lpad, unsigned* counter,
                          unsigned* abort_flag, unsigned* status) {
  extern __shared__ float S[];  // [rpc][lds]
  __shared__ float vhead[kMaxL], beta[kMaxL], alph[kMaxL], wv[kMaxL];
  __shared__ float red[kQrThreads / 32];
  __shared__ int abort_sh;
  const int lds = l | 1;
  const int g = blockIdx.x, G = gridDim.x;
  const int r0 = g * rpc;
  const int nr = max(0, min(m, r0 + rpc) - r0);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, nwarps = kQrThreads / 32;
  GridSync gs{counter, abort_flag, status, 0};
  if (tid == 0) abort_sh = 0;
  for (int e = tid; e < nr * l; e += kQrThreads) {
    const int i = e / l, k = e - i * l;
    S[i * lds + k] = A[static_cast<int64_t>(r0 + i) * l + k];
  }
  __syncthreads();

  float* partA = part;                              // [G][lpad]: column norms and heads
  float* partB = part + static_cast<int64_t>(G) * lpad;  // [G][lpad]: w partials
  bool ok = true;
  for (int j = 0; j < l && ok; ++j) {
    // (1) norm of the part of column j below the diagonal, and its head
    float ss = 0.0f;
    for (int i = tid; i < nr; i += kQrThreads) {
      const int gi = r0 + i;
      if (gi > j) {
        const float v = S[i * lds + j];
        ss = fmaf(v, v, ss);
      }
    }
    ss = block_sum(ss, red);
    if (tid == 0) {
      partA[g * lpad + 0] = ss;
      partA[g * lpad + 1] = (j >= r0 && j < r0 + nr) ? S[(j - r0) * lds + j] : 0.0f;
    }
    ok = grid_sync(gs, &abort_sh);
    if (!ok) break;
    if (tid == 0) {
      float sigma = 0.0f, xj = 0.0f;
      for (int h = 0; h < G; ++h) {
        sigma += partA[h * lpad + 0];
        xj += partA[h * lpad + 1];
      }
      float a, b, vj;
      if (sigma == 0.0f) {
        a = xj;
        b = 0.0f;
        vj = 1.0f;
      } else {
        const float nrm = sqrtf(fmaf(xj, xj, sigma));
        a = xj >= 0.0f ? -nrm : nrm;
        vj = xj - a;
        b = 2.0f / fmaf(vj, vj, sigma);
      }
      alph[j] = a;
      beta[j] = b;
      vhead[j] = vj;
    }
    __syncthreads();
    const float bj = beta[j], vj = vhead[j];
    // (2) partial w_k = sum_{i >= j} v_i S[i][k] for k > j; one warp per column
    for (int k = j + 1 + warp; k < l; k += nwarps) {
      float acc = 0.0f;
      for (int i = lane; i < nr; i += 32) {
        const int gi = r0 + i;
        if (gi >= j) {
          const float vi = gi == j ? vj : S[i * lds + j];
          acc = fmaf(vi, S[i * lds + k], acc);
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      if (lane == 0) partB[g * lpad + k] = acc;
    }
    ok = grid_sync(gs, &abort_sh);
    if (!ok) break;
    for (int k = j + 1 + tid; k < l; k += kQrThreads) {
      float s = 0.0f;
      for (int h = 0; h < G; ++h) s += partB[h * lpad + k];
      wv[k] = s;
    }
    __syncthreads();
    // (3) S[i][k] -= beta v_i w_k for i >= j, k > j
    if (bj != 0.0f) {
      const int w = l - j - 1;
      for (int e = tid; e < nr * w; e += kQrThreads) {
        const int i = e / w, k = j + 1 + (e - i * w);
        const int gi = r0 + i;
        if (gi >= j) {
          const float vi = gi == j ? vj : S[i * lds + j];
          S[i * lds + k] = fmaf(-bj * vi, wv[k], S[i * lds + k]);
        }
      }
    }
    __syncthreads();
  }

  // R factor: rows j < l owned by this CTA
  if (ok && Rout != nullptr) {
    for (int e = tid; e < nr * l; e += kQrThreads) {
      const int i = e / l, k = e - i * l;
      const int gi = r0 + i;
      if (gi < l) Rout[static_cast<int64_t>(gi) * l + k] = k < gi ? 0.0f : (k == gi ? alph[gi] : S[i * lds + k]);
    }
  }

  // Explicit thin Q = H_0 ... H_{l-1} [I; 0], accumulated backwards into A's rows.
  for (int e = tid; e < nr * l; e += kQrThreads) {
    const int i = e / l, c = e - i * l;
    A[static_cast<int64_t>(r0 + i) * l + c] = (r0 + i == c) ? 1.0f : 0.0f;
  }
  __syncthreads();
  for (int j = l - 1; j >= 0 && ok; --j) {
    const float bj = beta[j], vj = vhead[j];
    float* pb = (j & 1) ? partA : partB;
    if (bj != 0.0f) {
      for (int c = j + warp; c < l; c += nwarps) {
        float acc = 0.0f;
        for (int i = lane; i < nr; i += 32) {
          const int gi = r0 + i;
          if (gi >= j) {
            const float vi = gi == j ? vj : S[i * lds + j];
            acc = fmaf(vi, A[static_cast<int64_t>(gi) * l + c], acc);
          }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (lane == 0) pb[g * lpad + c] = acc;
      }
    }
    ok = grid_sync(gs, &abort_sh);
    if (!ok) break;
    if (bj == 0.0f) continue;
    for (int c = j + tid; c < l; c += kQrThreads) {
      float s = 0.0f;
      for (int h = 0; h < G; ++h) s += pb[h * lpad + c];
      wv[c] = s;
    }
    __syncthreads();
    const int w = l - j;
    for (int e = tid; e < nr * w; e += kQrThreads) {
      const int i = e / w, c = j + (e - i * w);
      const int gi = r0 + i;
      if (gi >= j) {
        const float vi = gi == j ? vj : S[i * lds + j];
        float* q = A + static_cast<int64_t>(gi) * l + c;
        *q = fmaf(-bj * vi, wv[c], *q);
      }
    }
    __syncthreads();
  }
}

// ---------------------------------------------- shifted CholeskyQR3 (fp64)
// Orthonormalisation of a tall A[m, l] (l <= kCholMaxL, l % 16 == 0) with no
// grid-wide barrier per column: three passes Q_i = Q_{i-1} R_i^{-1}, R_i the
// upper Cholesky factor of the fp64 Gram matrix Q_{i-1}^T Q_{i-1}, the first
// with the diagonal shift s = 11 (m l + l (l + 1)) u ||A||_F^2 (u = 2^-53) that
// keeps the factorisation defined for any conditioning of A (Fukaya,
// Kannan, Nakatsukasa, Yamamoto & Yanagisawa, "Shifted Cholesky QR for
// computing the QR factorization of ill-conditioned matrices", SIAM J. Sci.
// Comput. 2020; the next two passes are CholeskyQR2). A = Q R, R = R3 R2 R1.
// Each pass: partial Gram matrices of row slices (gram_partial_kernel), their
// sum in slice order (gram_reduce_kernel), the factorisation on one CTA
// (chol_kernel), and the triangular solve of every row (chol_apply_kernel).
constexpr int kCholMaxL = 160;
constexpr int kGramThreads = 512;
constexpr int kGramRows = 64;       // rows of a slice staged in shared memory at a time
constexpr int kCholThreads = 1024;

// part[g] = X[rows of slice g]^T X[rows of slice g], l x l, fp64. Thread t
// accumulates up to two 4 x 4 blocks (bi <= bj) over the slice in registers.
template <typename T>
__global__ void __launch_bounds__(kGramThreads) gram_partial_kernel(const T* __restrict__ X, int m, int l, int rpc,
                                                                    double* __restrict__ part) {
  extern __shared__ double xsm[];   // [kGramRows][l]
  const int tid = threadIdx.x;
  const int r0 = blockIdx.x * rpc, r1 = min(m, r0 + rpc);
  const int nb = l / 4, nblk = nb * (nb + 1) / 2;
  int bi[2], bj[2];
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    int b = tid + q * kGramThreads;
    bi[q] = bj[q] = -1;
    if (b < nblk) {   // b -> (i, j), i <= j, row-major over the upper block triangle
      int i = 0;
      while (b >= nb - i) { b -= nb - i; ++i; }
      bi[q] = i;
      bj[q] = i + b;
    }
  }
  double acc[2][4][4] = {};
  for (int c0 = r0; c0 < r1; c0 += kGramRows) {
    const int nr = min(kGramRows, r1 - c0);
    __syncthreads();
    for (int e = tid; e < nr * l; e += kGramThreads) xsm[e] = static_cast<double>(X[static_cast<int64_t>(c0) * l + e]);
    __syncthreads();
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      if (bi[q] < 0) continue;
      for (int r = 0; r < nr; ++r) {
        const double* xr = xsm + r * l;
        double a[4], c[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          a[u] = xr[4 * bi[q] + u];
          c[u] = xr[4 * bj[q] + u];
        }
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
          for (int v = 0; v < 4; ++v) acc[q][u][v] = fma(a[u], c[v], acc[q][u][v]);
      }
    }
  }
  double* dst = part + static_cast<int64_t>(blockIdx.x) * l * l;
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    if (bi[q] < 0) continue;
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        dst[(4 * bi[q] + u) * l + 4 * bj[q] + v] = acc[q][u][v];
        dst[(4 * bj[q] + v) * l + 4 * bi[q] + u] = acc[q][u][v];
      }
  }
}

// G = sum of the G slices' partial Gram matrices, added in slice order.
__global__ void __launch_bounds__(256) gram_reduce_kernel(const double* __restrict__ part, int G, int64_t ll,
                                                          double* __restrict__ out) {
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < ll;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    double s = 0.0;
    for (int g = 0; g < G; ++g) s += part[g * ll + e];
    out[e] = s;
  }
}

// Upper Cholesky factor R (G = R^T R) of the l x l Gram matrix, right-looking,
// in shared memory; with `shift`, G + s I with s from ||A||_F^2 = trace(G).
// Writes R (zeros below the diagonal) and 1 / R[j][j]; when rtot != nullptr
// also rtot = R rtot (first pass: rtot = R). A non-positive pivot (only
// non-finite input can cause one) records SVDQ_EINVAL.
__global__ void __launch_bounds__(kCholThreads, 1) chol_kernel(const double* __restrict__ Gm, int l, int m, int shift,
                                                               double* __restrict__ R, double* __restrict__ rdiag,
                                                               double* __restrict__ rtot, int first,
                                                               unsigned* status) {
  extern __shared__ double gs[];   // [l][l]
  __shared__ double red[kCholThreads / 32];
  const int tid = threadIdx.x;
  for (int e = tid; e < l * l; e += kCholThreads) gs[e] = Gm[e];
  __syncthreads();
  if (shift) {
    double t = 0.0;
    for (int i = tid; i < l; i += kCholThreads) t += gs[i * l + i];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
    if ((tid & 31) == 0) red[tid >> 5] = t;
    __syncthreads();
    if (tid == 0) {
      double tr = 0.0;
      for (int w = 0; w < kCholThreads / 32; ++w) tr += red[w];
      red[0] = 11.0 * (static_cast<double>(m) * l + static_cast<double>(l) * (l + 1)) * 0x1p-53 * tr;
    }
    __syncthreads();
    const double sh = red[0];
    for (int i = tid; i < l; i += kCholThreads) gs[i * l + i] += sh;
    __syncthreads();
  }
  for (int j = 0; j < l; ++j) {
    if (tid == 0) {
      double d = gs[j * l + j];
      if (!(d > 0.0) || !(d <= 1.7976931348623157e308)) {
        record_status(status, kStatusEinval);
        d = 1.0;
      }
      gs[j * l + j] = sqrt(d);
    }
    __syncthreads();
    const double dj = gs[j * l + j];
    for (int k = j + 1 + tid; k < l; k += kCholThreads) gs[j * l + k] /= dj;
    __syncthreads();
    const int w = l - j - 1;
    for (int e = tid; e < w * w; e += kCholThreads) {
      const int i = j + 1 + e / w, k = j + 1 + e % w;
      if (k >= i) gs[i * l + k] = fma(-gs[j * l + i], gs[j * l + k], gs[i * l + k]);
    }
    __syncthreads();
  }
  for (int e = tid; e < l * l; e += kCholThreads) {
    const int i = e / l, k = e % l;
    R[e] = k >= i ? gs[e] : 0.0;
  }
  for (int i = tid; i < l; i += kCholThreads) rdiag[i] = 1.0 / gs[i * l + i];
  if (rtot != nullptr) {
    if (first) {
      for (int e = tid; e < l * l; e += kCholThreads) rtot[e] = (e % l) >= (e / l) ? gs[e] : 0.0;
    } else {
      // row i of R rtot needs rows j >= i of the old rtot: rows in increasing order
      for (int i = 0; i < l; ++i) {
        __syncthreads();
        double v = 0.0;
        const int k = i + tid;
        if (k < l)
          for (int j = i; j <= k; ++j) v = fma(gs[i * l + j], rtot[j * l + k], v);
        __syncthreads();
        if (k < l) rtot[i * l + k] = v;
      }
    }
  }
}

// Q = X R^{-1} row by row (x = q R, R upper): one warp per row, lane owns the
// columns lane + 32 t; step j takes q_j = x_j / R[j][j] from its owner and
// removes q_j R[j][k] from the later columns. kFinal: fp32 Q [m, l] and its
// transpose Qt [l, m]; else fp64 Qd [m, l] (may be X itself).
template <typename Tin, bool kFinal>
__global__ void __launch_bounds__(kCholThreads, 1) chol_apply_kernel(const Tin* X, int m, int l,
                                                                     const double* __restrict__ R,
                                                                     const double* __restrict__ rdiag, double* Qd,
                                                                     float* __restrict__ Q, float* __restrict__ Qt) {
  constexpr int kT = kCholMaxL / 32;
  extern __shared__ double rs[];   // [l][l] then rdiag[l]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int e = tid; e < l * l; e += kCholThreads) rs[e] = R[e];
  for (int e = tid; e < l; e += kCholThreads) rs[l * l + e] = rdiag[e];
  __syncthreads();
  const double* rd = rs + l * l;
  for (int row = blockIdx.x * (kCholThreads / 32) + warp; row < m; row += gridDim.x * (kCholThreads / 32)) {
    double x[kT];
#pragma unroll
    for (int t = 0; t < kT; ++t) {
      const int k = lane + 32 * t;
      x[t] = k < l ? static_cast<double>(X[static_cast<int64_t>(row) * l + k]) : 0.0;
    }
#pragma unroll
    for (int jb = 0; jb < kT; ++jb) {
      if (jb * 32 >= l) break;
      for (int jj = 0; jj < 32; ++jj) {
        const int j = jb * 32 + jj;
        if (j >= l) break;   // uniform across the warp: l need not be a multiple of 32
        const double qj = __shfl_sync(0xffffffffu, x[jb], jj) * rd[j];
        if (lane == jj) x[jb] = qj;
#pragma unroll
        for (int t = jb; t < kT; ++t) {
          const int k = lane + 32 * t;
          if (k > j && k < l) x[t] = fma(-qj, rs[j * l + k], x[t]);
        }
      }
    }
#pragma unroll
    for (int t = 0; t < kT; ++t) {
      const int k = lane + 32 * t;
      if (k < l) {
        if constexpr (kFinal) {
          Q[static_cast<int64_t>(row) * l + k] = static_cast<float>(x[t]);
          Qt[static_cast<int64_t>(k) * m + row] = static_cast<float>(x[t]);
        } else {
          Qd[static_cast<int64_t>(row) * l + k] = x[t];
        }
      }
    }
  }
}

// out[c][r] = in[r][c] for in [rows, cols] (fp32), 32 x 32 tiles.
__global__ void __launch_bounds__(256) transpose_kernel(const float* __restrict__ in, int64_t rows, int64_t cols,
                                                        float* __restrict__ out) {
  __shared__ float t[32][33];
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  const int64_t tr = (rows + 31) / 32, tc = (cols + 31) / 32;
  for (int64_t tile = blockIdx.x; tile < tr * tc; tile += gridDim.x) {
    const int64_t r0 = (tile / tc) * 32, c0 = (tile % tc) * 32;
    __syncthreads();
    for (int i = ty; i < 32; i += 8)
      if (r0 + i < rows && c0 + tx < cols) t[i][tx] = in[(r0 + i) * cols + c0 + tx];
    __syncthreads();
    for (int i = ty; i < 32; i += 8)
      if (c0 + i < cols && r0 + tx < rows) out[(c0 + i) * rows + r0 + tx] = t[tx][i];
  }
}

// -------------------------------------------------- one-sided Jacobi SVD
// X[n x n] (column-major, fp64, in global memory) is rotated in place until its
// columns are orthogonal; J accumulates the rotations. Parallel round-robin
// ordering: in each of the n-1 rounds of a sweep the n/2 column pairs are
// disjoint, one warp per pair. Then sigma_i = |X[:, i]|, U = X / sigma, V = J,
// sorted by decreasing sigma; the first r columns are written out (fp32) as the
// rows of UrT [r, l] and VrT [r, l] (the K-major operands of the next GEMMs).
__global__ void __launch_bounds__(1024, 1)
    jacobi_svd_kernel(const float* __restrict__ Rb, int l, int n, double* __restrict__ X,
                      double* __restrict__ J, int r, float* __restrict__ Ur,
                      float* __restrict__ Vr, float* __restrict__ sig, int max_sweeps) {
  __shared__ int rotated;
  __shared__ int perm[kMaxL + 1];
  __shared__ double norms[kMaxL + 1];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, nwarps = blockDim.x >> 5;
  // X = Rb^T padded to n (even) with zeros; J = I
  for (int e = tid; e < n * n; e += blockDim.x) {
    const int col = e / n, row = e - col * n;  // X[row, col] = Rb[col, row]
    X[e] = (row < l && col < l) ? static_cast<double>(Rb[static_cast<int64_t>(col) * l + row]) : 0.0;
    J[e] = row == col ? 1.0 : 0.0;
  }
  __syncthreads();
  for (int sweep = 0; sweep < max_sweeps; ++sweep) {
    if (tid == 0) rotated = 0;
    __syncthreads();
    for (int round = 0; round < n - 1; ++round) {
      for (int pi = warp; pi < n / 2; pi += nwarps) {
        // round-robin pairing: slot 0 fixed, the others rotate
        auto slot = [&](int s) { return s == 0 ? 0 : 1 + (s - 1 + round) % (n - 1); };
        int p = slot(pi), q = slot(n - 1 - pi);
        if (p > q) { const int t = p; p = q; q = t; }
        double a = 0.0, b = 0.0, c = 0.0;
        for (int i = lane; i < n; i += 32) {
          const double xp = X[static_cast<int64_t>(p) * n + i], xq = X[static_cast<int64_t>(q) * n + i];
          a += xp * xp;
          b += xq * xq;
          c += xp * xq;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          a += __shfl_xor_sync(0xffffffffu, a, o);
          b += __shfl_xor_sync(0xffffffffu, b, o);
          c += __shfl_xor_sync(0xffffffffu, c, o);
        }
        if (c != 0.0 && fabs(c) > 1e-15 * sqrt(a * b)) {
          const double zeta = (b - a) / (2.0 * c);
          const double t = (zeta >= 0.0 ? 1.0 : -1.0) / (fabs(zeta) + sqrt(1.0 + zeta * zeta));
          const double cs = 1.0 / sqrt(1.0 + t * t), sn = cs * t;
          for (int i = lane; i < n; i += 32) {
            double* xp = X + static_cast<int64_t>(p) * n + i;
            double* xq = X + static_cast<int64_t>(q) * n + i;
            const double u = *xp, v = *xq;
            *xp = cs * u - sn * v;
            *xq = sn * u + cs * v;
            double* jp = J + static_cast<int64_t>(p) * n + i;
            double* jq = J + static_cast<int64_t>(q) * n + i;
            const double ju = *jp, jv = *jq;
            *jp = cs * ju - sn * jv;
            *jq = sn * ju + cs * jv;
          }
          if (lane == 0) rotated = 1;
        }
        __syncwarp();
      }
      __syncthreads();
    }
    const int any = rotated;  // read by every thread before thread 0 may reset it
    __syncthreads();
    if (!any) break;
  }
  // singular values and ordering
  for (int col = warp; col < n; col += nwarps) {
    double s = 0.0;
    for (int i = lane; i < n; i += 32) {
      const double v = X[static_cast<int64_t>(col) * n + i];
      s += v * v;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) norms[col] = sqrt(s);
  }
  __syncthreads();
  if (tid == 0) {
    for (int i = 0; i < n; ++i) perm[i] = i;
    for (int i = 1; i < n; ++i) {  // insertion sort, decreasing
      const int pv = perm[i];
      int k = i - 1;
      while (k >= 0 && norms[perm[k]] < norms[pv]) {
        perm[k + 1] = perm[k];
        --k;
      }
      perm[k + 1] = pv;
    }
  }
  __syncthreads();
  for (int e = tid; e < l * r; e += blockDim.x) {
    const int k = e / l, i = e - k * l;  // row k of the r x l (transposed) outputs
    const int col = perm[k];
    const double s = norms[col];
    Ur[e] = s > 0.0 ? static_cast<float>(X[static_cast<int64_t>(col) * n + i] / s) : 0.0f;
    Vr[e] = static_cast<float>(J[static_cast<int64_t>(col) * n + i]);
  }
  for (int k = tid; k < r; k += blockDim.x) sig[k] = static_cast<float>(norms[perm[k]]);
}

// ld[j, m] = bf16(U[m, j] sigma_j / scale[m]); lu[n, j] = lu[n, rp + j] = bf16(V[n, j])
__global__ void __launch_bounds__(256) factor_finalize_kernel(
    const float* __restrict__ U, const float* __restrict__ V, const float* __restrict__ sig,
    const float* __restrict__ scale, int64_t M, int64_t N, int r, int rp,
    __nv_bfloat16* __restrict__ ld, float* __restrict__ ld32, __nv_bfloat16* __restrict__ lu) {
  const int64_t tl = static_cast<int64_t>(rp) * M;
  const int64_t tu = N * rp;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < tl + tu;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    if (i < tl) {
      const int64_t j = i / M, m = i - j * M;
      float v = 0.0f;
      if (j < r) v = __fdiv_rn(__fmul_rn(U[m * r + j], sig[j]), scale[m]);
      const __nv_bfloat16 b = __float2bfloat16_rn(v);
      ld[i] = b;
      if (ld32) ld32[i] = __bfloat162float(b);
    } else {
      const int64_t e = i - tl;
      const int64_t n = e / rp, j = e - n * rp;
      const __nv_bfloat16 b = __float2bfloat16_rn(j < r ? V[n * r + j] : 0.0f);
      lu[n * 2 * rp + j] = b;
      lu[n * 2 * rp + rp + j] = b;
    }
  }
}

// R[m, n] = ws[m, n] - scale[m] * sum_j ld[j, m] lu[n, j]   (in place over ws)
__global__ void __launch_bounds__(256) residual_kernel(float* __restrict__ ws,
                                                       const float* __restrict__ scale,
                                                       const __nv_bfloat16* __restrict__ ld,
                                                       const __nv_bfloat16* __restrict__ lu,
                                                       int64_t M, int64_t N, int r, int rp) {
  __shared__ float Ls[32][65];  // [j][m]
  __shared__ float Us[32][65];  // [j][n]
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int64_t m0 = static_cast<int64_t>(blockIdx.y) * 64, n0 = static_cast<int64_t>(blockIdx.x) * 64;
  float acc[4][4] = {};
  for (int j0 = 0; j0 < r; j0 += 32) {
    for (int e = threadIdx.x; e < 32 * 64; e += 256) {
      const int jj = e >> 6, c = e & 63;
      const int j = j0 + jj;
      Ls[jj][c] = (j < r && m0 + c < M) ? __bfloat162float(ld[static_cast<int64_t>(j) * M + m0 + c]) : 0.0f;
      Us[jj][c] = (j < r && n0 + c < N) ? __bfloat162float(lu[(n0 + c) * 2 * rp + j]) : 0.0f;
    }
    __syncthreads();
#pragma unroll 8
    for (int jj = 0; jj < 32; ++jj) {
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) acc[a][b] = fmaf(Ls[jj][ty * 4 + a], Us[jj][tx * 4 + b], acc[a][b]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const int64_t m = m0 + ty * 4 + a;
    if (m >= M) continue;
    const float s = scale[m];
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const int64_t n = n0 + tx * 4 + b;
      if (n < N) ws[m * N + n] = ws[m * N + n] - __fmul_rn(s, acc[a][b]);
    }
  }
}

int grid_for(int64_t work, int per_block = 256) {
  return static_cast<int>(std::max<int64_t>(
      1, std::min<int64_t>(ceil_div(work, per_block), static_cast<int64_t>(num_sms()) * 16)));
}

int choose_l(int64_t M, int64_t N, int r, int p) {
  // a multiple of 16 (the MMA's N and 64-byte rows for the TMA); M and N are
  // multiples of 16, so the cap keeps that
  return static_cast<int>(std::min<int64_t>({round_up(static_cast<int64_t>(r) + p, 16), M, N}));
}

struct TgPlan {
  int ptiles, ksplit, nkb, Lpad, nboxb;
  size_t smem;
  int64_t part_floats;
};

TgPlan plan_tgemm(int64_t P, int64_t K, int64_t L) {
  TgPlan t{};
  t.ptiles = static_cast<int>(ceil_div(P, 128));
  t.nkb = static_cast<int>(ceil_div(K, 32));
  t.ksplit = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(t.nkb, ceil_div(2 * num_sms(), t.ptiles))));
  t.Lpad = static_cast<int>(round_up(L, 16));
  t.nboxb = t.Lpad > 256 ? 2 : 1;
  t.smem = static_cast<size_t>(kTgStages) * tg_stage_bytes(t.Lpad) + 1024;
  t.part_floats = static_cast<int64_t>(t.ksplit) * P * L;
  return t;
}

// C[P, L] = A[P, K] Bt[L, K]^T on the tensor core (tf32), split over K and
// summed in split order. lda, ldb in elements (multiples of 4); L <= 512.
cudaError_t run_tgemm(const float* A, int64_t lda, const float* Bt, int64_t ldb, int64_t P, int64_t K, int64_t L,
                      float* part, float* C, unsigned* status, cudaStream_t st) {
  const TgPlan t = plan_tgemm(P, K, L);
  CUtensorMap ta, tb;
  if (!make_tmap_2d(&ta, A, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, K, P, lda, 32, 128, true) ||
      !make_tmap_2d(&tb, Bt, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, K, L, ldb, 32, t.Lpad / t.nboxb, true))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(tf32_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(t.smem));
  if (e != cudaSuccess) return e;
  TgArgs g{};
  g.P = static_cast<int>(P);
  g.L = static_cast<int>(L);
  g.Lpad = t.Lpad;
  g.nkb = t.nkb;
  g.ksplit = t.ksplit;
  g.ptiles = t.ptiles;
  g.nboxb = t.nboxb;
  g.part = part;
  g.status = status;
  tf32_gemm_kernel<<<t.ptiles * t.ksplit, kTgThreads, t.smem, st>>>(ta, tb, g);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int64_t cnt = P * L;
  sum_parts_kernel<<<grid_for(cnt), 256, 0, st>>>(part, t.ksplit, cnt, C);
  return cudaGetLastError();
}

struct QrPlan {
  int G, rpc;
  size_t smem;
};

QrPlan plan_qr(int64_t m, int l) {
  QrPlan q{};
  const int min_rows = 8;
  q.G = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(num_sms(), ceil_div(m, min_rows))));
  q.rpc = static_cast<int>(ceil_div(m, q.G));
  q.G = static_cast<int>(ceil_div(m, q.rpc));
  q.smem = static_cast<size_t>(q.rpc) * (l | 1) * sizeof(float);
  return q;
}

cudaError_t run_householder(float* A, int64_t m, int l, float* Rout, float* part, int lpad, unsigned* sync,
                            unsigned* status, cudaStream_t st) {
  const QrPlan q = plan_qr(m, l);
  cudaError_t e = cudaMemsetAsync(sync, 0, 2 * sizeof(unsigned), st);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(householder_qr_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(q.smem));
  if (e != cudaSuccess) return e;
  int mi = static_cast<int>(m), li = l, rpc = q.rpc;
  unsigned* counter = sync;
  unsigned* abort_flag = sync + 1;
  void* args[] = {&A, &mi, &li, &rpc, &Rout, &part, &lpad, &counter, &abort_flag, &status};
  return cudaLaunchCooperativeKernel(reinterpret_cast<void*>(householder_qr_kernel), dim3(q.G),
                                     dim3(kQrThreads), args, q.smem, st);
}

// Slices of the Gram kernels: about two per SM, rows per slice a multiple of 16.
int gram_slices(int64_t m) {
  const int64_t rpc = std::max<int64_t>(16, round_up(ceil_div(m, 2 * num_sms()), 16));
  return static_cast<int>(ceil_div(m, rpc));
}

struct QrScratch {
  double* Qd;     // [m, l]
  double* gpart;  // [slices][l][l]
  double* G;      // [l][l]
  double* R;      // [l][l]
  double* rdiag;  // [l]
  double* rtot;   // [l][l]
  float* hpart;   // Householder partial sums [2][G][lpad]
  unsigned* sync;
};

// Thin QR of A[m, l] (fp32, row-major): Q overwrites A and its transpose goes
// to At [l, m]; Rout [l, l] (nullable) receives R. Shifted CholeskyQR3 for
// l <= kCholMaxL, the Householder kernel above that.
cudaError_t run_qr(float* A, float* At, int64_t m, int l, float* Rout, const QrScratch& q, unsigned* status,
                   cudaStream_t st) {
  cudaError_t e;
  if (l > kCholMaxL) {
    const int lpad = (l + 2 + 3) / 4 * 4;
    e = run_householder(A, m, l, Rout, q.hpart, lpad, q.sync, status, st);
    if (e != cudaSuccess) return e;
    transpose_kernel<<<grid_for(ceil_div(m, 32) * ceil_div(l, 32), 1), 256, 0, st>>>(A, m, l, At);
    return cudaGetLastError();
  }
  const int mi = static_cast<int>(m);
  const int S = gram_slices(m);
  const int rpc = static_cast<int>(ceil_div(m, S));
  const int64_t ll = static_cast<int64_t>(l) * l;
  const size_t gsm = static_cast<size_t>(kGramRows) * l * sizeof(double);
  const size_t csm = static_cast<size_t>(ll) * sizeof(double);
  const size_t asm_ = csm + static_cast<size_t>(l) * sizeof(double);
  for (auto fn : {reinterpret_cast<const void*>(gram_partial_kernel<float>),
                  reinterpret_cast<const void*>(gram_partial_kernel<double>)}) {
    e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(gsm));
    if (e != cudaSuccess) return e;
  }
  e = cudaFuncSetAttribute(chol_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(csm));
  if (e != cudaSuccess) return e;
  for (auto fn : {reinterpret_cast<const void*>(chol_apply_kernel<float, false>),
                  reinterpret_cast<const void*>(chol_apply_kernel<double, false>),
                  reinterpret_cast<const void*>(chol_apply_kernel<double, true>)}) {
    e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(asm_));
    if (e != cudaSuccess) return e;
  }
  const int agrid = static_cast<int>(std::min<int64_t>(num_sms(), ceil_div(m, kCholThreads / 32)));
  for (int pass = 0; pass < 3; ++pass) {
    if (pass == 0)
      gram_partial_kernel<float><<<S, kGramThreads, gsm, st>>>(A, mi, l, rpc, q.gpart);
    else
      gram_partial_kernel<double><<<S, kGramThreads, gsm, st>>>(q.Qd, mi, l, rpc, q.gpart);
    gram_reduce_kernel<<<grid_for(ll), 256, 0, st>>>(q.gpart, S, ll, q.G);
    chol_kernel<<<1, kCholThreads, csm, st>>>(q.G, l, mi, pass == 0 ? 1 : 0, q.R, q.rdiag,
                                               Rout != nullptr ? q.rtot : nullptr, pass == 0 ? 1 : 0, status);
    if (pass == 0)
      chol_apply_kernel<float, false><<<agrid, kCholThreads, asm_, st>>>(A, mi, l, q.R, q.rdiag, q.Qd, nullptr,
                                                                         nullptr);
    else if (pass == 1)
      chol_apply_kernel<double, false><<<agrid, kCholThreads, asm_, st>>>(q.Qd, mi, l, q.R, q.rdiag, q.Qd,
                                                                          nullptr, nullptr);
    else
      chol_apply_kernel<double, true><<<agrid, kCholThreads, asm_, st>>>(q.Qd, mi, l, q.R, q.rdiag, nullptr, A,
                                                                         At);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (Rout != nullptr) {
    to_f32_kernel<<<grid_for(ll), 256, 0, st>>>(q.rtot, ll, Rout);
    e = cudaGetLastError();
  }
  return e;
}

struct PrepCarve {
  float* ws;      // [M, N]
  float* wsT;     // [N, M]
  float* omegaT;  // [l, N]
  float* Y;       // [M, l]
  float* Yt;      // [l, M]
  float* Z;       // [N, l]
  float* Zt;      // [l, N]
  float* Rb;      // [l, l]
  double* X;      // [n, n]
  double* J;      // [n, n]
  float* UrT;     // [r, l]
  float* VrT;     // [r, l]
  float* sig;     // [r]
  float* U;       // [M, r]
  float* V;       // [N, r]
  float* gpart;   // GEMM split-K partials
  QrScratch qr;
  void* qscratch; // residual quantiser scratch
  size_t bytes;
  bool ok;
};

PrepCarve carve_prepare(int64_t M, int64_t N, int r, int p, void* base, size_t cap) {
  const int l = r > 0 ? choose_l(M, N, r, p) : 0;
  const int n = (l + 1) / 2 * 2;
  Carver cv(base, cap);
  PrepCarve c{};
  c.ws = static_cast<float*>(cv.take(static_cast<size_t>(M * N) * 4));
  if (r > 0) {
    c.wsT = static_cast<float*>(cv.take(static_cast<size_t>(M * N) * 4));
    c.omegaT = static_cast<float*>(cv.take(static_cast<size_t>(N) * l * 4));
    c.Y = static_cast<float*>(cv.take(static_cast<size_t>(M) * l * 4));
    c.Yt = static_cast<float*>(cv.take(static_cast<size_t>(M) * l * 4));
    c.Z = static_cast<float*>(cv.take(static_cast<size_t>(N) * l * 4));
    c.Zt = static_cast<float*>(cv.take(static_cast<size_t>(N) * l * 4));
    c.Rb = static_cast<float*>(cv.take(static_cast<size_t>(l) * l * 4));
    c.X = static_cast<double*>(cv.take(static_cast<size_t>(n) * n * 8));
    c.J = static_cast<double*>(cv.take(static_cast<size_t>(n) * n * 8));
    c.UrT = static_cast<float*>(cv.take(static_cast<size_t>(l) * r * 4));
    c.VrT = static_cast<float*>(cv.take(static_cast<size_t>(l) * r * 4));
    c.sig = static_cast<float*>(cv.take(static_cast<size_t>(r) * 4));
    c.U = static_cast<float*>(cv.take(static_cast<size_t>(M) * r * 4));
    c.V = static_cast<float*>(cv.take(static_cast<size_t>(N) * r * 4));
    const int64_t gp = std::max({plan_tgemm(M, N, l).part_floats, plan_tgemm(N, M, l).part_floats,
                                 plan_tgemm(M, l, r).part_floats, plan_tgemm(N, l, r).part_floats});
    c.gpart = static_cast<float*>(cv.take(static_cast<size_t>(gp) * 4));
    const int64_t mx = std::max(M, N);
    const int64_t ll = static_cast<int64_t>(l) * l;
    c.qr.Qd = static_cast<double*>(cv.take(static_cast<size_t>(mx) * l * 8));
    c.qr.gpart = static_cast<double*>(cv.take(static_cast<size_t>(std::max(gram_slices(M), gram_slices(N))) * ll * 8));
    c.qr.G = static_cast<double*>(cv.take(static_cast<size_t>(ll) * 8));
    c.qr.R = static_cast<double*>(cv.take(static_cast<size_t>(ll) * 8));
    c.qr.rdiag = static_cast<double*>(cv.take(static_cast<size_t>(l) * 8));
    c.qr.rtot = static_cast<double*>(cv.take(static_cast<size_t>(ll) * 8));
    const int lpad = (l + 2 + 3) / 4 * 4;
    const int G = std::max(plan_qr(M, l).G, plan_qr(N, l).G);
    c.qr.hpart = static_cast<float*>(cv.take(static_cast<size_t>(2) * G * lpad * 4));
    c.qr.sync = static_cast<unsigned*>(cv.take(64));
  }
  c.qscratch = cv.take(residual_scratch_bytes(M, N));
  c.bytes = cv.off;
  c.ok = cv.ok;
  return c;
}

}  // namespace

size_t prepare_scratch_bytes(int64_t M, int64_t N, int32_t rank, int32_t oversample) {
  const int p = oversample > 0 ? oversample : kDefaultOversample;
  return carve_prepare(M, N, rank, p, nullptr, 0).bytes + 256;
}

svdq_status run_prepare(const void* W, svdq_dtype wdt, int64_t M, int64_t N, int64_t ldW,
                        const float* scale, int32_t rank, svdq_fmt fmt, uint64_t seed,
                        int32_t oversample, int32_t power_iters, void* workspace,
                        size_t ws_bytes, svdq_weight* out, cudaStream_t st) {
  const int p = oversample > 0 ? oversample : kDefaultOversample;
  const int q = power_iters > 0 ? power_iters : kDefaultPowerIters;
  const int r = rank;
  const int rp = rank_pad_of(rank);
  PrepCarve c = carve_prepare(M, N, r, p, workspace, ws_bytes);
  if (!c.ok) return SVDQ_EWORKSPACE;
  const int l = r > 0 ? choose_l(M, N, r, p) : 0;
  if (l > kMaxL) return SVDQ_EUNSUPPORTED;
  if (r > 0 && l > kCholMaxL) {
    // the Householder kernel's row slices must fit in shared memory
    const size_t smem_cap = 200 * 1024;
    if (plan_qr(M, l).smem > smem_cap || plan_qr(N, l).smem > smem_cap) return SVDQ_EUNSUPPORTED;
  }
  unsigned* status = device_status_word();
  if (!status) return SVDQ_ECUDA;
  // clear a stale status word so this call reports only its own errors
  if (cudaMemsetAsync(status, 0, sizeof(unsigned), st) != cudaSuccess) return SVDQ_ECUDA;

  out->M = M;
  out->N = N;
  out->rank = r;
  out->rank_pad = rp;
  out->fmt = fmt;
  out->scale = scale;

  const int64_t total = M * N;
  if (wdt == SVDQ_BF16)
    smooth_weight_kernel<__nv_bfloat16><<<grid_for(total), 256, 0, st>>>(
        static_cast<const __nv_bfloat16*>(W), ldW, scale, M, N, c.ws, status);
  else
    smooth_weight_kernel<float><<<grid_for(total), 256, 0, st>>>(static_cast<const float*>(W), ldW,
                                                                 scale, M, N, c.ws, status);
  if (cudaGetLastError() != cudaSuccess) return SVDQ_ECUDA;

  if (r > 0) {
    const int n = (l + 1) / 2 * 2;
    auto chk = [](cudaError_t e) { return e == cudaSuccess; };
    bool ok = true;
    // ws^T, the A operand of the products with ws^T
    transpose_kernel<<<grid_for(ceil_div(M, 32) * ceil_div(N, 32), 1), 256, 0, st>>>(c.ws, M, N, c.wsT);
    ok = ok && chk(cudaGetLastError());
    gaussian_kernel<<<grid_for(ceil_div(N * l, 4)), 256, 0, st>>>(c.omegaT, N * l, seed);   // Omega^T [l, N]
    ok = ok && chk(cudaGetLastError());
    ok = ok && chk(run_tgemm(c.ws, N, c.omegaT, N, M, N, l, c.gpart, c.Y, status, st));   // Y = ws Omega
    ok = ok && chk(run_qr(c.Y, c.Yt, M, l, nullptr, c.qr, status, st));                  // Q = orth(Y)
    for (int it = 0; it < q && ok; ++it) {
      ok = ok && chk(run_tgemm(c.wsT, M, c.Yt, M, N, M, l, c.gpart, c.Z, status, st));    // Z = ws^T Q
      ok = ok && chk(run_qr(c.Z, c.Zt, N, l, nullptr, c.qr, status, st));
      ok = ok && chk(run_tgemm(c.ws, N, c.Zt, N, M, N, l, c.gpart, c.Y, status, st));     // Y = ws Z
      ok = ok && chk(run_qr(c.Y, c.Yt, M, l, nullptr, c.qr, status, st));
    }
    ok = ok && chk(run_tgemm(c.wsT, M, c.Yt, M, N, M, l, c.gpart, c.Z, status, st));      // Bt = ws^T Q
    ok = ok && chk(run_qr(c.Z, c.Zt, N, l, c.Rb, c.qr, status, st));                     // Bt = Qb Rb
    jacobi_svd_kernel<<<1, 1024, 0, st>>>(c.Rb, l, n, c.X, c.J, r, c.UrT, c.VrT, c.sig, 40);
    ok = ok && chk(cudaGetLastError());
    ok = ok && chk(run_tgemm(c.Y, l, c.UrT, l, M, l, r, c.gpart, c.U, status, st));      // U = Q Ur
    ok = ok && chk(run_tgemm(c.Z, l, c.VrT, l, N, l, r, c.gpart, c.V, status, st));      // V = Qb Vr
    factor_finalize_kernel<<<grid_for(static_cast<int64_t>(rp) * (M + N)), 256, 0, st>>>(
        c.U, c.V, c.sig, scale, M, N, r, rp, static_cast<__nv_bfloat16*>(out->ld),
        static_cast<float*>(out->ld32), static_cast<__nv_bfloat16*>(out->lu));
    ok = ok && chk(cudaGetLastError());
    dim3 rg(static_cast<unsigned>(ceil_div(N, 64)), static_cast<unsigned>(ceil_div(M, 64)));
    residual_kernel<<<rg, 256, 0, st>>>(c.ws, scale, static_cast<const __nv_bfloat16*>(out->ld),
                                        static_cast<const __nv_bfloat16*>(out->lu), M, N, r, rp);
    ok = ok && chk(cudaGetLastError());
    if (!ok) return SVDQ_ECUDA;
  }
  if (launch_quantize_residual(c.ws, M, N, N, fmt, out->codes, out->sf, out->w_scale, c.qscratch,
                               st) != cudaSuccess)
    return SVDQ_ECUDA;
  if (out->codes4 && fmt.kind == SVDQ_KIND_INT && fmt.bits <= 4 &&
      launch_pack_int4(static_cast<const int8_t*>(out->codes), N, M, static_cast<uint8_t*>(out->codes4),
                       st) != cudaSuccess)
    return SVDQ_ECUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return SVDQ_ECUDA;
  unsigned v = 0;
  if (cudaMemcpy(&v, status, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return SVDQ_ECUDA;
  if (v != 0) {
    const unsigned zero = 0;
    cudaMemcpy(status, &zero, sizeof(zero), cudaMemcpyHostToDevice);
    return static_cast<svdq_status>(v);
  }
  return SVDQ_OK;
}

}  // namespace svdq
