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

// ------------------------------------------------------- tall-skinny SGEMM
// Cpart[z] = op(A)[P, Kz] . B[Kz, L] over the z-th K chunk; op(A)[p, k] is
// A[p * lda + k] (TRANS = false) or A[k * lda + p] (TRANS = true). B is [K, L].
template <bool TRANS>
__global__ void __launch_bounds__(256) sgemm_kernel(const float* __restrict__ A, int64_t lda,
                                                    const float* __restrict__ Bm, int64_t P,
                                                    int64_t K, int64_t L, int64_t kchunk,
                                                    float* __restrict__ Cpart) {
  __shared__ float As[16][64 + 4];
  __shared__ float Bs[16][64 + 4];
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;
  const int64_t p0 = static_cast<int64_t>(blockIdx.x) * 64;
  const int64_t l0 = static_cast<int64_t>(blockIdx.y) * 64;
  const int64_t kbeg = static_cast<int64_t>(blockIdx.z) * kchunk;
  const int64_t kend = K < kbeg + kchunk ? K : kbeg + kchunk;
  float acc[4][4] = {};
  for (int64_t k0 = kbeg; k0 < kend; k0 += 16) {
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const int e = tid + 256 * t;
      int kk, pp;
      if (TRANS) {
        pp = e & 63;
        kk = e >> 6;
      } else {
        kk = e & 15;
        pp = e >> 4;
      }
      const int64_t p = p0 + pp, k = k0 + kk;
      float v = 0.0f;
      if (p < P && k < kend) v = TRANS ? A[k * lda + p] : A[p * lda + k];
      As[kk][pp] = v;
      const int ll = e & 63, kb = e >> 6;
      const int64_t l = l0 + ll, kb2 = k0 + kb;
      Bs[kb][ll] = (l < L && kb2 < kend) ? Bm[kb2 * L + l] : 0.0f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
  float* C = Cpart + static_cast<int64_t>(blockIdx.z) * P * L;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t p = p0 + ty * 4 + i;
    if (p >= P) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t l = l0 + tx * 4 + j;
      if (l < L) C[p * L + l] = acc[i][j];
    }
  }
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

// -------------------------------------------------- one-sided Jacobi SVD
// X[n x n] (column-major, fp64, in global memory) is rotated in place until its
// columns are orthogonal; J accumulates the rotations. Parallel round-robin
// ordering: in each of the n-1 rounds of a sweep the n/2 column pairs are
// disjoint, one warp per pair. Then sigma_i = |X[:, i]|, U = X / sigma, V = J,
// sorted by decreasing sigma; the first r columns are written out (fp32).
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
    const int i = e / r, k = e - i * r;  // row i of the l x r outputs
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

struct Dims {
  int64_t M, N;
  int r, rp, l, n_even, qr_grid_max;
  int64_t gemm_part_floats;
};

int choose_l(int64_t M, int64_t N, int r, int p) {
  return static_cast<int>(std::min<int64_t>({static_cast<int64_t>(r) + p, M, N}));
}

int64_t gemm_ksplit(int64_t P, int64_t K, int64_t L) {
  const int64_t tiles = ceil_div(P, 64) * ceil_div(L, 64);
  int64_t ks = ceil_div(2 * num_sms(), tiles);
  return std::max<int64_t>(1, std::min<int64_t>(ks, ceil_div(K, 64)));
}

int64_t gemm_part_floats(int64_t P, int64_t K, int64_t L) { return gemm_ksplit(P, K, L) * P * L; }

cudaError_t run_gemm(bool trans, const float* A, int64_t lda, const float* Bm, int64_t P, int64_t K,
                     int64_t L, float* part, float* C, cudaStream_t st) {
  const int64_t ks = gemm_ksplit(P, K, L);
  const int64_t kchunk = round_up(ceil_div(K, ks), 16);
  const int64_t nz = ceil_div(K, kchunk);
  dim3 grid(static_cast<unsigned>(ceil_div(P, 64)), static_cast<unsigned>(ceil_div(L, 64)),
            static_cast<unsigned>(nz));
  if (trans)
    sgemm_kernel<true><<<grid, 256, 0, st>>>(A, lda, Bm, P, K, L, kchunk, part);
  else
    sgemm_kernel<false><<<grid, 256, 0, st>>>(A, lda, Bm, P, K, L, kchunk, part);
  const int64_t cnt = P * L;
  sum_parts_kernel<<<grid_for(cnt), 256, 0, st>>>(part, static_cast<int>(nz), cnt, C);
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

cudaError_t run_qr(float* A, int64_t m, int l, float* Rout, float* part, int lpad, unsigned* sync,
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

struct PrepCarve {
  float* ws;      // [M, N]
  float* omega;   // [N, l]
  float* Y;       // [M, l]
  float* Z;       // [N, l]
  float* Rb;      // [l, l]
  double* X;      // [n, n]
  double* J;      // [n, n]
  float* Ur;      // [l, r]
  float* Vr;      // [l, r]
  float* sig;     // [r]
  float* U;       // [M, r]
  float* V;       // [N, r]
  float* gpart;   // GEMM split-K partials
  float* qpart;   // QR partial sums [2][G][lpad]
  unsigned* sync;
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
    c.omega = static_cast<float*>(cv.take(static_cast<size_t>(N) * l * 4));
    c.Y = static_cast<float*>(cv.take(static_cast<size_t>(M) * l * 4));
    c.Z = static_cast<float*>(cv.take(static_cast<size_t>(N) * l * 4));
    c.Rb = static_cast<float*>(cv.take(static_cast<size_t>(l) * l * 4));
    c.X = static_cast<double*>(cv.take(static_cast<size_t>(n) * n * 8));
    c.J = static_cast<double*>(cv.take(static_cast<size_t>(n) * n * 8));
    c.Ur = static_cast<float*>(cv.take(static_cast<size_t>(l) * r * 4));
    c.Vr = static_cast<float*>(cv.take(static_cast<size_t>(l) * r * 4));
    c.sig = static_cast<float*>(cv.take(static_cast<size_t>(r) * 4));
    c.U = static_cast<float*>(cv.take(static_cast<size_t>(M) * r * 4));
    c.V = static_cast<float*>(cv.take(static_cast<size_t>(N) * r * 4));
    const int64_t gp = std::max({gemm_part_floats(M, N, l), gemm_part_floats(N, M, l),
                                 gemm_part_floats(M, l, r), gemm_part_floats(N, l, r)});
    c.gpart = static_cast<float*>(cv.take(static_cast<size_t>(gp) * 4));
    const int lpad = (l + 2 + 3) / 4 * 4;
    const int G = std::max(plan_qr(M, l).G, plan_qr(N, l).G);
    c.qpart = static_cast<float*>(cv.take(static_cast<size_t>(2) * G * lpad * 4));
    c.sync = static_cast<unsigned*>(cv.take(64));
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
  if (r > 0) {
    // the QR slices must fit in shared memory
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
    const int lpad = (l + 2 + 3) / 4 * 4;
    const int n = (l + 1) / 2 * 2;
    auto chk = [](cudaError_t e) { return e == cudaSuccess; };
    bool ok = true;
    gaussian_kernel<<<grid_for(ceil_div(N * l, 4)), 256, 0, st>>>(c.omega, N * l, seed);
    ok = ok && chk(cudaGetLastError());
    ok = ok && chk(run_gemm(false, c.ws, N, c.omega, M, N, l, c.gpart, c.Y, st));   // Y = ws Omega
    ok = ok && chk(run_qr(c.Y, M, l, nullptr, c.qpart, lpad, c.sync, status, st));
    for (int it = 0; it < q && ok; ++it) {
      ok = ok && chk(run_gemm(true, c.ws, N, c.Y, N, M, l, c.gpart, c.Z, st));     // Z = ws^T Q
      ok = ok && chk(run_qr(c.Z, N, l, nullptr, c.qpart, lpad, c.sync, status, st));
      ok = ok && chk(run_gemm(false, c.ws, N, c.Z, M, N, l, c.gpart, c.Y, st));    // Y = ws Z
      ok = ok && chk(run_qr(c.Y, M, l, nullptr, c.qpart, lpad, c.sync, status, st));
    }
    ok = ok && chk(run_gemm(true, c.ws, N, c.Y, N, M, l, c.gpart, c.Z, st));       // Bt = ws^T Q
    ok = ok && chk(run_qr(c.Z, N, l, c.Rb, c.qpart, lpad, c.sync, status, st));    // Bt = Qb Rb
    jacobi_svd_kernel<<<1, 1024, 0, st>>>(c.Rb, l, n, c.X, c.J, r, c.Ur, c.Vr, c.sig, 40);
    ok = ok && chk(cudaGetLastError());
    ok = ok && chk(run_gemm(false, c.Y, l, c.Ur, M, l, r, c.gpart, c.U, st));      // U = Q Ur
    ok = ok && chk(run_gemm(false, c.Z, l, c.Vr, N, l, r, c.gpart, c.V, st));      // V = Qb Vr
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
