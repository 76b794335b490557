// fold.cu - the smoothing scale chosen as the optimal diagonal fold of the
// quantized product (svdq_fold_scale), upstream of svdq_prepare.
//
// "Contraction-Gauge Preconditioning for Quantized Matrix Multiplication"
// (abstract): with independent zero-mean quantization errors of known variance,
// the expected squared error of a product of two quantized factors has an exact
// expression; the product is unchanged by a gauge A B = (A T)(T^-1 B), and within
// positive diagonal gauges (folds) a geometric program gives the globally optimal
// shared fold. Here A = x, B = W and the fold is the smoothing of "SVDQuant
// Smoothing, Low-rank and Residual Quantization" (Formula item 1): t = 1 / scale.
// With per-tensor grids of qmax = 2^(bits-1) - 1 on both operands and the dither
// variance Delta^2 / 12, the program is
//
//   minimise  c1 U^2 sum_k beta_k / t_k^2 + c2 V^2 sum_k alpha_k t_k^2 + c3 U^2 V^2
//   subject to a_k t_k <= U,  b_k / t_k <= V,
//   c1 = m / (12 q^2), c2 = n / (12 q^2), c3 = K m n / (144 q^4),
//
// a_k, alpha_k the maximum and the sum of squares of |x[:, k]|, b_k, beta_k those
// of W[k, :]. The objective is invariant under t -> c t, so U = 1. For a fixed V
// each t_k solves a one-dimensional problem convex in log t_k:
//   t_k = clamp((c1 beta_k / (c2 V^2 alpha_k))^(1/4), b_k / V, 1 / a_k),
// and what remains is convex in log V (a partial minimum of a function jointly
// convex in log t and log V), minimised by golden-section search on
// [log max_k a_k b_k, that + 40]. Channels with a_k = 0 or b_k = 0 carry no
// product term: they take the geometric mean of the other t_k, moved only as far
// as needed to keep U = 1 and V.
//
// Three launches: column statistics of x in row chunks (partials), row
// statistics of W (a warp per row), and the solver on one CTA (it adds the
// partials in chunk order, so the result does not depend on scheduling).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "internal.h"

namespace svdq {

namespace {

constexpr int kColTile = 256;
constexpr int kRowsPerChunk = 256;
constexpr int kSolveThreads = 1024;
constexpr int kGoldenIters = 200;

template <typename T>
__device__ __forceinline__ double to_d(T v) {
  return static_cast<double>(static_cast<float>(v));
}

template <typename T>
__global__ void __launch_bounds__(kColTile) fold_xstats_kernel(const T* __restrict__ x, int64_t B, int64_t M,
                                                               int64_t ldx, float* __restrict__ pmax,
                                                               double* __restrict__ pss) {
  const int64_t col = static_cast<int64_t>(blockIdx.x) * kColTile + threadIdx.x;
  if (col >= M) return;
  const int64_t r0 = static_cast<int64_t>(blockIdx.y) * kRowsPerChunk;
  const int64_t r1 = min(B, r0 + kRowsPerChunk);
  float m = 0.0f;
  double ss = 0.0;
  for (int64_t r = r0; r < r1; ++r) {
    const double v = to_d(x[r * ldx + col]);
    m = fmaxf(m, static_cast<float>(fabs(v)));
    ss = fma(v, v, ss);
  }
  pmax[blockIdx.y * M + col] = m;
  pss[blockIdx.y * M + col] = ss;
}

template <typename T>
__global__ void __launch_bounds__(256) fold_wstats_kernel(const T* __restrict__ w, int64_t M, int64_t N,
                                                          int64_t ldw, double* __restrict__ b,
                                                          double* __restrict__ beta) {
  const int64_t row = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= M) return;
  double m = 0.0, ss = 0.0;
  for (int64_t n = lane; n < N; n += 32) {
    const double v = to_d(w[row * ldw + n]);
    m = fmax(m, fabs(v));
    ss = fma(v, v, ss);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    m = fmax(m, __shfl_xor_sync(0xffffffffu, m, o));
    ss += __shfl_xor_sync(0xffffffffu, ss, o);
  }
  if (lane == 0) {
    b[row] = m;
    beta[row] = ss;
  }
}

// Block-wide sum and max (deterministic: fixed thread-to-value mapping).
__device__ double block_sum(double v, double* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  double t = 0.0;
  for (int w = 0; w < kSolveThreads / 32; ++w) t += red[w];
  return t;
}
__device__ double block_max(double v, double* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmax(v, __shfl_xor_sync(0xffffffffu, v, o));
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  double t = red[0];
  for (int w = 1; w < kSolveThreads / 32; ++w) t = fmax(t, red[w]);
  return t;
}

struct FoldArgs {
  int64_t M, B, N;
  int nchunks;
  double c1, c2, c3;
  const float* pmax;
  const double* pss;
  double* a;
  double* alpha;
  const double* b;
  const double* beta;
  double* t;
  float* scale;
};

__device__ __forceinline__ double t_of(double V, double a, double al, double b, double be, double c1,
                                       double c2) {
  const double t = sqrt(sqrt(c1 * be / (c2 * V * V * al)));
  return fmin(fmax(t, b / V), 1.0 / a);
}

__global__ void __launch_bounds__(kSolveThreads, 1) fold_solve_kernel(const FoldArgs f) {
  __shared__ double red[kSolveThreads / 32];
  const int tid = threadIdx.x;
  // column statistics of x: partials added in chunk order
  double vmin = 0.0;
  for (int64_t k = tid; k < f.M; k += kSolveThreads) {
    float m = 0.0f;
    double ss = 0.0;
    for (int c = 0; c < f.nchunks; ++c) {
      m = fmaxf(m, f.pmax[c * f.M + k]);
      ss += f.pss[c * f.M + k];
    }
    f.a[k] = m;
    f.alpha[k] = ss;
    if (m > 0.0f && f.b[k] > 0.0) vmin = fmax(vmin, static_cast<double>(m) * f.b[k]);
  }
  vmin = block_max(vmin, red);
  if (vmin <= 0.0) {   // no channel carries a product term: the identity fold
    for (int64_t k = tid; k < f.M; k += kSolveThreads) f.scale[k] = 1.0f;
    return;
  }
  // F(log V), the objective at the per-channel optimum for that V
  auto F = [&](double lv) -> double {
    const double V = exp(lv);
    double s1 = 0.0, s2 = 0.0;
    for (int64_t k = tid; k < f.M; k += kSolveThreads) {
      const double a = f.a[k], b = f.b[k];
      if (a > 0.0 && b > 0.0) {
        const double t = t_of(V, a, f.alpha[k], b, f.beta[k], f.c1, f.c2);
        s1 += f.beta[k] / (t * t);
        s2 += f.alpha[k] * t * t;
      }
    }
    s1 = block_sum(s1, red);
    s2 = block_sum(s2, red);
    return f.c1 * s1 + f.c2 * V * V * s2 + f.c3 * V * V;
  };
  const double g = 0.6180339887498949;   // (sqrt(5) - 1) / 2
  double lo = log(vmin), hi = lo + 40.0;
  double x1 = hi - g * (hi - lo), x2 = lo + g * (hi - lo);
  double f1 = F(x1), f2 = F(x2);
  for (int it = 0; it < kGoldenIters; ++it) {
    if (f1 <= f2) {
      hi = x2;
      x2 = x1;
      f2 = f1;
      x1 = hi - g * (hi - lo);
      f1 = F(x1);
    } else {
      lo = x1;
      x1 = x2;
      f1 = f2;
      x2 = lo + g * (hi - lo);
      f2 = F(x2);
    }
  }
  const double V = exp(0.5 * (lo + hi));
  // the fold; the geometric mean of the live channels' t for the others
  double slog = 0.0, nlive = 0.0, vmax = 0.0;
  for (int64_t k = tid; k < f.M; k += kSolveThreads) {
    const double a = f.a[k], b = f.b[k];
    if (a > 0.0 && b > 0.0) {
      const double t = t_of(V, a, f.alpha[k], b, f.beta[k], f.c1, f.c2);
      f.t[k] = t;
      slog += log(t);
      nlive += 1.0;
      vmax = fmax(vmax, b / t);
    }
  }
  slog = block_sum(slog, red);
  nlive = block_sum(nlive, red);
  vmax = block_max(vmax, red);
  const double gm = exp(slog / nlive);
  for (int64_t k = tid; k < f.M; k += kSolveThreads) {
    const double a = f.a[k], b = f.b[k];
    double t;
    if (a > 0.0 && b > 0.0) {
      t = f.t[k];
    } else {
      t = gm;
      if (a > 0.0) t = fmin(t, 1.0 / a);
      if (b > 0.0) t = fmax(t, b / vmax);
    }
    f.scale[k] = static_cast<float>(1.0 / t);
  }
}

int fold_chunks(int64_t B) { return static_cast<int>(std::max<int64_t>(1, ceil_div(B, kRowsPerChunk))); }

}  // namespace

size_t fold_scratch_bytes(int64_t B, int64_t M) {
  const int64_t R = fold_chunks(B);
  return static_cast<size_t>(round_up(R * M * 4, 256) + round_up(R * M * 8, 256) + 5 * round_up(M * 8, 256)) + 256;
}

cudaError_t launch_fold_scale(const void* x, svdq_dtype xdt, int64_t B, int64_t M, int64_t ldx, const void* w,
                              svdq_dtype wdt, int64_t N, int64_t ldw, int bits, float* scale, void* workspace,
                              cudaStream_t st) {
  const int R = fold_chunks(B);
  Carver cv(workspace, ~size_t(0));
  FoldArgs f{};
  f.M = M;
  f.B = B;
  f.N = N;
  f.nchunks = R;
  const double q = static_cast<double>((1 << (bits - 1)) - 1);
  f.c1 = static_cast<double>(B) / (12.0 * q * q);
  f.c2 = static_cast<double>(N) / (12.0 * q * q);
  f.c3 = static_cast<double>(M) * B * N / (144.0 * q * q * q * q);
  float* pmax = static_cast<float*>(cv.take(static_cast<size_t>(R * M) * 4));
  double* pss = static_cast<double*>(cv.take(static_cast<size_t>(R * M) * 8));
  f.a = static_cast<double*>(cv.take(static_cast<size_t>(M) * 8));
  f.alpha = static_cast<double*>(cv.take(static_cast<size_t>(M) * 8));
  double* b = static_cast<double*>(cv.take(static_cast<size_t>(M) * 8));
  double* beta = static_cast<double*>(cv.take(static_cast<size_t>(M) * 8));
  f.t = static_cast<double*>(cv.take(static_cast<size_t>(M) * 8));
  f.pmax = pmax;
  f.pss = pss;
  f.b = b;
  f.beta = beta;
  f.scale = scale;
  dim3 gx(static_cast<unsigned>(ceil_div(M, kColTile)), static_cast<unsigned>(R));
  if (xdt == SVDQ_BF16)
    fold_xstats_kernel<__nv_bfloat16><<<gx, kColTile, 0, st>>>(static_cast<const __nv_bfloat16*>(x), B, M, ldx,
                                                                pmax, pss);
  else
    fold_xstats_kernel<float><<<gx, kColTile, 0, st>>>(static_cast<const float*>(x), B, M, ldx, pmax, pss);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const unsigned gw = static_cast<unsigned>(ceil_div(M, 8));
  if (wdt == SVDQ_BF16)
    fold_wstats_kernel<__nv_bfloat16><<<gw, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(w), M, N, ldw, b, beta);
  else
    fold_wstats_kernel<float><<<gw, 256, 0, st>>>(static_cast<const float*>(w), M, N, ldw, b, beta);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  fold_solve_kernel<<<1, kSolveThreads, 0, st>>>(f);
  return cudaGetLastError();
}

}  // namespace svdq
