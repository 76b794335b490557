// smooth.cu - the per-channel smoothing scale (svdq_smooth_scale), upstream of
// svdq_prepare.
//
// "SVDQuant Smoothing, Low-rank and Residual Quantization", Formula item 1 divides
// x by a per-input-channel scale and multiplies the weight rows by it; the scale
// itself is a given input there. The "SVDQuant parameter configuration guide"
// (msModelSlim), step 3 "choose and tune the parameters", tunes the migration
// strength of that scale (iter_smooth.alpha: 0.25 in its diffusion example, 0.9
// as the tool's default).
// Read as the usual migration scale of strength alpha:
//   scale_j = max_b |x[b, j]|^alpha / max_n |W[j, n]|^(1 - alpha),
// with a channel whose maximum is zero taking 1 for that factor.
//
// Three launches: zero the two maxima arrays, take the maxima (|x| column
// maxima by atomicMax on the fp32 bit patterns of |x|, which order like the
// values and make the result independent of the order; |W| row maxima by one
// warp per row), then the scale.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "internal.h"

namespace svdq {

namespace {

constexpr int kColTile = 256;
constexpr int kRowsPerBlock = 64;

template <typename T>
__device__ __forceinline__ uint32_t abs_bits(T v) {
  return __float_as_uint(fabsf(static_cast<float>(v))) & 0x7FFFFFFFu;
}

template <typename T>
__global__ void __launch_bounds__(kColTile) col_absmax_kernel(const T* x, int64_t B, int64_t M, int64_t ldx,
                                                              uint32_t* xmax) {
  const int64_t col = static_cast<int64_t>(blockIdx.x) * kColTile + threadIdx.x;
  if (col >= M) return;
  const int64_t r0 = static_cast<int64_t>(blockIdx.y) * kRowsPerBlock;
  const int64_t r1 = min(B, r0 + kRowsPerBlock);
  uint32_t m = 0u;
  for (int64_t r = r0; r < r1; ++r) m = max(m, abs_bits(x[r * ldx + col]));
  atomicMax(xmax + col, m);
}

template <typename T>
__global__ void __launch_bounds__(256) row_absmax_kernel(const T* w, int64_t M, int64_t N, int64_t ldw,
                                                         uint32_t* wmax) {
  const int64_t row = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= M) return;
  uint32_t m = 0u;
  for (int64_t n = lane; n < N; n += 32) m = max(m, abs_bits(w[row * ldw + n]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (lane == 0) wmax[row] = m;
}

__global__ void scale_kernel(const uint32_t* xmax, const uint32_t* wmax, int64_t M, float alpha, float* scale) {
  const int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (j >= M) return;
  const float xm = __uint_as_float(xmax[j]), wm = __uint_as_float(wmax[j]);
  const float a = xm > 0.0f ? powf(xm, alpha) : 1.0f;
  const float b = wm > 0.0f ? powf(wm, 1.0f - alpha) : 1.0f;
  scale[j] = __fdiv_rn(a, b);
}

template <typename T>
cudaError_t launch_absmax_x(const void* x, int64_t B, int64_t M, int64_t ldx, uint32_t* xmax, cudaStream_t st) {
  const dim3 grid(static_cast<unsigned>(ceil_div(M, kColTile)), static_cast<unsigned>(ceil_div(B, kRowsPerBlock)));
  col_absmax_kernel<T><<<grid, kColTile, 0, st>>>(static_cast<const T*>(x), B, M, ldx, xmax);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_absmax_w(const void* w, int64_t M, int64_t N, int64_t ldw, uint32_t* wmax, cudaStream_t st) {
  row_absmax_kernel<T><<<static_cast<unsigned>(ceil_div(M, 8)), 256, 0, st>>>(static_cast<const T*>(w), M, N, ldw,
                                                                              wmax);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_smooth_scale(const void* x, svdq_dtype xdt, int64_t B, int64_t M, int64_t ldx, const void* w,
                                svdq_dtype wdt, int64_t N, int64_t ldw, float alpha, float* scale, void* workspace,
                                cudaStream_t st) {
  uint32_t* xmax = static_cast<uint32_t*>(workspace);
  uint32_t* wmax = xmax + M;
  cudaError_t e = cudaMemsetAsync(xmax, 0, static_cast<size_t>(2 * M) * sizeof(uint32_t), st);
  if (e != cudaSuccess) return e;
  if (B > 0) {
    e = xdt == SVDQ_BF16 ? launch_absmax_x<__nv_bfloat16>(x, B, M, ldx, xmax, st)
                         : launch_absmax_x<float>(x, B, M, ldx, xmax, st);
    if (e != cudaSuccess) return e;
  }
  e = wdt == SVDQ_BF16 ? launch_absmax_w<__nv_bfloat16>(w, M, N, ldw, wmax, st)
                       : launch_absmax_w<float>(w, M, N, ldw, wmax, st);
  if (e != cudaSuccess) return e;
  scale_kernel<<<static_cast<unsigned>(ceil_div(M, 256)), 256, 0, st>>>(xmax, wmax, M, alpha, scale);
  return cudaGetLastError();
}

}  // namespace svdq
