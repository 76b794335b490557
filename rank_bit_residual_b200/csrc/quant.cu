// quant.cu - quantisation of the residual weight R[M, N] (fp32).
//
// INT: the per-tensor grid of "SVDQuant Smoothing, Low-rank and Residual
// Quantization" (Formula item 3): s_w = fl(max|R| / qmax) and
// codes = clamp(round_half_even(R / s_w), -qmax, qmax), the quotient rounded
// exactly (estimated as fl(R u) with u = fl(1 / s_w), re-decided by an fp32
// fma next to a half-integer), written K-major as codes[N, M] (row n =
// column n of R).
// NVFP4: 16-element blocks along M of each column of R, ue4m3 block scales in
// the 128x4 layout and an fp32 global scale (the weight_fp4 / weight_sf /
// alpha storage of "flashinfer.gemm.svdquant_linear"), same recipe as the
// activation pass: gs = 448*6 / max|R|, sf = ue4m3(fl(amax_b / 6) * gs),
// code = the exact e2m1 rounding of R * fl(gs / sf).
// MXFP4 (the "mxfp4" per-block format of the SVDQuant parameter configuration
// guide): 32-element blocks along M, E8M0 scales 2^X with X = floor(log2 amax) - 2,
// codes e2m1(R * 2^-X), no global scale.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "encode.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace svdq {

namespace {

constexpr int kMaxParts = 1024;

__global__ void __launch_bounds__(256) absmax_partial_kernel(const float* __restrict__ R, int64_t M,
                                                             int64_t N, int64_t ldR,
                                                             float* __restrict__ parts) {
  float m = 0.0f;
  const int64_t total = M * N;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = i / N, c = i - r * N;
    m = fmaxf(m, fabsf(R[r * ldR + c]));
  }
  __shared__ float red[8];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = red[0];
    for (int w = 1; w < 8; ++w) t = fmaxf(t, red[w]);
    parts[blockIdx.x] = t;
  }
}

__device__ float reduce_parts(const float* __restrict__ parts, int nparts) {
  __shared__ float red[8];
  float m = 0.0f;
  for (int i = threadIdx.x; i < nparts; i += blockDim.x) m = fmaxf(m, parts[i]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = red[0];
    for (int w = 1; w < static_cast<int>(blockDim.x >> 5); ++w) t = fmaxf(t, red[w]);
    red[0] = t;
  }
  __syncthreads();
  return red[0];
}

// 32 x 32 tiles: read R coalesced along N, write codes coalesced along M.
__global__ void __launch_bounds__(256) quant_int_transpose_kernel(
    const float* __restrict__ R, int64_t M, int64_t N, int64_t ldR, int qmax,
    const float* __restrict__ parts, int nparts, int8_t* __restrict__ codes,
    float* __restrict__ w_scale) {
  const float m = reduce_parts(parts, nparts);
  const float s = __fdiv_rn(m, static_cast<float>(qmax));
  const float u = s > 0.0f ? __frcp_rn(s) : 0.0f;
  if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) *w_scale = s;
  __shared__ int8_t tile[32][33];
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;  // 32 x 8
  const int64_t m0 = static_cast<int64_t>(blockIdx.y) * 32, n0 = static_cast<int64_t>(blockIdx.x) * 32;
  for (int i = ty; i < 32; i += 8) {
    const int64_t r = m0 + i, c = n0 + tx;
    int q = 0;
    if (r < M && c < N && s > 0.0f) q = int_code_residual(R[r * ldR + c], s, u, qmax);
    tile[i][tx] = static_cast<int8_t>(q);
  }
  __syncthreads();
  for (int i = ty; i < 32; i += 8) {
    const int64_t n = n0 + i, mm = m0 + tx;
    if (n < N && mm < M) codes[n * M + mm] = tile[tx][i];
  }
}

// One thread per (column n, 16-row block kb) of R; consecutive threads take
// consecutive n so every row read is coalesced.
__global__ void __launch_bounds__(256) quant_nvfp4_kernel(
    const float* __restrict__ R, int64_t M, int64_t N, int64_t ldR, const float* __restrict__ parts,
    int nparts, uint8_t* __restrict__ codes, uint8_t* __restrict__ sf,
    float* __restrict__ w_scale) {
  const float m = reduce_parts(parts, nparts);
  const float gs = m > 0.0f ? __fdiv_rn(2688.0f, m) : 1.0f;
  if (blockIdx.x == 0 && threadIdx.x == 0) *w_scale = gs;
  const int64_t kb = M / 16;
  const int64_t kbp = (kb + 3) / 4 * 4;
  const int64_t np = (N + 127) / 128 * 128;
  const int64_t total = np * kbp;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t b = i / np;
    const int64_t n = i - b * np;
    const int64_t off = ((n >> 7) * (kbp >> 2) + (b >> 2)) * 512 + (n & 31) * 16 +
                        ((n & 127) >> 5) * 4 + (b & 3);
    if (n >= N || b >= kb) {
      sf[off] = 0;
      continue;
    }
    float rv[16], v[16];
    float amax = 0.0f;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      rv[j] = R[(b * 16 + j) * ldR + n];
      amax = fmaxf(amax, fabsf(rv[j]));
    }
    const uint8_t sfb = f32_to_ue4m3(__fmul_rn(__fdiv_rn(amax, 6.0f), gs));
    const float d = ue4m3_to_f32(sfb);
    const float enc = d > 0.0f ? __fdiv_rn(gs, d) : 0.0f;
#pragma unroll
    for (int j = 0; j < 16; ++j) v[j] = __fmul_rn(rv[j], enc);
    *reinterpret_cast<uint2*>(codes + n * (M / 2) + b * 8) =
        make_uint2(e2m1x8_exact(v, rv, enc, nullptr), e2m1x8_exact(v + 8, rv + 8, enc, nullptr));
    sf[off] = sfb;
  }
}

// MXFP4: one thread per (column n, 32-row block b) of R; e2m1 codes of R * 2^-X
// with X from the block's amax (encode.cuh), E8M0 byte X + 127; w_scale = 1.
__global__ void __launch_bounds__(256) quant_mxfp4_kernel(const float* __restrict__ R, int64_t M, int64_t N,
                                                          int64_t ldR, uint8_t* __restrict__ codes,
                                                          uint8_t* __restrict__ sf, float* __restrict__ w_scale) {
  if (blockIdx.x == 0 && threadIdx.x == 0) *w_scale = 1.0f;
  const int64_t kb = M / 32;
  const int64_t kbp = (kb + 3) / 4 * 4;
  const int64_t np = (N + 127) / 128 * 128;
  const int64_t total = np * kbp;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t b = i / np;
    const int64_t n = i - b * np;
    const int64_t off = sf_swizzle_offset(n, b, kbp);
    if (n >= N || b >= kb) {
      sf[off] = 0;
      continue;
    }
    float v[32];
    float amax = 0.0f;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      v[j] = R[(b * 32 + j) * ldR + n];
      amax = fmaxf(amax, fabsf(v[j]));
    }
    const int X = mx_block_exponent(amax);
    const float inv = mx_inv_scale(X);
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] = __fmul_rn(v[j], inv);
    *reinterpret_cast<uint4*>(codes + n * (M / 2) + b * 16) =
        make_uint4(f32x8_to_e2m1(v), f32x8_to_e2m1(v + 8), f32x8_to_e2m1(v + 16), f32x8_to_e2m1(v + 24));
    sf[off] = static_cast<uint8_t>(X + 127);
  }
}

// 32 codes (32 bytes) -> 16 packed bytes per thread; element 2j in the low nibble.
__global__ void __launch_bounds__(256) pack_int4_kernel(const int8_t* __restrict__ codes, int64_t n16,
                                                        uint8_t* __restrict__ packed) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n16;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const uint4 a = __ldg(reinterpret_cast<const uint4*>(codes) + 2 * i);
    const uint4 b = __ldg(reinterpret_cast<const uint4*>(codes) + 2 * i + 1);
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    uint32_t o[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      // bytes e0..e7 of two words -> nibbles: even elements low, odd elements high
      const uint32_t lo = __byte_perm(w[2 * j], w[2 * j + 1], 0x6420) & 0x0F0F0F0Fu;
      const uint32_t hi = __byte_perm(w[2 * j], w[2 * j + 1], 0x7531) & 0x0F0F0F0Fu;
      o[j] = lo | (hi << 4);
    }
    reinterpret_cast<uint4*>(packed)[i] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

int parts_for(int64_t M, int64_t N) {
  return static_cast<int>(std::max<int64_t>(
      1, std::min<int64_t>(kMaxParts, ceil_div(M * N, 256 * 16))));
}

}  // namespace

size_t residual_scratch_bytes(int64_t M, int64_t N) {
  return static_cast<size_t>(parts_for(M, N)) * sizeof(float) + 256;
}

cudaError_t launch_quantize_residual(const float* R, int64_t M, int64_t N, int64_t ldR,
                                     svdq_fmt fmt, void* codes, void* sf, float* w_scale,
                                     void* scratch, cudaStream_t stream) {
  const int nparts = parts_for(M, N);
  float* parts = static_cast<float*>(scratch);
  absmax_partial_kernel<<<nparts, 256, 0, stream>>>(R, M, N, ldR, parts);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (fmt.kind == SVDQ_KIND_INT) {
    const int qmax = (1 << (fmt.bits - 1)) - 1;
    dim3 grid(static_cast<unsigned>(ceil_div(N, 32)), static_cast<unsigned>(ceil_div(M, 32)));
    quant_int_transpose_kernel<<<grid, 256, 0, stream>>>(R, M, N, ldR, qmax, parts, nparts,
                                                          static_cast<int8_t*>(codes), w_scale);
  } else if (fmt.kind == SVDQ_KIND_MXFP4) {
    const int64_t work = round_up(N, 128) * round_up(M / 32, 4);
    const int blocks = static_cast<int>(std::max<int64_t>(
        1, std::min<int64_t>(ceil_div(work, 256), static_cast<int64_t>(num_sms()) * 8)));
    quant_mxfp4_kernel<<<blocks, 256, 0, stream>>>(R, M, N, ldR, static_cast<uint8_t*>(codes),
                                                    static_cast<uint8_t*>(sf), w_scale);
  } else {
    const int64_t work = round_up(N, 128) * round_up(M / 16, 4);
    const int blocks = static_cast<int>(std::max<int64_t>(
        1, std::min<int64_t>(ceil_div(work, 256), static_cast<int64_t>(num_sms()) * 8)));
    quant_nvfp4_kernel<<<blocks, 256, 0, stream>>>(R, M, N, ldR, parts, nparts,
                                                    static_cast<uint8_t*>(codes),
                                                    static_cast<uint8_t*>(sf), w_scale);
  }
  return cudaGetLastError();
}

cudaError_t launch_pack_int4(const int8_t* codes, int64_t N, int64_t M, uint8_t* packed,
                             cudaStream_t stream) {
  const int64_t n16 = N * M / 32;   // 16-byte outputs (M is a multiple of 32)
  const int blocks = static_cast<int>(std::max<int64_t>(
      1, std::min<int64_t>(ceil_div(n16, 256), static_cast<int64_t>(num_sms()) * 8)));
  pack_int4_kernel<<<blocks, 256, 0, stream>>>(codes, n16, packed);
  return cudaGetLastError();
}

}  // namespace svdq
