// gemm_common.cuh - pieces shared by the residual GEMM kernels (gemm_pair.cu,
// gemm_skinny.cu): the argument block and the epilogue that turns 128-row slabs
// of TMEM accumulators into Y.
#pragma once

#include <cuda_bf16.h>

#include "internal.h"
#include "ptx.cuh"

namespace svdq {

// INT: kind::i8; NVFP4: e2m1 with ue4m3 scales per 16 elements and fp32 global
// scales; MXFP4: e2m1 with E8M0 scales per 32 elements, global scales 1.
enum GemmKind { kKindInt = 0, kKindNvfp4 = 1, kKindMxfp4 = 2 };
enum GemmOut { kOutF32 = 0, kOutBF16 = 1, kOutI32 = 2 };

struct GemmArgs {
  int B, N, M, lr_steps;
  const float* s_x;               // INT: s_x, fp4: gs_x (1 for MXFP4)
  const float* s_w;               // INT: s_w, fp4: gs_w (1 for MXFP4)
  const __nv_bfloat16* bias;
  void* y;
  int64_t ldy;
  int vec_ok;
  const uint8_t* sfa;             // fp4 activation scales (128x4 layout)
  const uint8_t* sfb;             // fp4 weight scales (128x4 layout)
  int katoms;                     // fp4: 4-scale atoms per row tile, ceil(M / 64) NVFP4, ceil(M / 128) MXFP4
  // pair kernel: K split of the last round's tiles (nsplit 1: none); the
  // workspace for the split (partials, then one counter per split tile)
  int nsplit;
  uint32_t* split_part;
  unsigned* split_cnt;
  unsigned* status;
};

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);  // a -> low half
  return *reinterpret_cast<const uint32_t*>(&h);
}

// Dequantisation factor of the residual accumulator.
template <int kKind, int kOut>
__device__ __forceinline__ float epilogue_alpha(const GemmArgs& args) {
  if (kOut == kOutI32) return 0.0f;
  if (kKind != kKindInt) return __fdiv_rn(1.0f, __fmul_rn(__ldg(args.s_x), __ldg(args.s_w)));
  return __ldg(args.s_x) * __ldg(args.s_w);
}

// Adds bias[n .. n + 32) to v (columns past N get nothing).
__device__ __forceinline__ void add_bias32(const GemmArgs& args, int n, float (&v)[32]) {
  if (args.bias == nullptr) return;
  if (n + 32 <= args.N) {
    const uint4* bp = reinterpret_cast<const uint4*>(args.bias + n);
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      const uint4 bb = __ldg(bp + g);
      const uint32_t w4[4] = {bb.x, bb.y, bb.z, bb.w};
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        v[8 * g + 2 * h] += __uint_as_float(w4[h] << 16);
        v[8 * g + 2 * h + 1] += __uint_as_float(w4[h] & 0xFFFF0000u);
      }
    }
  } else {
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if (n + j < args.N) v[j] += __bfloat162float(args.bias[n + j]);
  }
}

// alpha * accumulator (+ the INT up-projection) for 32 columns.
template <int kKind>
__device__ __forceinline__ void dequant32(const uint32_t (&acc)[32], const uint32_t (&up)[32],
                                          float alpha, bool sep_lr, float (&v)[32]) {
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    if (kKind != kKindInt) {
      v[j] = alpha * __uint_as_float(acc[j]);
    } else {
      v[j] = alpha * static_cast<float>(static_cast<int32_t>(acc[j]));
      if (sep_lr) v[j] += __uint_as_float(up[j]);
    }
  }
}

// Stores 32 finished columns of one row (fp32 values, or bf16 pairs packed
// low-first in 16 words).
template <int kOut>
__device__ __forceinline__ void store_row32(const GemmArgs& args, int row, int n, const uint32_t* w) {
  const bool full = args.vec_ok && (n + 32 <= args.N);
  if (kOut == kOutF32 || kOut == kOutI32) {
    uint32_t* dst = static_cast<uint32_t*>(args.y) + static_cast<int64_t>(row) * args.ldy + n;
    if (full) {
#pragma unroll
      for (int j = 0; j < 32; j += 4) *reinterpret_cast<uint4*>(dst + j) = make_uint4(w[j], w[j + 1], w[j + 2], w[j + 3]);
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (n + j < args.N) dst[j] = w[j];
    }
  } else {
    uint16_t* dst = static_cast<uint16_t*>(args.y) + static_cast<int64_t>(row) * args.ldy + n;
    if (full) {
#pragma unroll
      for (int j = 0; j < 16; j += 4) *reinterpret_cast<uint4*>(dst + 2 * j) = make_uint4(w[j], w[j + 1], w[j + 2], w[j + 3]);
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (n + j < args.N) dst[j] = static_cast<uint16_t>(j & 1 ? w[j >> 1] >> 16 : w[j >> 1] & 0xFFFFu);
    }
  }
}

// One warp, 32 rows x 32 columns straight from the accumulator(s) to Y.
// lane_addr is the TMEM address of this warp's lane quarter at column 0; the
// residual accumulator starts at column 0 (int32 for INT; fp32 for NVFP4,
// holding the low-rank branch too) and the INT low-rank fp32 accumulator at
// column 256.
template <int kKind, int kOut>
__device__ __forceinline__ void epilogue_chunk_direct(const GemmArgs& args, uint32_t lane_addr, int row,
                                                      int n, uint32_t col, float alpha, bool sep_lr) {
  __syncwarp();  // the TMEM loads below are warp-collective
  uint32_t acc[32], up[32];
  tmem_ld_32x32b_x32(lane_addr + col, acc);
  if (sep_lr) tmem_ld_32x32b_x32(lane_addr + 256 + col, up);
  tmem_ld_wait_regs(acc);
  if (sep_lr) tmem_ld_wait_regs(up);
  if (row >= args.B || n >= args.N) return;
  if (kOut == kOutI32) {
    store_row32<kOutI32>(args, row, n, acc);
    return;
  }
  float v[32];
  dequant32<kKind>(acc, up, alpha, sep_lr, v);
  add_bias32(args, n, v);
  if (kOut == kOutF32) {
    store_row32<kOutF32>(args, row, n, reinterpret_cast<const uint32_t*>(v));
  } else {
    uint32_t p[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) p[j] = pack_bf16x2(v[2 * j], v[2 * j + 1]);
    store_row32<kOutBF16>(args, row, n, p);
  }
}

// Two-pass epilogue (overlaps the global stores with the next tile's MMAs).
// Pass 1 from accumulator values already in registers (the accumulator columns
// are free again): the INT up-projection columns at lr_col are read, and the
// result goes to dst_col (bf16 pairs in 16 columns, or fp32 in 32).
template <int kKind, int kOut>
__device__ __forceinline__ void epilogue_combine_regs(const GemmArgs& args, uint32_t lane_addr, int n,
                                                      const uint32_t (&acc)[32], uint32_t lr_col,
                                                      uint32_t dst_col, float alpha, bool sep_lr) {
  __syncwarp();
  uint32_t up[32];
  if (sep_lr) {
    tmem_ld_32x32b_x32(lane_addr + lr_col, up);
    tmem_ld_wait_regs(up);
  }
  float v[32];
  dequant32<kKind>(acc, up, alpha, sep_lr, v);
  add_bias32(args, n, v);
  if (kOut == kOutBF16) {
    uint32_t p[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) p[j] = pack_bf16x2(v[2 * j], v[2 * j + 1]);
    tmem_st_32x32b_x16(lane_addr + dst_col, p);
  } else {
    uint32_t p[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) p[j] = __float_as_uint(v[j]);
    tmem_st_32x32b_x32(lane_addr + dst_col, p);
  }
}

// Pass 2: the finished 32 columns from TMEM to Y.
template <int kOut>
__device__ __forceinline__ void epilogue_store(const GemmArgs& args, uint32_t lane_addr, int row, int n,
                                               uint32_t src_col) {
  __syncwarp();
  if (kOut == kOutBF16) {
    uint32_t p[16];
    tmem_ld_32x32b_x16(lane_addr + src_col, p);
    tmem_ld_wait_regs(p);
    if (row < args.B) store_row32<kOutBF16>(args, row, n, p);
  } else {
    uint32_t p[32];
    tmem_ld_32x32b_x32(lane_addr + src_col, p);
    tmem_ld_wait_regs(p);
    if (row < args.B) store_row32<kOutF32>(args, row, n, p);
  }
}

// Host: the short-batch kernel (gemm_skinny.cu, B <= 128); false if a tensor map
// cannot be encoded. pdl: launch with programmatic serialization (only right
// after this library's activation pass, which writes nothing the weight loads read).
bool launch_gemm_skinny(int kind, int out, const GemmArgs& g, const void* act_codes, const uint8_t* act_sf,
                        const void* down2, const svdq_weight* w, bool pdl, cudaStream_t stream,
                        cudaError_t* err);

// Host: the CTA-pair kernel (gemm_pair.cu); false if a tensor map cannot be encoded.
// split_ws (may be null: no split) holds pair_split_bytes(B, N) bytes.
bool launch_gemm_pair(int kind, int out, const GemmArgs& args, const void* act_codes,
                      const void* down2, const svdq_weight* w, void* split_ws, cudaStream_t stream,
                      cudaError_t* err);

}  // namespace svdq
