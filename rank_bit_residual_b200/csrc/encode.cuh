// encode.cuh - element encoders shared by the activation kernels and the
// residual quantiser: ue4m3 block scales, e2m1 codes, INT codes by the
// round-to-nearest-even add trick, the 128x4 scale layout and bf16/fp32 loads.
//
// Formats ("flashinfer.gemm.svdquant_linear", Parameters: packed e2m1 residual,
// ue4m3 scales in the 128x4 layout): e2m1 magnitudes {0, .5, 1, 1.5, 2, 3, 4, 6},
// ue4m3 = e4m3 (bias 7, max 448) restricted to >= 0; the INT grid of "SVDQuant
// Smoothing, Low-rank and Residual Quantization" (Formula item 3); MXFP4 block
// exponents (the "mxfp4" per-block format of the SVDQuant parameter
// configuration guide).
#pragma once

#include <cstdint>

namespace svdq {

// fp32 -> ue4m3 byte, round to nearest even, saturating at 448.
__device__ __forceinline__ uint8_t f32_to_ue4m3(float v) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(v));
  return static_cast<uint8_t>(r & 0xFFu);
}

// Exact value of a non-negative e4m3 byte (bias 7; exponent 0 is subnormal).
__device__ __forceinline__ float ue4m3_to_f32(uint8_t b) {
  const uint32_t e = (b >> 3) & 0xFu, m = b & 7u;
  return e == 0 ? static_cast<float>(m) * 0.001953125f  // m * 2^-9
                : __uint_as_float(((e + 120u) << 23) | (m << 20));
}

// Eight floats -> eight e2m1 nibbles, element j in nibble j (low nibble first);
// a code whose magnitude is zero is stored as +0.
__device__ __forceinline__ uint32_t f32x8_to_e2m1(const float* v) {
  uint32_t out;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(out)
      : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
  const uint32_t mag = out & 0x77777777u;
  const uint32_t nz = (mag + 0x77777777u) & 0x88888888u;
  return out & (0x77777777u | nz);
}

// MXFP4 block exponent (OCP microscaling, the "mxfp4" per-block MinMax format):
// X = floor(log2(amax)) - 2 (2 = the exponent of e2m1's largest value 6),
// clamped to [-127, 127]; a zero (or subnormal) amax gives -127. The E8M0 scale
// byte is X + 127 and the block's values are encoded as e2m1(v * 2^-X).
__device__ __forceinline__ int mx_block_exponent(float amax) {
  const int e = static_cast<int>((__float_as_uint(amax) >> 23) & 0xFFu);   // amax >= 0
  return e == 0 ? -127 : max(-127, e - 129);
}

// 2^-X as an fp32 (exact: -X lies in [-125, 127]).
__device__ __forceinline__ float mx_inv_scale(int X) {
  return __uint_as_float(static_cast<uint32_t>(127 - X) << 23);
}

// Byte offset of scale (row, col) in the 128x4 layout: 128-row x 4-column atoms
// of 512 bytes, byte (row % 32) * 16 + ((row % 128) / 32) * 4 + col % 4 inside an
// atom, atoms along the scale columns first (kbp / 4 per 128 rows), then rows.
__device__ __forceinline__ int64_t sf_swizzle_offset(int64_t row, int64_t col, int64_t kbp) {
  return ((row >> 7) * (kbp >> 2) + (col >> 2)) * 512 + (row & 31) * 16 + ((row & 127) >> 5) * 4 +
         (col & 3);
}

// 16 bytes of x as floats: 8 bf16 or 4 fp32
template <typename TIn>
__device__ __forceinline__ void unpack16(const uint4 u, float* v) {
  if constexpr (sizeof(TIn) == 2) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      v[2 * j] = __uint_as_float(w[j] << 16);
      v[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
    }
  } else {
    v[0] = __uint_as_float(u.x);
    v[1] = __uint_as_float(u.y);
    v[2] = __uint_as_float(u.z);
    v[3] = __uint_as_float(u.w);
  }
}

// INT codes of 8 elements: rint(fl(x c_k)), packed as 8 bytes. Adding
// 1.5 * 2^23 rounds an fp32 value below 2^22 in magnitude to the nearest
// integer, ties to even, and leaves that integer in the low bits of the sum,
// so the low byte of the sum is the two's-complement code. The clamp to
// [-qmax, qmax] of the definition is omitted: with s = fl(m / qmax) and
// c_k = fl(fl(1 / scale_k) fl(1 / s)), every |fl(x c_k)| is at most
// qmax (1 + 6 * 2^-24) < qmax + 1/2, so no code can leave the range.
__device__ __forceinline__ uint2 int_codes8(const float (&v)[8], const float (&ck)[8]) {
  uint32_t f[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) f[j] = __float_as_uint(__fadd_rn(__fmul_rn(v[j], ck[j]), 12582912.0f));
  const uint32_t lo = __byte_perm(__byte_perm(f[0], f[1], 0x0040), __byte_perm(f[2], f[3], 0x0040), 0x5410);
  const uint32_t hi = __byte_perm(__byte_perm(f[4], f[5], 0x0040), __byte_perm(f[6], f[7], 0x0040), 0x5410);
  return make_uint2(lo, hi);
}

}  // namespace svdq
