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

// 16 packed bytes (32 two's-complement nibbles, element 2j in the low nibble
// of byte j) -> 32 int8 codes in element order.
__device__ __forceinline__ void widen_int4(const uint4 v, uint32_t (&o)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint32_t lo = w[i] & 0x0F0F0F0Fu;          // elements 8i + 0, 2, 4, 6
    uint32_t hi = (w[i] >> 4) & 0x0F0F0F0Fu;   // elements 8i + 1, 3, 5, 7
    lo |= (lo & 0x08080808u) * 0x1Eu;          // sign-extend each nibble to its byte
    hi |= (hi & 0x08080808u) * 0x1Eu;
    o[2 * i] = __byte_perm(lo, hi, 0x5140);
    o[2 * i + 1] = __byte_perm(lo, hi, 0x7362);
  }
}

// ------------------------------------------------------------ exact rounding
// Every code is the correctly rounded value of a real quotient (the grid of
// "SVDQuant Smoothing, Low-rank and Residual Quantization", Formula item 3:
// round half to even of X_hat / s with X_hat = x / scale; the e2m1 encoding of
// the NVFP4 / MXFP4 blocks). The kernels first form an fp32 estimate of the
// quotient with a few multiplies by rounded reciprocals; the estimate lies
// within 2^-21 of the quotient, relatively, so it can only round to the wrong
// side when the quotient is that close to a rounding boundary. Those rare
// elements are flagged by cheap tests and decided again with exact arithmetic:
// a boundary test "a > b * d" is the sign of fma(-b, d, a), computed from the
// exact product and rounded once, so its sign is exact.

// The exact INT code of a / (scale_k s), given an estimate q_est that is off by
// at most one: round half to even, clamped to [-qmax, qmax]. scale_k * s is
// exact in double (24 + 24 significant bits), and fma(-(q + 1/2), D, |a|)
// has the sign of |a| - (q + 1/2) scale_k s exactly.
static __device__ __noinline__ int int_code_fix(float a, float scale_k, float s, int q_est, int qmax) {
  const double D = static_cast<double>(scale_k) * static_cast<double>(s);
  const double aa = fabs(static_cast<double>(a));
  int q = abs(q_est);
  const double up = fma(-(static_cast<double>(q) + 0.5), D, aa);
  if (up > 0.0 || (up == 0.0 && (q & 1))) {
    q += 1;
  } else if (q > 0) {
    const double dn = fma(-(static_cast<double>(q) - 0.5), D, aa);
    if (dn < 0.0 || (dn == 0.0 && (q & 1))) q -= 1;
  }
  q = min(q, qmax);
  return a < 0.0f ? -q : q;
}

// Adding 1.5 * 2^23 rounds an fp32 value below 2^22 in magnitude to the
// nearest integer, ties to even, and leaves that integer in the low bits of
// the sum (the low byte is then the two's-complement code); subtracting the
// constant again gives the rounded value exactly.
constexpr float kRintMagic = 12582912.0f;
// An estimate whose distance to its rounded value exceeds this lies near a
// half-integer: with |t| <= 128 (qmax <= 127) its error is below 2^-15.
constexpr float kNearHalf = 0.5f - 1.0f / 8192.0f;

// The same limit for the activation codes' estimate x c_k. Its error is below
// 3 (qmax + 1) 2^-24: c_k carries three roundings relative to 1 / (scale_k s),
// and |x / (scale_k s)| <= qmax (1 + 2^-23). A distance of at most
// 1/2 - 8 (qmax + 1) 2^-24 (that error plus the 2^-26 rounding of the distance
// itself, with room to spare) puts the exact quotient within 1/2 of the same
// integer. For INT4 the band is 2^-18 wide on each side of a half-integer.
__device__ __forceinline__ float act_near_limit(int qmax) {
  return __fmaf_rn(-static_cast<float>(qmax + 1), 1.0f / 2097152.0f, 0.5f);
}

// Packed pairs of fp32 (sm_100a f32x2 arithmetic): each lane of the pair is
// rounded to nearest even on its own, exactly as the scalar operation.
__device__ __forceinline__ uint64_t pk2(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void upk2(uint64_t r, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(r));
}
__device__ __forceinline__ uint64_t fmul2_rn(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t fadd2_rn(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t fsub2_rn(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t ffma2_rn(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}

// INT codes of 8 consecutive columns in each of kP rows, packed as 8 bytes per
// row: the exact round_half_even(x / (scale_k s)), estimated as rint(x c_k)
// with the per-column constant c_k = fl(fl(1 / scale_k) fl(1 / s)) and
// re-decided by int_code_fix where the estimate is near a half-integer.
// The estimate takes one fused rounding, fma(x, c_k, 1.5 * 2^23) (the magic
// constant's unit spacing makes that rounding the rint of the exact product),
// and the distance to it is a second fma, x c_k - rint; the largest distance of
// the group decides whether any element needs the rare path. scale8 points at
// the 8 columns' smoothing scales (read only on that rare path). The estimate
// never exceeds qmax (1 + 6 * 2^-24) < qmax + 1/2 in magnitude, so the fast
// path needs no clamp. The fast path runs on pairs of elements (f32x2) for all
// rows before the one test, so the rows' chains interleave; the rare path
// finds the flagged elements again with the same scalar operations.
template <int kP>
__device__ __forceinline__ void int_codes8_rows(const float (&v)[kP][8], const float (&ck)[8],
                                                const float* scale8, float s, int qmax, uint2 (&out)[kP]) {
  uint32_t f[kP][8];
  float dmax = 0.0f;
  const uint64_t mg = pk2(kRintMagic, kRintMagic);
#pragma unroll
  for (int p = 0; p < kP; ++p)
#pragma unroll
    for (int j = 0; j < 8; j += 2) {
      const uint64_t x2 = pk2(v[p][j], v[p][j + 1]);
      const uint64_t c2 = pk2(ck[j], ck[j + 1]);
      const uint64_t fs = ffma2_rn(x2, c2, mg);           // 1.5 * 2^23 + rint(x c_k)
      const uint64_t d = ffma2_rn(x2, c2, fsub2_rn(mg, fs));   // x c_k - rint(x c_k)
      float d0, d1, s0, s1;
      upk2(d, d0, d1);
      upk2(fs, s0, s1);
      f[p][j] = __float_as_uint(s0);
      f[p][j + 1] = __float_as_uint(s1);
      dmax = fmaxf(dmax, fmaxf(fabsf(d0), fabsf(d1)));
    }
  const float lim = act_near_limit(qmax);
  if (__builtin_expect(dmax > lim, 0)) {
#pragma unroll
    for (int p = 0; p < kP; ++p)
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float fs = __fmaf_rn(v[p][j], ck[j], kRintMagic);
        if (fabsf(__fmaf_rn(v[p][j], ck[j], __fsub_rn(kRintMagic, fs))) > lim) {
          const int q_est = static_cast<int>(f[p][j] & 0xFFu) - static_cast<int>((f[p][j] & 0x80u) << 1);
          f[p][j] = static_cast<uint32_t>(int_code_fix(v[p][j], __ldg(scale8 + j), s, q_est, qmax)) & 0xFFu;
        }
      }
  }
#pragma unroll
  for (int p = 0; p < kP; ++p) {
    const uint32_t lo = __byte_perm(__byte_perm(f[p][0], f[p][1], 0x0040), __byte_perm(f[p][2], f[p][3], 0x0040), 0x5410);
    const uint32_t hi = __byte_perm(__byte_perm(f[p][4], f[p][5], 0x0040), __byte_perm(f[p][6], f[p][7], 0x0040), 0x5410);
    out[p] = make_uint2(lo, hi);
  }
}

// The same for one row.
__device__ __forceinline__ uint2 int_codes8(const float (&v)[8], const float (&ck)[8],
                                            const float* scale8, float s, int qmax) {
  uint2 out[1];
  int_codes8_rows<1>(reinterpret_cast<const float(&)[1][8]>(v), ck, scale8, s, qmax, out);
  return out[0];
}

// Residual INT code of one fp32 element: round_half_even(R / s) clamped, with
// the estimate rint(fl(R u)), u = fl(1 / s), re-decided exactly near a
// half-integer (fp32 fma: R - (q + 1/2) s is formed exactly and rounded once).
__device__ __forceinline__ int int_code_residual(float r, float s, float u, int qmax) {
  const float t = __fmul_rn(r, u);
  const float rt = __fsub_rn(__fadd_rn(t, kRintMagic), kRintMagic);
  int q = static_cast<int>(rt);
  if (__builtin_expect(fabsf(__fsub_rn(t, rt)) > kNearHalf, 0)) {
    const float ar = fabsf(r);
    q = abs(q);
    const float up = __fmaf_rn(-(static_cast<float>(q) + 0.5f), s, ar);
    if (up > 0.0f || (up == 0.0f && (q & 1))) {
      q += 1;
    } else if (q > 0) {
      const float dn = __fmaf_rn(-(static_cast<float>(q) - 0.5f), s, ar);
      if (dn < 0.0f || (dn == 0.0f && (q & 1))) q -= 1;
    }
    q = r < 0.0f ? -q : q;
  }
  return min(max(q, -qmax), qmax);
}

// fp32 rounding of max_j |x_j| / scale_j over n elements, exactly: est[j] =
// fl(|x_j| fl(1 / scale_j)) is within 2^-23 of the quotient, relatively, so
// every element whose estimate is within 2^-21 of the largest estimate is a
// candidate, and the maximum of their IEEE quotients fl(|x_j| / scale_j)
// (rounding is monotone) is the rounded maximum. Usually the element with the
// largest estimate is the only candidate: its quotient is taken alone, and
// the others only when a second candidate exists.
template <int N>
__device__ __forceinline__ float block_amax_exact(const float (&x)[N], const float (&est)[N],
                                                  const float* scale_n) {
  float e = 0.0f, xa = 0.0f;
  int ja = 0;
#pragma unroll
  for (int j = 0; j < N; ++j) {
    const float a = fabsf(est[j]);
    if (a > e) {
      e = a;
      xa = fabsf(x[j]);
      ja = j;
    }
  }
  if (e == 0.0f) return 0.0f;
  const float lim = __fmul_rn(e, 1.0f - 1.0f / 2097152.0f);
  int ncand = 0;
#pragma unroll
  for (int j = 0; j < N; ++j) ncand += fabsf(est[j]) >= lim ? 1 : 0;
  float m = __fdiv_rn(xa, __ldg(scale_n + ja));
  if (__builtin_expect(ncand > 1, 0)) {
    // unrolled like the loops above, so x and est stay in registers
#pragma unroll
    for (int j = 0; j < N; ++j)
      if (fabsf(est[j]) >= lim && j != ja) m = fmaxf(m, __fdiv_rn(fabsf(x[j]), __ldg(scale_n + j)));
  }
  return m;
}

// Exact e2m1 magnitude index (0..7 for {0, .5, 1, 1.5, 2, 3, 4, 6}) of P / C,
// P, C >= 0 exact doubles, given an estimate off by at most one: the boundaries
// are the midpoints {.25, .75, 1.25, 1.75, 2.5, 3.5, 5}, a tie goes to the even
// index, and values from 5 up saturate at 6.
static __device__ __noinline__ uint32_t e2m1_index_fix(double P, double C, uint32_t idx) {
  const double mid[7] = {0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0};
  if (idx < 7) {
    const double Q = mid[idx] * C;   // exact: mid has at most 3 significant bits
    if (P > Q || (P == Q && (idx & 1u))) return idx + 1;
  }
  if (idx > 0) {
    const double Q = mid[idx - 1] * C;
    if (P < Q || (P == Q && (idx & 1u))) return idx - 1;
  }
  return idx;
}

// e2m1 codes of 8 elements: the exact round-to-nearest-even of |a_j| g / c_j
// onto the e2m1 grid (saturating at 6; +0 for zero), sign of a_j. v holds the
// fp32 estimates (a fl(1 / c) g, rounded at each step) and a is the raw
// element; c8 points at the 8 divisors (NULL: every c_j = 1). An element is
// re-decided exactly when the estimate scaled by 1 -+ 2^-19 encodes to two
// different codes, i.e. when it lies near a boundary (its error is below
// 2^-21); |a_j| g is exact in double (24 + 24 bits) and so is mid * c_j.
__device__ __forceinline__ uint32_t e2m1x8_exact(const float* v, const float* a, float g,
                                                 const float* c8) {
  float lo[8], hi[8];
  const uint64_t ml = pk2(1.0f - 1.0f / 524288.0f, 1.0f - 1.0f / 524288.0f);
  const uint64_t mh = pk2(1.0f + 1.0f / 524288.0f, 1.0f + 1.0f / 524288.0f);
#pragma unroll
  for (int j = 0; j < 8; j += 2) {
    const uint64_t vv = pk2(v[j], v[j + 1]);
    upk2(fmul2_rn(vv, ml), lo[j], lo[j + 1]);
    upk2(fmul2_rn(vv, mh), hi[j], hi[j + 1]);
  }
  uint32_t out = f32x8_to_e2m1(v);
  const uint32_t wl = f32x8_to_e2m1(lo), wh = f32x8_to_e2m1(hi);
  const uint32_t diff = (wl ^ wh) | (wl ^ out);   // nibbles of the elements near a boundary
  if (__builtin_expect(diff != 0u, 0)) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (((diff >> (4 * j)) & 0xFu) == 0u) continue;
      const uint32_t idx_est = (out >> (4 * j)) & 7u;
      const double P = fabs(static_cast<double>(a[j])) * static_cast<double>(g);
      const double C = c8 != nullptr ? static_cast<double>(__ldg(c8 + j)) : 1.0;
      const uint32_t idx = e2m1_index_fix(P, C, idx_est);
      const uint32_t sign = (a[j] < 0.0f && idx != 0u) ? 8u : 0u;
      out = (out & ~(0xFu << (4 * j))) | ((sign | idx) << (4 * j));
    }
  }
  return out;
}

}  // namespace svdq
