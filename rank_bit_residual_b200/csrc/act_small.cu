// act_small.cu - the activation pass for short batches (B <= 128 rows).
//
// Same result as the large-batch kernel in act.cu ("SVDQuant Smoothing,
// Low-rank and Residual Quantization", Formula items 1 and 3; steps 1-2 of
// "flashinfer.gemm.svdquant_linear"): X_hat = x / scale quantised per tensor
// (INT), per 16-element block (NVFP4) or per 32-element block with a
// power-of-two scale (MXFP4), and the down-projection x ld^T as
// bf16 hi | lo. At decode sizes the whole of x is a few hundred KB, so the work
// is latency-bound: the columns of x are spread over one CTA per SM, and the
// pass is two plain kernels whose boundary replaces a grid barrier (a barrier
// word would need zeroing before every launch, a graph node that costs more
// than the kernels). No TMEM: the down-projection is a handful of warp-level
// MMAs per CTA.
//
//   stats kernel  chunk of x and of ld -> shared memory; column maxima of |x|
//                 divided by scale_k (IEEE) -> one partial maximum per CTA;
//                 partial down-projection of the chunk -> ws_down[g][b][j]
//   codes kernel  launched as a dependent of the stats kernel: loads its chunk
//                 of x while that kernel runs, then takes the per-tensor scale
//                 from the partial maxima, writes the codes of the chunk, and
//                 sums its share of the (b, j) down outputs over the partials
//                 in a fixed order
//
// Rounding as act.cu documents it: one fp32 rounding per stored scalar (s, gs,
// block maxima, sf = ue4m3(fl(fl(amax_b / 6) gs)), enc = fl(gs / sf)), every
// code the exactly rounded value of its quotient (x / (scale_k s) for INT,
// x enc / scale_k or x 2^-X / scale_k onto e2m1), estimated with reciprocals
// r_k = fl(1 / scale_k) and re-decided exactly next to a boundary.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "encode.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace svdq {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kZParts = 8;   // threads that share one down output's sum in phase 2
constexpr int kZBatch = 20;  // partials one thread loads at once (covers 160 CTAs in one batch)

struct SmallArgs {
  int B, M, wc, G, rank_pad, fmt_kind, qmax, has_ld;
  int chained;        // the stats kernel is a programmatic dependent of the previous kernel
  int64_t ldx;
  const void* x;
  const float* scale;
  const float* gs_given;
  const float* gs_w;
  const void* ld;     // [rank_pad][M], x's dtype
  float* ws_max;      // [G] partial maxima
  float* ws_down;     // [G][B][rank_pad] partial down tiles
  void* codes;
  uint8_t* sf;
  __nv_bfloat16* down;
  float* act_scale;
  unsigned* status;
};

// Row pitch (bytes) of a shared-memory chunk of `wc` elements: 16 bytes of
// padding make the 8 rows read by one MMA fragment load hit distinct banks.
__host__ __device__ constexpr int chunk_pitch(int wc, int esz) { return wc * esz + 16; }

template <typename TIn>
__global__ void __launch_bounds__(kThreads, 1) act_small_stats_kernel(const SmallArgs a) {
  constexpr int kEsz = static_cast<int>(sizeof(TIn));
  extern __shared__ __align__(16) uint8_t smem[];
  __shared__ float red[kWarps];

  // the codes kernel launched after this one may start loading x now; when
  // chained after another linear, x is that linear's output: first the
  // weight-side loads, then the wait for the previous kernel, then the trigger
  if (!a.chained) pdl_trigger();

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = blockIdx.x;
  const int c0 = g * a.wc;
  const int ncols = min(a.wc, a.M - c0);     // a multiple of 32
  const int B = a.B;
  const int bp16 = (B + 15) & ~15;
  const int pitch = chunk_pitch(a.wc, kEsz);
  uint8_t* xs = smem;                                               // bp16 rows
  uint8_t* lds = xs + static_cast<size_t>(bp16) * pitch;            // rank_pad rows
  float* scl = reinterpret_cast<float*>(lds + static_cast<size_t>(a.has_ld ? a.rank_pad : 0) * pitch);
  uint32_t* cm = reinterpret_cast<uint32_t*>(scl + a.wc);           // kThreads column-max slots

  // ------------------------------------------------------------ loads
  // weight side (ld, scale) first: it does not depend on the previous kernel
  const int vpr = ncols * kEsz / 16;   // 16-byte vectors per chunk row
  if (a.has_ld) {
    for (int i = tid; i < (bp16 - B) * vpr; i += kThreads) {   // zero rows up to a multiple of 16
      const int r = B + i / vpr, v = i % vpr;
      *reinterpret_cast<uint4*>(xs + r * pitch + v * 16) = make_uint4(0u, 0u, 0u, 0u);
    }
    for (int i = tid; i < a.rank_pad * vpr; i += kThreads) {
      const int r = i / vpr, v = i - r * vpr;
      const uint4 u = __ldg(reinterpret_cast<const uint4*>(
          static_cast<const uint8_t*>(a.ld) + (static_cast<int64_t>(r) * a.M + c0) * kEsz) + v);
      *reinterpret_cast<uint4*>(lds + r * pitch + v * 16) = u;
    }
  }
  for (int k = tid; k < ncols; k += kThreads) scl[k] = __ldg(a.scale + c0 + k);
  if (a.chained) {
    pdl_wait();
    pdl_trigger();
  }
  // x through L2 (it may be the output of the kernel just waited for)
  for (int i = tid; i < B * vpr; i += kThreads) {
    const int r = i / vpr, v = i - r * vpr;
    const uint4 u = __ldcg(reinterpret_cast<const uint4*>(
        static_cast<const uint8_t*>(a.x) + (static_cast<int64_t>(r) * a.ldx + c0) * kEsz) + v);
    *reinterpret_cast<uint4*>(xs + r * pitch + v * 16) = u;
  }
  __syncthreads();

  // ------------------------------------------------- column maxima of |x|
  // thread -> (column, row slice); |x| compared as integers (monotone for
  // non-negative floats), then fl(colmax / scale_k)
  {
    auto abs_bits = [&](int r, int col) -> uint32_t {
      if constexpr (kEsz == 2)
        return static_cast<uint32_t>(*reinterpret_cast<const uint16_t*>(xs + r * pitch + col * 2) & 0x7FFFu) << 16;
      else
        return *reinterpret_cast<const uint32_t*>(xs + r * pitch + col * 4) & 0x7FFFFFFFu;
    };
    float run = 0.0f;
    if (ncols <= kThreads) {
      const int nsl = kThreads / ncols;
      uint32_t m = 0u;
      if (tid < ncols * nsl) {
        const int col = tid % ncols, sl = tid / ncols;
        for (int r = sl; r < B; r += nsl) m = max(m, abs_bits(r, col));
      }
      cm[tid] = m;
      __syncthreads();
      if (tid < ncols) {
        uint32_t mm = 0u;
        for (int sl = 0; sl < nsl; ++sl) mm = max(mm, cm[sl * ncols + tid]);
        run = __fdiv_rn(__uint_as_float(mm), scl[tid]);
      }
    } else {
      for (int col = tid; col < ncols; col += kThreads) {
        uint32_t m = 0u;
        for (int r = 0; r < B; ++r) m = max(m, abs_bits(r, col));
        run = fmaxf(run, __fdiv_rn(__uint_as_float(m), scl[col]));
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) run = fmaxf(run, __shfl_xor_sync(0xffffffffu, run, o));
    if (lane == 0) red[warp] = run;
    __syncthreads();
    if (tid == 0) {
      float t = red[0];
      for (int w = 1; w < kWarps; ++w) t = fmaxf(t, red[w]);
      a.ws_max[g] = t;
    }
  }

  // ------------------------------------------- partial down-projection
  // 16 x 8 output tiles (rows b, factor columns j) spread over the warps; the
  // chunk's columns are the K of each tile's MMA chain
  if (a.has_ld) {
    const int gid = lane >> 2, tig = lane & 3;
    const int mt = bp16 / 16, nt = a.rank_pad / 8, ntile = mt * nt;
    // up to four tiles per warp at a time: their MMAs are independent, so they
    // issue back to back instead of waiting on one accumulator
    for (int t0 = warp; t0 < ntile; t0 += 4 * kWarps) {
      float d[4][4];
#pragma unroll
      for (int q = 0; q < 4; ++q) d[q][0] = d[q][1] = d[q][2] = d[q][3] = 0.0f;
      constexpr int kStep = kEsz == 2 ? 16 : 8;
      for (int k = 0; k < ncols; k += kStep) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int t = t0 + q * kWarps;
          if (t >= ntile) break;
          const int b0 = (t / nt) * 16, j0 = (t % nt) * 8;
          const uint8_t* xa = xs + (b0 + gid) * pitch;
          const uint8_t* xb = xa + 8 * pitch;
          const uint8_t* lb = lds + (j0 + gid) * pitch;
          if constexpr (kEsz == 2) {
            const int o0 = (k + 2 * tig) * 2, o1 = o0 + 16;
            const uint32_t af[4] = {*reinterpret_cast<const uint32_t*>(xa + o0), *reinterpret_cast<const uint32_t*>(xb + o0),
                                    *reinterpret_cast<const uint32_t*>(xa + o1), *reinterpret_cast<const uint32_t*>(xb + o1)};
            const uint32_t bf[2] = {*reinterpret_cast<const uint32_t*>(lb + o0), *reinterpret_cast<const uint32_t*>(lb + o1)};
            mma_bf16_16816(d[q], af, bf);
          } else {
            const int o0 = (k + tig) * 4, o1 = o0 + 16;
            const uint32_t af[4] = {to_tf32(*reinterpret_cast<const uint32_t*>(xa + o0)),
                                    to_tf32(*reinterpret_cast<const uint32_t*>(xb + o0)),
                                    to_tf32(*reinterpret_cast<const uint32_t*>(xa + o1)),
                                    to_tf32(*reinterpret_cast<const uint32_t*>(xb + o1))};
            const uint32_t bf[2] = {to_tf32(*reinterpret_cast<const uint32_t*>(lb + o0)),
                                    to_tf32(*reinterpret_cast<const uint32_t*>(lb + o1))};
            mma_tf32_1688(d[q], af, bf);
          }
        }
      }
      float* base = a.ws_down + static_cast<int64_t>(g) * B * a.rank_pad;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int t = t0 + q * kWarps;
        if (t >= ntile) break;
        const int r0 = (t / nt) * 16 + gid, r1 = r0 + 8, j = (t % nt) * 8 + 2 * tig;
        if (r0 < B) *reinterpret_cast<float2*>(base + static_cast<int64_t>(r0) * a.rank_pad + j) = make_float2(d[q][0], d[q][1]);
        if (r1 < B) *reinterpret_cast<float2*>(base + static_cast<int64_t>(r1) * a.rank_pad + j) = make_float2(d[q][2], d[q][3]);
      }
    }
  }

}

template <typename TIn>
__global__ void __launch_bounds__(kThreads, 1) act_small_codes_kernel(const SmallArgs a) {
  constexpr int kEsz = static_cast<int>(sizeof(TIn));
  extern __shared__ __align__(16) uint8_t smem[];
  __shared__ float red[kWarps];

  pdl_trigger();   // a GEMM launched after this kernel may start its weight loads now

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = blockIdx.x;
  const int c0 = g * a.wc;
  const int ncols = min(a.wc, a.M - c0);     // a multiple of 32
  const int B = a.B;
  const int pitch = chunk_pitch(a.wc, kEsz);
  uint8_t* xs = smem;
  float* rcp = reinterpret_cast<float*>(xs + static_cast<size_t>((B + 15) & ~15) * pitch);

  // x and the scale do not come from the stats kernel: loaded while it runs
  const int vpr = ncols * kEsz / 16;
  for (int i = tid; i < B * vpr; i += kThreads) {
    const int r = i / vpr, v = i - r * vpr;
    const uint4 u = __ldcg(reinterpret_cast<const uint4*>(
        static_cast<const uint8_t*>(a.x) + (static_cast<int64_t>(r) * a.ldx + c0) * kEsz) + v);
    *reinterpret_cast<uint4*>(xs + r * pitch + v * 16) = u;
  }
  for (int k = tid; k < ncols; k += kThreads) rcp[k] = __frcp_rn(__ldg(a.scale + c0 + k));
  pdl_wait();   // the partial maxima and down tiles of every CTA of the stats kernel
  float m = 0.0f;
  for (int i = tid; i < a.G; i += kThreads) m = fmaxf(m, __ldcg(a.ws_max + i));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (lane == 0) red[warp] = m;
  __syncthreads();
  m = red[0];
  for (int w = 1; w < kWarps; ++w) m = fmaxf(m, red[w]);

  const bool nv = a.fmt_kind == SVDQ_KIND_NVFP4;
  const bool mx = a.fmt_kind == SVDQ_KIND_MXFP4;
  float s = 0.0f, u = 0.0f, gs_x = 1.0f;   // MXFP4: no global scale (1)
  if (nv || mx) {
    if (nv) gs_x = a.gs_given != nullptr ? __ldg(a.gs_given) : (m > 0.0f ? __fdiv_rn(2688.0f, m) : 1.0f);
    if (g == 0 && tid == 0) *a.act_scale = gs_x;
  } else {
    s = __fdiv_rn(m, static_cast<float>(a.qmax));
    u = s > 0.0f ? __frcp_rn(s) : 0.0f;
    if (g == 0 && tid == 0) *a.act_scale = s;
  }

  constexpr int kPer16 = 16 / kEsz;   // elements per 16 bytes
  if (!nv && !mx) {
    // 8 codes per item: one 8-byte store
    const int per_row = ncols / 8;
    for (int i = tid; i < B * per_row; i += kThreads) {
      const int r = i / per_row, c8 = (i - r * per_row) * 8;
      float v[8], ck[8];
#pragma unroll
      for (int h = 0; h < 8 / kPer16; ++h)
        unpack16<TIn>(*reinterpret_cast<const uint4*>(xs + r * pitch + (c8 + h * kPer16) * kEsz), v + h * kPer16);
#pragma unroll
      for (int j = 0; j < 8; ++j) ck[j] = __fmul_rn(rcp[c8 + j], u);
      *reinterpret_cast<uint2*>(static_cast<int8_t*>(a.codes) + static_cast<int64_t>(r) * a.M + c0 + c8) =
          int_codes8(v, ck, a.scale + c0 + c8, s, a.qmax);
    }
  } else if (mx) {
    // one 32-element block per item: a scale byte and 16 code bytes
    const int per_row = ncols / 32;
    const int64_t kbp = (a.M / 32 + 3) / 4 * 4;
    for (int i = tid; i < B * per_row; i += kThreads) {
      const int r = i / per_row, c32 = (i - r * per_row) * 32;
      float xr[32], v[32];   // the raw elements and the estimates fl(x r_k)
#pragma unroll
      for (int h = 0; h < 32 / kPer16; ++h)
        unpack16<TIn>(*reinterpret_cast<const uint4*>(xs + r * pitch + (c32 + h * kPer16) * kEsz), xr + h * kPer16);
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] = __fmul_rn(xr[j], rcp[c32 + j]);
      const float* sc32 = a.scale + c0 + c32;
      const int X = mx_block_exponent(block_amax_exact<32>(xr, v, sc32));
      const float enc = mx_inv_scale(X);
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] = __fmul_rn(v[j], enc);
      const int64_t col = c0 + c32;
      *reinterpret_cast<uint4*>(static_cast<uint8_t*>(a.codes) + static_cast<int64_t>(r) * (a.M / 2) + col / 2) =
          make_uint4(e2m1x8_exact(v, xr, enc, sc32), e2m1x8_exact(v + 8, xr + 8, enc, sc32 + 8),
                     e2m1x8_exact(v + 16, xr + 16, enc, sc32 + 16), e2m1x8_exact(v + 24, xr + 24, enc, sc32 + 24));
      a.sf[sf_swizzle_offset(r, col / 32, kbp)] = static_cast<uint8_t>(X + 127);
    }
  } else {
    // one 16-element block per item: a scale byte and 8 code bytes
    const int per_row = ncols / 16;
    const int64_t kbp = (a.M / 16 + 3) / 4 * 4;
    for (int i = tid; i < B * per_row; i += kThreads) {
      const int r = i / per_row, c16 = (i - r * per_row) * 16;
      float xr[16], v[16];   // the raw elements and the estimates fl(x r_k)
#pragma unroll
      for (int h = 0; h < 16 / kPer16; ++h)
        unpack16<TIn>(*reinterpret_cast<const uint4*>(xs + r * pitch + (c16 + h * kPer16) * kEsz), xr + h * kPer16);
#pragma unroll
      for (int j = 0; j < 16; ++j) v[j] = __fmul_rn(xr[j], rcp[c16 + j]);
      const float* sc16 = a.scale + c0 + c16;
      const float amax = block_amax_exact<16>(xr, v, sc16);
      const uint8_t sfb = f32_to_ue4m3(__fmul_rn(__fdiv_rn(amax, 6.0f), gs_x));
      const float dsf = ue4m3_to_f32(sfb);
      const float enc = dsf > 0.0f ? __fdiv_rn(gs_x, dsf) : 0.0f;
#pragma unroll
      for (int j = 0; j < 16; ++j) v[j] = __fmul_rn(v[j], enc);
      const int64_t col = c0 + c16;
      *reinterpret_cast<uint2*>(static_cast<uint8_t*>(a.codes) + static_cast<int64_t>(r) * (a.M / 2) + col / 2) =
          make_uint2(e2m1x8_exact(v, xr, enc, sc16), e2m1x8_exact(v + 8, xr + 8, enc, sc16 + 8));
      a.sf[sf_swizzle_offset(r, col / 16, kbp)] = sfb;
    }
  }
  if (nv || mx) {
    // zero the scale padding: rows B..127 of every scale column, and the
    // columns past M / block (up to a multiple of 4) of rows < B
    const int64_t kb = a.M / (mx ? 32 : 16);
    const int64_t kbp = (kb + 3) / 4 * 4;
    const int64_t pad_cols = kbp - kb;
    const int64_t n_pad = (128 - B) * kbp + static_cast<int64_t>(B) * pad_cols;
    for (int64_t i = static_cast<int64_t>(g) * kThreads + tid; i < n_pad; i += static_cast<int64_t>(a.G) * kThreads) {
      int64_t row, c;
      if (i < static_cast<int64_t>(B) * pad_cols) {
        row = i / pad_cols;
        c = kb + (i - row * pad_cols);
      } else {
        const int64_t j = i - static_cast<int64_t>(B) * pad_cols;
        row = B + j / kbp;
        c = j - (j / kbp) * kbp;
      }
      a.sf[sf_swizzle_offset(row, c, kbp)] = 0;
    }
  }

  // down: this CTA's share of the B * rank_pad outputs; kZParts threads split
  // the G partials of one output (partial z to thread z % kZParts) and their
  // sums are added in thread order: a fixed summation order
  if (a.has_ld) {
    const int total = B * a.rank_pad;
    const int lo = static_cast<int>((static_cast<int64_t>(total) * g) / a.G);
    const int hi = static_cast<int>((static_cast<int64_t>(total) * (g + 1)) / a.G);
    const float mult = nv ? (a.gs_w != nullptr ? __fmul_rn(gs_x, __ldg(a.gs_w)) : gs_x) : 1.0f;
    const int zp = tid % kZParts;
    const int64_t stride = static_cast<int64_t>(B) * a.rank_pad;
    for (int base = lo; base < hi; base += kThreads / kZParts) {
      const int idx = base + tid / kZParts;
      float acc = 0.0f;
      if (idx < hi) {
        // all of this thread's partials are loaded before any is added, so the
        // loads overlap instead of paying the L2 latency one after another
        for (int z0 = zp; z0 < a.G; z0 += kZParts * kZBatch) {
          float v[kZBatch];
#pragma unroll
          for (int u = 0; u < kZBatch; ++u) {
            const int z = z0 + u * kZParts;
            v[u] = z < a.G ? __ldcg(a.ws_down + z * stride + idx) : 0.0f;
          }
#pragma unroll
          for (int u = 0; u < kZBatch; ++u) acc += v[u];
        }
      }
      // fixed-order combine of the kZParts partial sums (lanes zp = 0..7 of a group)
#pragma unroll
      for (int o = 1; o < kZParts; o <<= 1) {
        const float other = __shfl_down_sync(0xffffffffu, acc, o);
        if ((zp & (2 * o - 1)) == 0) acc += other;
      }
      if (zp == 0 && idx < hi) {
        acc = __fmul_rn(acc, mult);
        const int b = idx / a.rank_pad, j = idx - b * a.rank_pad;
        const __nv_bfloat16 h = __float2bfloat16_rn(acc);
        const __nv_bfloat16 l = __float2bfloat16_rn(acc - __bfloat162float(h));
        a.down[static_cast<int64_t>(b) * 2 * a.rank_pad + j] = h;
        a.down[static_cast<int64_t>(b) * 2 * a.rank_pad + a.rank_pad + j] = l;
      }
    }
  }
}

size_t small_smem(const ActPlan& p, bool has_ld) {
  const int esz = p.bf16 ? 2 : 4;
  const int bp16 = static_cast<int>(round_up(p.B, 16));
  return static_cast<size_t>(bp16 + (has_ld ? p.rank_pad : 0)) * chunk_pitch(p.wc, esz) +
         static_cast<size_t>(p.wc) * 4 + kThreads * 4 + 64;
}

// The stats kernel, then the codes kernel as a dependent launch (it may start
// while the stats kernel runs and waits for it with griddepcontrol.wait). Both
// take the largest shared-memory configuration, the one the GEMM launched after
// them needs, so CTAs of the three kernels can share SMs.
template <typename K1, typename K2>
cudaError_t launch_pair_of_kernels(K1 k1, K2 k2, const SmallArgs& a, int grid, size_t smem1, size_t smem2,
                                   cudaStream_t stream) {
  cudaError_t err = cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem1));
  if (err == cudaSuccess)
    err = cudaFuncSetAttribute(k1, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
  if (err == cudaSuccess)
    err = cudaFuncSetAttribute(k2, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem2));
  if (err == cudaSuccess)
    err = cudaFuncSetAttribute(k2, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
  if (err != cudaSuccess) return err;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem1;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = a.chained ? 1 : 0;   // chained: a dependent of the previous kernel too
  err = cudaLaunchKernelEx(&cfg, k1, a);
  if (err != cudaSuccess) return err;
  cfg.dynamicSmemBytes = smem2;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k2, a);
}

}  // namespace

void finish_act_plan_small(ActPlan& p) {
  p.wc = static_cast<int>(round_up(ceil_div(p.M, std::max(p.ksplit, 1)), 32));
  p.grid = static_cast<int>(ceil_div(p.M, p.wc));
  p.ksplit = p.grid;
  p.nunits = p.grid;
  p.nparts = p.grid;
  p.stages = 0;
  p.smem = small_smem(p, p.rank_pad > 0);
}

cudaError_t launch_act_small(const ActPlan& p, const void* x, svdq_dtype xdt, int64_t ldx,
                             const float* scale, svdq_fmt fmt, const float* act_global_scale,
                             const float* w_global_scale, const void* ld, void* codes, void* sf,
                             float* act_scale, void* down, void* scratch, cudaStream_t stream,
                             bool* bad_args) {
  *bad_args = false;
  const bool has_ld = ld != nullptr && p.rank_pad > 0 && down != nullptr;
  const int esz = xdt == SVDQ_BF16 ? 2 : 4;
  if ((reinterpret_cast<uintptr_t>(x) & 15) || (ldx * esz) % 16 ||
      (has_ld && (reinterpret_cast<uintptr_t>(ld) & 15))) {
    *bad_args = true;
    return cudaSuccess;
  }
  Carver cv(scratch, ~size_t(0));
  float* ws_max = static_cast<float*>(cv.take(static_cast<size_t>(p.grid) * 4));
  float* ws_down = has_ld ? static_cast<float*>(cv.take(static_cast<size_t>(p.grid) * p.B * p.rank_pad * 4))
                          : nullptr;
  SmallArgs a{};
  a.B = static_cast<int>(p.B);
  a.M = static_cast<int>(p.M);
  a.wc = p.wc;
  a.G = p.grid;
  a.rank_pad = has_ld ? p.rank_pad : 0;
  a.fmt_kind = fmt.kind;
  a.qmax = fmt.kind == SVDQ_KIND_INT ? (1 << (fmt.bits - 1)) - 1 : 0;
  a.has_ld = has_ld ? 1 : 0;
  a.chained = p.chained;
  a.ldx = ldx;
  a.x = x;
  a.scale = scale;
  a.gs_given = fmt.kind == SVDQ_KIND_NVFP4 ? act_global_scale : nullptr;
  a.gs_w = fmt.kind == SVDQ_KIND_NVFP4 ? w_global_scale : nullptr;
  a.ld = has_ld ? ld : nullptr;
  a.ws_max = ws_max;
  a.ws_down = ws_down;
  a.codes = codes;
  a.sf = static_cast<uint8_t*>(sf);
  a.down = has_ld ? static_cast<__nv_bfloat16*>(down) : nullptr;
  a.act_scale = act_scale;
  a.status = device_status_word();
  const size_t smem1 = small_smem(p, has_ld);
  const size_t smem2 = small_smem(p, false);
  if (xdt == SVDQ_BF16)
    return launch_pair_of_kernels(act_small_stats_kernel<__nv_bfloat16>, act_small_codes_kernel<__nv_bfloat16>, a,
                                  p.grid, smem1, smem2, stream);
  return launch_pair_of_kernels(act_small_stats_kernel<float>, act_small_codes_kernel<float>, a, p.grid, smem1,
                                smem2, stream);
}

}  // namespace svdq
