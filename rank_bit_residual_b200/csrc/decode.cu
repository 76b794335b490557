// decode.cu - the whole SVDQuant linear for one or two rows of x with INT
// weights, in one launch.
//
// "SVDQuant Smoothing, Low-rank and Residual Quantization", Formula items 1-3:
// Y = x ld^T lu^T + s_x s_w (Q(X_hat) . Q(R)), X_hat = x / scale, per-tensor
// INT grid. With one or two rows the activation pass is a few thousand
// elements and the cost of the step is launches and the dependencies between
// them, not the weight stream. So one kernel does everything:
//   1. each CTA copies all of x (8-16 KB, from L2) and the part of ld that is
//      its share of the down-projection into shared memory, then its weight
//      rows (packed 4-bit or int8 codes) and their up-factor rows; the weight
//      copies stay in flight through steps 2-3. (A dependent launch copies
//      the weight side first and waits for the kernel before it only then.)
//   2. the 8 CTAs of a cluster split K: each takes the maximum of |X_hat| and
//      the fp32 down-projection x ld^T over its share, and every CTA combines
//      the 8 partials from distributed shared memory in rank order (the same
//      per-tensor maximum and the same sums everywhere);
//   3. every CTA writes the codes of all of x itself into shared memory
//      (exact rounding as in encode.cuh);
//   4. each warp forms the int32 dot products of its weight rows with the
//      codes (dp4a, lanes split K), then Y = s_x s_w acc + down . lu + bias.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "encode.cuh"
#include "gemm_common.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace svdq {

namespace {

constexpr int kDecThreads = 512;
constexpr int kDecWarps = kDecThreads / 32;
constexpr int kDecCluster = 8;
constexpr int kDecMaxB = 2;
constexpr int kDecRB = 2;                 // weight rows per warp at a time
constexpr uint32_t kDecPiece = 16384;     // bytes per bulk copy of the weight rows
constexpr size_t kDecSmemMax = 200 * 1024;

struct DecodeArgs {
  int B, N, M, rp, rows_per_cta, row_bytes, qmax, chained, kslice;
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

struct DecodeLayout {
  size_t ws, lus, xs, lds, acts, part, down, total;
};

__host__ __device__ inline DecodeLayout decode_layout(int rows, int row_bytes, int B, int M, int rp, int kslice,
                                                      int esz) {
  DecodeLayout L{};
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o = (o + bytes + 15) / 16 * 16;
    return at;
  };
  L.ws = take(static_cast<size_t>(rows) * row_bytes);
  L.lus = take(static_cast<size_t>(rows) * rp * 4);   // whole lu rows (both copies of L2^T)
  L.xs = take(static_cast<size_t>(B) * M * esz);
  L.lds = take(static_cast<size_t>(rp) * kslice * esz);
  L.acts = take(static_cast<size_t>(B) * M);
  L.part = take(static_cast<size_t>(B) * rp * 4);
  L.down = take(static_cast<size_t>(B) * rp * 4);
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

// sum over a 16-byte piece of x times the same piece of an ld row
template <typename TIn>
__device__ __forceinline__ float dot16(uint4 a, uint4 b, float acc) {
  if constexpr (sizeof(TIn) == 2) {
    const uint32_t av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 fa = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&av[i]));
      const float2 fb = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&bv[i]));
      acc = fmaf(fa.x, fb.x, acc);
      acc = fmaf(fa.y, fb.y, acc);
    }
  } else {
    acc = fmaf(__uint_as_float(a.x), __uint_as_float(b.x), acc);
    acc = fmaf(__uint_as_float(a.y), __uint_as_float(b.y), acc);
    acc = fmaf(__uint_as_float(a.z), __uint_as_float(b.z), acc);
    acc = fmaf(__uint_as_float(a.w), __uint_as_float(b.w), acc);
  }
  return acc;
}

template <typename TIn, bool kPacked, int kOut>
__global__ void __launch_bounds__(kDecThreads, 1) decode_kernel(const DecodeArgs g) {
  constexpr int kEsz = static_cast<int>(sizeof(TIn));
  constexpr int kPer16 = 16 / kEsz;
  extern __shared__ __align__(16) uint8_t dsm[];
  __shared__ float red[kDecWarps];
  __shared__ float pmax;
  __shared__ __align__(8) uint64_t bar[2];   // 0: x and the ld share, 1: weight and lu rows
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int crank = static_cast<int>(cluster_ctarank());
  const int n0 = blockIdx.x * g.rows_per_cta;
  const int rows = max(0, min(g.rows_per_cta, g.N - n0));
  const DecodeLayout L = decode_layout(g.rows_per_cta, g.row_bytes, g.B, g.M, g.rp, g.kslice, kEsz);
  uint8_t* ws = dsm + L.ws;
  uint8_t* lus = dsm + L.lus;
  uint8_t* xs = dsm + L.xs;
  uint8_t* lds = dsm + L.lds;
  int8_t* acts = reinterpret_cast<int8_t*>(dsm + L.acts);
  float* part = reinterpret_cast<float*>(dsm + L.part);
  float* down = reinterpret_cast<float*>(dsm + L.down);
  const int k0 = min(g.M, crank * g.kslice), k1 = min(g.M, k0 + g.kslice);
  if (tid == 0) {
    mbar_init(&bar[0], 1);
    mbar_init(&bar[1], 1);
    fence_mbar_init();
  }
  __syncthreads();
  // a chained linear queued after this kernel may start its weight-side setup
  // now (it reads this kernel's output only after griddepcontrol.wait)
  pdl_trigger();

  // ---- 1. warp 0 issues every copy as bulk copies: x and the ld share on
  // bar[0], the weight rows (in 16 KB pieces over the lanes) and the lu rows on
  // bar[1]; all rows of a CTA are contiguous in global memory
  if (warp == 0) {
    auto issue_x = [&]() {
      const uint32_t share = static_cast<uint32_t>(k1 - k0) * kEsz;
      if (lane == 0)
        mbar_arrive_expect_tx(&bar[0], static_cast<uint32_t>(g.B * g.M * kEsz) + static_cast<uint32_t>(g.rp) * share);
      __syncwarp();
      for (int b = lane; b < g.B; b += 32)
        bulk_load(xs + static_cast<size_t>(b) * g.M * kEsz,
                  static_cast<const uint8_t*>(g.x) + static_cast<int64_t>(b) * g.ldx * kEsz,
                  static_cast<uint32_t>(g.M * kEsz), &bar[0]);
      if (share > 0)
        for (int j = lane; j < g.rp; j += 32)
          bulk_load(lds + static_cast<size_t>(j) * g.kslice * kEsz,
                    static_cast<const uint8_t*>(g.ld) + (static_cast<int64_t>(j) * g.M + k0) * kEsz, share, &bar[0]);
    };
    auto issue_w = [&]() {
      const uint32_t wtot = static_cast<uint32_t>(rows) * static_cast<uint32_t>(g.row_bytes);
      const uint32_t ltot = static_cast<uint32_t>(rows) * static_cast<uint32_t>(g.rp) * 4u;
      if (lane == 0) mbar_arrive_expect_tx(&bar[1], wtot + ltot);
      __syncwarp();
      const uint32_t pieces = (wtot + kDecPiece - 1) / kDecPiece;
      for (uint32_t p = lane; p < pieces; p += 32)
        bulk_load(ws + static_cast<size_t>(p) * kDecPiece,
                  g.w + static_cast<int64_t>(n0) * g.row_bytes + static_cast<int64_t>(p) * kDecPiece,
                  min(kDecPiece, wtot - p * kDecPiece), &bar[1]);
      if (ltot > 0 && lane == 31)
        bulk_load(lus, reinterpret_cast<const uint8_t*>(g.lu) + static_cast<int64_t>(n0) * g.rp * 4, ltot, &bar[1]);
    };
    // a chained launch (x is the previous linear's output) starts the weight
    // side before it waits for that kernel; otherwise x goes first, so the
    // activation arithmetic overlaps the weight stream
    if (g.chained) {
      issue_w();
      pdl_wait();
      issue_x();
    } else {
      issue_x();
      issue_w();
    }
  }
  // a wait that gives up records the timeout in g.status; the kernel then runs
  // to the end (every CTA must reach both cluster barriers)
  mbar_wait_warp(&bar[0], 0, g.status, nullptr);

  // ---- 2. this CTA's share of K: maximum of |X_hat| (IEEE quotients of the
  // column maxima) and the down-projection (8 lanes per output, 16-byte pieces)
  float m = 0.0f;
  for (int c = k0 + tid; c < k1; c += kDecThreads) {
    float cm = 0.0f;
    for (int b = 0; b < g.B; ++b) cm = fmaxf(cm, fabsf(to_f<TIn>(xs, b * g.M + c)));
    m = fmaxf(m, __fdiv_rn(cm, __ldg(g.scale + c)));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (lane == 0) red[warp] = m;
  const int nout = g.B * g.rp;
  const int nvec = (k1 - k0) / kPer16;
  for (int base = 0; base < nout * 8; base += kDecThreads) {
    const int idx = base + tid;
    const bool act = idx < nout * 8;
    const int o = idx >> 3, sub = idx & 7;
    float acc = 0.0f;
    if (act) {
      const int b = o / g.rp, j = o - b * g.rp;
      const uint32_t xa = smem_u32(xs + (static_cast<size_t>(b) * g.M + k0) * kEsz);
      const uint32_t la = smem_u32(lds + static_cast<size_t>(j) * g.kslice * kEsz);
      for (int v = sub; v < nvec; v += 8) acc = dot16<TIn>(ld_shared_v4(xa + 16 * v), ld_shared_v4(la + 16 * v), acc);
    }
    acc += __shfl_xor_sync(0xffffffffu, acc, 4);
    acc += __shfl_xor_sync(0xffffffffu, acc, 2);
    acc += __shfl_xor_sync(0xffffffffu, acc, 1);
    if (act && sub == 0) part[o] = acc;
  }
  __syncthreads();
  if (tid == 0) {
    float mm = red[0];
    for (int w = 1; w < kDecWarps; ++w) mm = fmaxf(mm, red[w]);
    pmax = mm;
  }
  cluster_sync();   // every CTA's partial maximum and down tile are written
  for (int o = tid; o < nout; o += kDecThreads) {
    float sum = 0.0f;
    for (int r = 0; r < kDecCluster; ++r) sum += ld_cluster_f32(mapa_shared(smem_u32(part + o), r));
    down[o] = sum;
  }
  m = 0.0f;
  for (int r = 0; r < kDecCluster; ++r) m = fmaxf(m, ld_cluster_f32(mapa_shared(smem_u32(&pmax), r)));
  const float s = __fdiv_rn(m, static_cast<float>(g.qmax));
  const float u = s > 0.0f ? __frcp_rn(s) : 0.0f;

  // ---- 3. codes of all of x, 8 columns per item
  for (int i = tid; i < g.B * (g.M / 8); i += kDecThreads) {
    const int b = i / (g.M / 8), c0 = (i - b * (g.M / 8)) * 8;
    float v[8], ck[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      v[j] = to_f<TIn>(xs, b * g.M + c0 + j);
      ck[j] = __fmul_rn(__frcp_rn(__ldg(g.scale + c0 + j)), u);
    }
    *reinterpret_cast<uint2*>(acts + static_cast<size_t>(b) * g.M + c0) = int_codes8(v, ck, g.scale + c0, s, g.qmax);
  }
  mbar_wait_warp(&bar[1], 0, g.status, nullptr);   // the weight and lu rows
  __syncthreads();                                 // the codes and down sums

  // ---- 4. dot products of this CTA's weight rows with the codes; the lanes
  // split K, then the up-projection over the lanes and Y = s_x s_w acc + up + bias
  const float alpha = s * __ldg(g.s_w);
  constexpr int kK = kPacked ? 32 : 16;   // codes per 16-byte weight chunk
  const int nchunks = g.row_bytes / 16;
  for (int r0 = warp * kDecRB; r0 < rows; r0 += kDecWarps * kDecRB) {
    int acc[kDecRB][kDecMaxB];
#pragma unroll
    for (int i = 0; i < kDecRB; ++i)
#pragma unroll
      for (int b = 0; b < kDecMaxB; ++b) acc[i][b] = 0;
    for (int j = lane; j < nchunks; j += 32) {
      uint32_t w8[kDecRB][kK / 4];
#pragma unroll
      for (int i = 0; i < kDecRB; ++i) {
        const int r = min(r0 + i, rows - 1);   // rows past the end repeat the last (not stored)
        const uint4 wv = ld_shared_v4(smem_u32(ws + static_cast<size_t>(r) * g.row_bytes + 16 * j));
        if constexpr (kPacked) {
          widen_int4(wv, *reinterpret_cast<uint32_t(*)[8]>(w8[i]));
        } else {
          w8[i][0] = wv.x; w8[i][1] = wv.y; w8[i][2] = wv.z; w8[i][3] = wv.w;
        }
      }
#pragma unroll
      for (int b = 0; b < kDecMaxB; ++b) {
        if (b >= g.B) break;
        const uint32_t abase = smem_u32(acts + static_cast<size_t>(b) * g.M + kK * j);
#pragma unroll
        for (int h = 0; h < kK / 16; ++h) {
          const uint4 av = ld_shared_v4(abase + 16 * h);
#pragma unroll
          for (int i = 0; i < kDecRB; ++i) {
            acc[i][b] = __dp4a(static_cast<int>(w8[i][4 * h + 0]), static_cast<int>(av.x), acc[i][b]);
            acc[i][b] = __dp4a(static_cast<int>(w8[i][4 * h + 1]), static_cast<int>(av.y), acc[i][b]);
            acc[i][b] = __dp4a(static_cast<int>(w8[i][4 * h + 2]), static_cast<int>(av.z), acc[i][b]);
            acc[i][b] = __dp4a(static_cast<int>(w8[i][4 * h + 3]), static_cast<int>(av.w), acc[i][b]);
          }
        }
      }
    }
#pragma unroll
    for (int i = 0; i < kDecRB; ++i) {
      const int r = r0 + i;
      if (r >= rows) break;
      const int n = n0 + r;
      const __nv_bfloat16* lr = reinterpret_cast<const __nv_bfloat16*>(lus + static_cast<size_t>(r) * g.rp * 4);
      const float bn = g.bias != nullptr ? __bfloat162float(g.bias[n]) : 0.0f;
#pragma unroll
      for (int b = 0; b < kDecMaxB; ++b) {
        if (b >= g.B) break;
        int v = acc[i][b];
        float up = 0.0f;
        for (int q = lane; q < g.rp; q += 32) up = fmaf(down[b * g.rp + q], __bfloat162float(lr[q]), up);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          v += __shfl_xor_sync(0xffffffffu, v, o);
          up += __shfl_xor_sync(0xffffffffu, up, o);
        }
        if (lane == 0) {
          const float yv = alpha * static_cast<float>(v) + up + bn;
          if constexpr (kOut == kOutF32)
            static_cast<float*>(g.y)[static_cast<int64_t>(b) * g.ldy + n] = yv;
          else
            static_cast<__nv_bfloat16*>(g.y)[static_cast<int64_t>(b) * g.ldy + n] = __float2bfloat16_rn(yv);
        }
      }
    }
  }
  cluster_sync();   // no CTA leaves while another may still read its partial
}

template <typename TIn, bool kPacked, int kOut>
cudaError_t launch_decode_one(const DecodeArgs& g, int grid, size_t smem, bool pdl, cudaStream_t st) {
  auto kern = decode_kernel<TIn, kPacked, kOut>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (err != cudaSuccess) return err;
  err = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
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
  const int row_bytes = static_cast<int>(packed ? M / 2 : M);
  const int rows = static_cast<int>(round_up(ceil_div(N, num_sms()), 8));
  const int grid = static_cast<int>(round_up(ceil_div(N, rows), kDecCluster));
  // each CTA's share of the down-projection: whole 16-byte pieces of an ld row
  const int kslice = static_cast<int>(round_up(ceil_div(M, kDecCluster), 16 / esz));
  const DecodeLayout L = decode_layout(rows, row_bytes, static_cast<int>(B), static_cast<int>(M), rp, kslice, esz);
  if (L.total > kDecSmemMax) return false;
  for (const void* q : {static_cast<const void*>(packed ? w->codes4 : w->codes), x, ld,
                        static_cast<const void*>(w->lu), bias})
    if (q != nullptr && (reinterpret_cast<uintptr_t>(q) & 15) != 0) return false;
  if ((ldx * esz) % 16 != 0) return false;
  DecodeArgs g{};
  g.B = static_cast<int>(B);
  g.N = static_cast<int>(N);
  g.M = static_cast<int>(M);
  g.rp = rp;
  g.rows_per_cta = rows;
  g.row_bytes = row_bytes;
  g.qmax = (1 << (w->fmt.bits - 1)) - 1;
  g.chained = chained ? 1 : 0;
  g.kslice = kslice;
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
#define SVDQ_DEC(T, P, O) *err = launch_decode_one<T, P, O>(g, grid, L.total, chained, st)
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
