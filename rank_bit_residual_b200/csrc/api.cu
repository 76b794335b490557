// api.cu - the C ABI of include/svdq.h: argument checks, workspace carving,
// tensor-map encoding and kernel launches. No call here allocates device
// memory; every buffer comes from the caller.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <mutex>

#include "internal.h"
#include "ptx.cuh"

namespace svdq {

namespace {

__device__ unsigned g_status_word;

constexpr int kMaxDevices = 64;
std::mutex g_mu;
unsigned* g_status_ptr[kMaxDevices] = {};
int g_sms[kMaxDevices] = {};

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

int current_device() {
  int d = 0;
  if (cudaGetDevice(&d) != cudaSuccess || d < 0 || d >= kMaxDevices) return 0;
  return d;
}

}  // namespace

unsigned* device_status_word() {
  const int d = current_device();
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_status_ptr[d]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_status_word) == cudaSuccess)
      g_status_ptr[d] = static_cast<unsigned*>(p);
  }
  return g_status_ptr[d];
}

int num_sms() {
  const int d = current_device();
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_sms[d]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, d) != cudaSuccess || n <= 0)
      n = 148;
    g_sms[d] = n;
  }
  return g_sms[d];
}

bool make_tmap_2d(CUtensorMap* map, const void* base, CUtensorMapDataType dtype, int elem_bytes,
                  uint64_t inner, uint64_t outer, uint64_t ld_elems, uint32_t box_inner,
                  uint32_t box_outer, bool swizzle128) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || base == nullptr) return false;
  if ((reinterpret_cast<uintptr_t>(base) & 15) != 0) return false;
  if ((ld_elems * elem_bytes) % 16 != 0 || inner == 0 || outer == 0) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {ld_elems * static_cast<uint64_t>(elem_bytes)};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  const CUresult r =
      fn(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
         CU_TENSOR_MAP_INTERLEAVE_NONE,
         swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

namespace {

__global__ void wait_selftest_kernel(long long limit_ns, unsigned* status) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 2);  // two arrivals expected, only one ever comes
    fence_mbar_init();
    mbar_arrive(&bar);
    mbar_wait(&bar, 0, status, nullptr, static_cast<unsigned long long>(limit_ns));
  }
}

svdq_status check_fmt(svdq_fmt fmt) {
  if (fmt.kind == SVDQ_KIND_INT) return (fmt.bits >= 2 && fmt.bits <= 8) ? SVDQ_OK : SVDQ_EINVAL;
  if (fmt.kind == SVDQ_KIND_NVFP4 || fmt.kind == SVDQ_KIND_MXFP4) return fmt.bits == 4 ? SVDQ_OK : SVDQ_EINVAL;
  return SVDQ_EINVAL;
}

// Layout and rank checks of "_check_smoothing" / "_check_rank", then this
// library's own limits.
svdq_status check_shape(int64_t M, int64_t N, int32_t rank, svdq_fmt fmt) {
  if (M <= 0 || N <= 0) return SVDQ_EINVAL;
  if (rank < 0 || rank > std::min(M, N)) return SVDQ_ERANK;
  const svdq_status f = check_fmt(fmt);
  if (f != SVDQ_OK) return f;
  if (M % 32 != 0 || N % 16 != 0) return SVDQ_EUNSUPPORTED;
  if (rank > 256) return SVDQ_EUNSUPPORTED;
  if (M > (int64_t(1) << 30) || N > (int64_t(1) << 30)) return SVDQ_EUNSUPPORTED;
  return SVDQ_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

svdq_status from_cuda(cudaError_t e) { return e == cudaSuccess ? SVDQ_OK : SVDQ_ECUDA; }

size_t al256(size_t b) { return (b + 255) / 256 * 256; }

size_t act_codes_bytes(int64_t B, int64_t M, svdq_fmt fmt) {
  return fmt.kind == SVDQ_KIND_INT ? static_cast<size_t>(B * M) : static_cast<size_t>(B * M / 2);
}

// Block-scale bytes of a [rows, M] fp4 operand: the 128x4 layout over
// [rows, M / block], block 16 (NVFP4) or 32 (MXFP4); 0 for INT.
size_t fp4_sf_bytes(int64_t rows, int64_t M, svdq_fmt fmt) {
  if (fmt.kind == SVDQ_KIND_INT) return 0;
  const int64_t block = fmt.kind == SVDQ_KIND_MXFP4 ? 32 : 16;
  return static_cast<size_t>(round_up(rows, 128) * round_up(M / block, 4));
}

svdq_status check_weight(const svdq_weight* w) {
  if (!w) return SVDQ_EINVAL;
  const svdq_status s = check_shape(w->M, w->N, w->rank, w->fmt);
  if (s != SVDQ_OK) return s;
  if (w->rank_pad != rank_pad_of(w->rank)) return SVDQ_EINVAL;
  if (!w->codes || !w->w_scale || !w->scale) return SVDQ_EINVAL;
  if (w->fmt.kind != SVDQ_KIND_INT && !w->sf) return SVDQ_EINVAL;
  if (w->rank > 0 && (!w->ld || !w->lu)) return SVDQ_EINVAL;
  if (w->codes4 && (w->fmt.kind != SVDQ_KIND_INT || w->fmt.bits > 4)) return SVDQ_EINVAL;
  if (!aligned16(w->codes) || !aligned16(w->scale) || (w->ld && !aligned16(w->ld)) ||
      (w->codes4 && !aligned16(w->codes4)) ||
      (w->lu && !aligned16(w->lu)) || (w->ld32 && !aligned16(w->ld32)))
    return SVDQ_EUNSUPPORTED;
  return SVDQ_OK;
}

svdq_status check_act_input(const void* x, svdq_dtype dt, int64_t B, int64_t M, int64_t ldx) {
  if (B < 0 || M <= 0) return SVDQ_EINVAL;
  if (dt != SVDQ_BF16 && dt != SVDQ_F32) return SVDQ_EINVAL;
  if (B == 0) return SVDQ_OK;
  if (!x || ldx < M) return SVDQ_EINVAL;
  const int esz = dt == SVDQ_BF16 ? 2 : 4;
  if (!aligned16(x) || (ldx * esz) % 16 != 0) return SVDQ_EUNSUPPORTED;
  if (B > (int64_t(1) << 30)) return SVDQ_EUNSUPPORTED;
  return SVDQ_OK;
}

struct LinearCarve {
  void* codes;
  void* sf;
  float* act_scale;
  void* down;
  void* act_scratch;
  void* split;
  size_t bytes;
  bool ok;
};

LinearCarve carve_linear(const svdq_weight* w, int64_t B, void* ws, size_t ws_bytes,
                         svdq_dtype xdt) {
  const ActPlan p = plan_act(B, w->M, w->rank_pad, xdt);
  Carver cv(ws, ws_bytes);
  LinearCarve c{};
  c.codes = cv.take(act_codes_bytes(B, w->M, w->fmt));
  c.sf = cv.take(fp4_sf_bytes(B, w->M, w->fmt));
  c.act_scale = static_cast<float*>(cv.take(16));
  c.down = cv.take(static_cast<size_t>(B) * 2 * w->rank_pad * 2);
  c.act_scratch = cv.take(act_scratch_bytes(p));
  // the pair GEMM's K split of its last round (INT, more than 128 rows)
  const size_t split = (w->fmt.kind == SVDQ_KIND_INT && B > 128) ? pair_split_bytes(B, w->M, w->N) : 0;
  c.split = split > 0 ? cv.take(split) : nullptr;
  c.bytes = cv.off;
  c.ok = cv.ok;
  return c;
}

}  // namespace

svdq_status check_quantize_act_args(const void* x, svdq_dtype x_dtype, int64_t B, int64_t M, int64_t ldx,
                                    const float* scale, svdq_fmt fmt, const void* ld, int32_t rank_pad,
                                    const void* codes, const void* sf, const float* act_scale,
                                    const void* down) {
  svdq_status s = check_act_input(x, x_dtype, B, M, ldx);
  if (s != SVDQ_OK) return s;
  if (check_fmt(fmt) != SVDQ_OK || !scale || rank_pad < 0 || rank_pad % 16 || rank_pad > 256)
    return SVDQ_EINVAL;
  if (M % 32 != 0) return SVDQ_EUNSUPPORTED;
  if (!aligned16(scale)) return SVDQ_EUNSUPPORTED;
  if (B == 0) return SVDQ_OK;
  if (!codes || !act_scale || (fmt.kind != SVDQ_KIND_INT && !sf)) return SVDQ_EINVAL;
  if (ld && rank_pad > 0 && (!down || !aligned16(ld))) return SVDQ_EINVAL;
  // the codes and the down tile are written in 8- and 16-byte pieces
  if (!aligned16(codes) || (ld && rank_pad > 0 && !aligned16(down))) return SVDQ_EUNSUPPORTED;
  return SVDQ_OK;
}

}  // namespace svdq

using namespace svdq;

extern "C" {

const char* svdq_version(void) { return "0.1.0"; }

const char* svdq_status_string(svdq_status s) {
  switch (s) {
    case SVDQ_OK: return "ok";
    case SVDQ_EINVAL: return "invalid argument (layout, scale or format)";
    case SVDQ_ERANK: return "rank outside [0, min(M, N)]";
    case SVDQ_EUNSUPPORTED: return "shape, alignment or rank outside this library's limits";
    case SVDQ_ECUDA: return "CUDA runtime error";
    case SVDQ_ETIMEOUT: return "a bounded device wait ran out";
    case SVDQ_EWORKSPACE: return "workspace missing or too small";
  }
  return "unknown status";
}

svdq_status svdq_weight_buffer_sizes(int64_t M, int64_t N, int32_t rank, svdq_fmt fmt,
                                     size_t sizes[7]) {
  if (!sizes) return SVDQ_EINVAL;
  const svdq_status s = check_shape(M, N, rank, fmt);
  if (s != SVDQ_OK) return s;
  const int64_t rp = rank_pad_of(rank);
  sizes[0] = fmt.kind == SVDQ_KIND_INT ? static_cast<size_t>(N * M) : static_cast<size_t>(N * M / 2);
  sizes[1] = fp4_sf_bytes(N, M, fmt);
  sizes[2] = sizeof(float);
  sizes[3] = static_cast<size_t>(rp * M * 2);
  sizes[4] = static_cast<size_t>(rp * M * 4);
  sizes[5] = static_cast<size_t>(N * 2 * rp * 2);
  sizes[6] = fmt.kind == SVDQ_KIND_INT && fmt.bits <= 4 ? static_cast<size_t>(N * M / 2) : 0;
  return SVDQ_OK;
}

svdq_status svdq_pack_int4(const int8_t* codes, int64_t N, int64_t M, uint8_t* packed,
                           svdq_stream_t stream) {
  if (N <= 0 || M <= 0 || !codes || !packed) return SVDQ_EINVAL;
  if (M % 32 != 0 || !aligned16(codes) || !aligned16(packed)) return SVDQ_EUNSUPPORTED;
  return from_cuda(launch_pack_int4(codes, N, M, packed, reinterpret_cast<cudaStream_t>(stream)));
}

svdq_status svdq_prepare_workspace_size(int64_t M, int64_t N, int32_t rank, svdq_fmt fmt,
                                        int32_t oversample, size_t* bytes) {
  if (!bytes) return SVDQ_EINVAL;
  const svdq_status s = check_shape(M, N, rank, fmt);
  if (s != SVDQ_OK) return s;
  *bytes = prepare_scratch_bytes(M, N, rank, oversample);
  return SVDQ_OK;
}

svdq_status svdq_prepare(const void* W, svdq_dtype w_dtype, int64_t M, int64_t N, int64_t ldW,
                         const float* scale, int32_t rank, svdq_fmt fmt, uint64_t seed,
                         int32_t oversample, int32_t power_iters, void* workspace,
                         size_t workspace_bytes, svdq_weight* out, svdq_stream_t stream) {
  const svdq_status s = check_shape(M, N, rank, fmt);
  if (s != SVDQ_OK) return s;
  if (!W || !scale || !out || ldW < N || (w_dtype != SVDQ_BF16 && w_dtype != SVDQ_F32))
    return SVDQ_EINVAL;
  if (!aligned16(scale)) return SVDQ_EUNSUPPORTED;
  if (!out->codes || !out->w_scale || (fmt.kind != SVDQ_KIND_INT && !out->sf) ||
      (rank > 0 && (!out->ld || !out->lu)))
    return SVDQ_EINVAL;
  // the weight's buffers are written (and later read) in 16-byte pieces
  if (!aligned16(out->codes) || (out->codes4 && !aligned16(out->codes4)) || (out->sf && !aligned16(out->sf)) ||
      (out->ld && !aligned16(out->ld)) || (out->ld32 && !aligned16(out->ld32)) || (out->lu && !aligned16(out->lu)))
    return SVDQ_EUNSUPPORTED;
  if (!workspace || workspace_bytes < prepare_scratch_bytes(M, N, rank, oversample))
    return SVDQ_EWORKSPACE;
  return run_prepare(W, w_dtype, M, N, ldW, scale, rank, fmt, seed, oversample, power_iters,
                     workspace, workspace_bytes, out, reinterpret_cast<cudaStream_t>(stream));
}

svdq_status svdq_quantize_residual_workspace_size(int64_t M, int64_t N, svdq_fmt fmt,
                                                  size_t* bytes) {
  if (!bytes) return SVDQ_EINVAL;
  const svdq_status s = check_shape(M, N, 0, fmt);
  if (s != SVDQ_OK) return s;
  *bytes = residual_scratch_bytes(M, N);
  return SVDQ_OK;
}

svdq_status svdq_quantize_residual(const float* R, int64_t M, int64_t N, int64_t ldR,
                                   svdq_fmt fmt, void* codes, void* sf, float* w_scale,
                                   void* workspace, size_t workspace_bytes,
                                   svdq_stream_t stream) {
  const svdq_status s = check_shape(M, N, 0, fmt);
  if (s != SVDQ_OK) return s;
  if (!R || ldR < N || !codes || !w_scale || (fmt.kind != SVDQ_KIND_INT && !sf))
    return SVDQ_EINVAL;
  if (!aligned16(codes)) return SVDQ_EUNSUPPORTED;   // fp4 codes go out 8 and 16 bytes at a time
  if (!workspace || workspace_bytes < residual_scratch_bytes(M, N)) return SVDQ_EWORKSPACE;
  return from_cuda(launch_quantize_residual(R, M, N, ldR, fmt, codes, sf, w_scale, workspace,
                                            reinterpret_cast<cudaStream_t>(stream)));
}

svdq_status svdq_quantize_act_workspace_size(int64_t B, int64_t M, svdq_fmt fmt, int32_t rank_pad,
                                             size_t* bytes) {
  if (!bytes || B < 0 || M <= 0 || rank_pad < 0 || rank_pad % 16 || rank_pad > 256)
    return SVDQ_EINVAL;
  if (check_fmt(fmt) != SVDQ_OK) return SVDQ_EINVAL;
  *bytes = act_scratch_bytes(plan_act(B, M, rank_pad, SVDQ_BF16));
  const size_t b32 = act_scratch_bytes(plan_act(B, M, rank_pad, SVDQ_F32));
  *bytes = std::max(*bytes, b32);
  return SVDQ_OK;
}

svdq_status svdq_quantize_act(const void* x, svdq_dtype x_dtype, int64_t B, int64_t M,
                              int64_t ldx, const float* scale, svdq_fmt fmt,
                              const float* act_global_scale, const float* w_global_scale,
                              const void* ld, int32_t rank_pad,
                              void* codes, void* sf, float* act_scale, void* down,
                              void* workspace, size_t workspace_bytes, svdq_stream_t stream) {
  const svdq_status s = check_quantize_act_args(x, x_dtype, B, M, ldx, scale, fmt, ld, rank_pad, codes,
                                                sf, act_scale, down);
  if (s != SVDQ_OK || B == 0) return s;
  const ActPlan p = plan_act(B, M, rank_pad, x_dtype);
  if (!workspace || workspace_bytes < act_scratch_bytes(p)) return SVDQ_EWORKSPACE;
  bool bad = false;
  const cudaError_t e =
      launch_act(p, x, x_dtype, ldx, scale, fmt, act_global_scale,
                 fmt.kind == SVDQ_KIND_NVFP4 ? w_global_scale : nullptr,
                 rank_pad > 0 ? ld : nullptr, codes, sf, act_scale, down, workspace,
                 reinterpret_cast<cudaStream_t>(stream), &bad);
  if (bad) return SVDQ_EUNSUPPORTED;
  return from_cuda(e);
}

svdq_status svdq_linear_workspace_size(const svdq_weight* w, int64_t B, size_t* bytes) {
  if (!bytes || B < 0) return SVDQ_EINVAL;
  const svdq_status s = check_weight(w);
  if (s != SVDQ_OK) return s;
  const size_t a = carve_linear(w, B, nullptr, 0, SVDQ_BF16).bytes;
  const size_t b = carve_linear(w, B, nullptr, 0, SVDQ_F32).bytes;
  *bytes = std::max(a, b);
  return SVDQ_OK;
}

svdq_status svdq_linear(const svdq_weight* w, const void* x, svdq_dtype x_dtype, int64_t B,
                        int64_t ldx, const void* bias, const float* act_global_scale, void* y,
                        svdq_dtype y_dtype, int64_t ldy, void* workspace, size_t workspace_bytes,
                        svdq_stream_t stream) {
  return svdq_linear_ex(w, x, x_dtype, B, ldx, bias, act_global_scale, y, y_dtype, ldy, workspace,
                        workspace_bytes, 0u, stream);
}

svdq_status svdq_linear_ex(const svdq_weight* w, const void* x, svdq_dtype x_dtype, int64_t B,
                           int64_t ldx, const void* bias, const float* act_global_scale, void* y,
                           svdq_dtype y_dtype, int64_t ldy, void* workspace, size_t workspace_bytes,
                           uint32_t flags, svdq_stream_t stream) {
  if (flags & ~SVDQ_LINEAR_PDL) return SVDQ_EINVAL;
  svdq_status s = check_weight(w);
  if (s != SVDQ_OK) return s;
  s = check_act_input(x, x_dtype, B, w->M, ldx);
  if (s != SVDQ_OK) return s;
  if (y_dtype != SVDQ_BF16 && y_dtype != SVDQ_F32) return SVDQ_EINVAL;
  if (B == 0) return SVDQ_OK;
  if (!y || ldy < w->N) return SVDQ_EINVAL;
  if (bias && !aligned16(bias)) return SVDQ_EUNSUPPORTED;
  const void* ld = x_dtype == SVDQ_BF16 ? w->ld : w->ld32;
  if (w->rank > 0 && !ld) return SVDQ_EINVAL;
  LinearCarve c = carve_linear(w, B, workspace, workspace_bytes, x_dtype);
  if (!c.ok) return SVDQ_EWORKSPACE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // up to 16 rows with INT weights: the whole linear in one launch (when its
  // shared memory holds the CTA's weight rows and the codes of x)
  {
    cudaError_t e = cudaSuccess;
    if (launch_decode(w, x, x_dtype, B, ldx, bias, y, y_dtype, ldy, (flags & SVDQ_LINEAR_PDL) != 0, st, &e))
      return from_cuda(e);
  }
  ActPlan p = plan_act(B, w->M, w->rank_pad, x_dtype);
  p.chained = (flags & SVDQ_LINEAR_PDL) ? 1 : 0;
  bool bad = false;
  // the pair GEMM's split counters are cleared by the activation pass
  unsigned* zero = c.split != nullptr
                       ? reinterpret_cast<unsigned*>(static_cast<uint8_t*>(c.split) +
                                                     pair_split_counter_offset(B, w->M, w->N))
                       : nullptr;
  cudaError_t e = launch_act(p, x, x_dtype, ldx, w->scale, w->fmt, act_global_scale,
                             w->fmt.kind == SVDQ_KIND_NVFP4 ? w->w_scale : nullptr,
                             w->rank > 0 ? ld : nullptr, c.codes, c.sf, c.act_scale,
                             w->rank > 0 ? c.down : nullptr, c.act_scratch, st, &bad, zero,
                             zero != nullptr ? pair_split_counters(B, w->M, w->N) : 0);
  if (bad) return SVDQ_EUNSUPPORTED;
  if (e != cudaSuccess) return SVDQ_ECUDA;
  if (w->fmt.kind == SVDQ_KIND_INT) {
    e = launch_gemm_int(w, static_cast<const int8_t*>(c.codes), c.act_scale,
                        w->rank > 0 ? c.down : nullptr, B, bias, y, y_dtype, ldy, false, true, st, &bad,
                        c.split);
  } else {
    e = launch_gemm_fp4(w, static_cast<const uint8_t*>(c.codes),
                          static_cast<const uint8_t*>(c.sf), c.act_scale,
                          w->rank > 0 ? c.down : nullptr, B, bias, y, y_dtype, ldy, true, st, &bad);
  }
  if (bad) return SVDQ_EUNSUPPORTED;
  return from_cuda(e);
}

svdq_status svdq_residual_linear(const svdq_weight* w, const void* act_codes, const void* act_sf,
                                 const float* act_scale, const void* down, int64_t B,
                                 const void* bias, void* y, svdq_dtype y_dtype, int64_t ldy,
                                 svdq_stream_t stream) {
  svdq_status s = check_weight(w);
  if (s != SVDQ_OK) return s;
  if (B < 0 || (y_dtype != SVDQ_BF16 && y_dtype != SVDQ_F32)) return SVDQ_EINVAL;
  if (B == 0) return SVDQ_OK;
  if (!act_codes || !act_scale || !y || ldy < w->N) return SVDQ_EINVAL;
  if (w->fmt.kind != SVDQ_KIND_INT && !act_sf) return SVDQ_EINVAL;
  if (w->rank > 0 && !down) return SVDQ_EINVAL;
  if (!aligned16(act_codes) || (down && !aligned16(down)) || (bias && !aligned16(bias)))
    return SVDQ_EUNSUPPORTED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  bool bad = false;
  cudaError_t e;
  if (w->fmt.kind == SVDQ_KIND_INT)
    e = launch_gemm_int(w, static_cast<const int8_t*>(act_codes), act_scale,
                        w->rank > 0 ? down : nullptr, B, bias, y, y_dtype, ldy, false, false, st, &bad);
  else
    e = launch_gemm_fp4(w, static_cast<const uint8_t*>(act_codes),
                          static_cast<const uint8_t*>(act_sf), act_scale,
                          w->rank > 0 ? down : nullptr, B, bias, y, y_dtype, ldy, false, st, &bad);
  if (bad) return SVDQ_EUNSUPPORTED;
  return from_cuda(e);
}

svdq_status svdq_residual_product_i32(const svdq_weight* w, const int8_t* act_codes, int64_t B,
                                      int32_t* acc, int64_t ldacc, svdq_stream_t stream) {
  svdq_status s = check_weight(w);
  if (s != SVDQ_OK) return s;
  if (w->fmt.kind != SVDQ_KIND_INT) return SVDQ_EINVAL;
  if (B < 0) return SVDQ_EINVAL;
  if (B == 0) return SVDQ_OK;
  if (!act_codes || !acc || ldacc < w->N) return SVDQ_EINVAL;
  if (!aligned16(act_codes)) return SVDQ_EUNSUPPORTED;
  bool bad = false;
  const cudaError_t e = launch_gemm_int(w, act_codes, nullptr, nullptr, B, nullptr, acc, SVDQ_F32,
                                        ldacc, true, false, reinterpret_cast<cudaStream_t>(stream), &bad);
  if (bad) return SVDQ_EUNSUPPORTED;
  return from_cuda(e);
}

svdq_status svdq_smooth_scale(const void* x, svdq_dtype x_dtype, int64_t B, int64_t M, int64_t ldx,
                              const void* W, svdq_dtype w_dtype, int64_t N, int64_t ldw, float alpha,
                              float* scale, void* workspace, size_t workspace_bytes, svdq_stream_t stream) {
  if (!W || !scale || M < 1 || N < 1 || B < 0 || ldw < N || !(alpha >= 0.0f && alpha <= 1.0f))
    return SVDQ_EINVAL;
  if (B > 0 && (!x || ldx < M)) return SVDQ_EINVAL;
  if ((x_dtype != SVDQ_BF16 && x_dtype != SVDQ_F32) || (w_dtype != SVDQ_BF16 && w_dtype != SVDQ_F32))
    return SVDQ_EINVAL;
  if (!workspace || workspace_bytes < static_cast<size_t>(8 * M)) return SVDQ_EWORKSPACE;
  return from_cuda(launch_smooth_scale(x, x_dtype, B, M, ldx, W, w_dtype, N, ldw, alpha, scale, workspace,
                                       reinterpret_cast<cudaStream_t>(stream)));
}

svdq_status svdq_fold_scale_workspace_size(int64_t B, int64_t M, size_t* bytes) {
  if (!bytes || B < 1 || M < 1) return SVDQ_EINVAL;
  *bytes = fold_scratch_bytes(B, M);
  return SVDQ_OK;
}

svdq_status svdq_fold_scale(const void* x, svdq_dtype x_dtype, int64_t B, int64_t M, int64_t ldx, const void* W,
                            svdq_dtype w_dtype, int64_t N, int64_t ldw, int32_t bits, float* scale,
                            void* workspace, size_t workspace_bytes, svdq_stream_t stream) {
  if (!x || !W || !scale || B < 1 || M < 1 || N < 1 || ldx < M || ldw < N || bits < 2 || bits > 8)
    return SVDQ_EINVAL;
  if ((x_dtype != SVDQ_BF16 && x_dtype != SVDQ_F32) || (w_dtype != SVDQ_BF16 && w_dtype != SVDQ_F32))
    return SVDQ_EINVAL;
  if (!workspace || workspace_bytes < fold_scratch_bytes(B, M)) return SVDQ_EWORKSPACE;
  return from_cuda(launch_fold_scale(x, x_dtype, B, M, ldx, W, w_dtype, N, ldw, bits, scale, workspace,
                                     reinterpret_cast<cudaStream_t>(stream)));
}

svdq_status svdq_check_status(svdq_stream_t stream) {
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return SVDQ_ECUDA;
  unsigned* p = device_status_word();
  if (!p) return SVDQ_ECUDA;
  unsigned v = 0;
  if (cudaMemcpy(&v, p, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return SVDQ_ECUDA;
  if (v != 0) {
    const unsigned zero = 0;
    if (cudaMemcpy(p, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess)
      return SVDQ_ECUDA;
  }
  return static_cast<svdq_status>(v);
}

svdq_status svdq_selftest_wait_timeout(int64_t limit_us, svdq_stream_t stream) {
  if (limit_us <= 0 || limit_us > 10000000) return SVDQ_EINVAL;
  unsigned* status = device_status_word();
  if (!status) return SVDQ_ECUDA;
  wait_selftest_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(limit_us * 1000,
                                                                               status);
  if (cudaGetLastError() != cudaSuccess) return SVDQ_ECUDA;
  return svdq_check_status(stream);
}

}  // extern "C"
