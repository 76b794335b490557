// noalloc.cu - svdq_quantize_act_noalloc: the activation pass with its scratch
// in a fixed device array that lives inside this library, for callers that
// cannot hand the library a workspace.
//
// Who needs it: code that runs inside a host runtime which owns every byte of
// device memory and exposes no allocator on the request path (static memory
// plans of inference servers, plugin interfaces of other engines, tightly
// budgeted real-time loops), so neither the caller nor this library may call
// cudaMalloc there. The caller still provides the inputs and outputs.
//
// The array is a file-scope __device__ variable, so every GPU that loads the
// library holds kNoallocScratchBytes of it until the process exits. Its device
// address is looked up once per device (cudaGetSymbolAddress, with that device
// current) on the first call made on that device; make that first call before
// any stream capture. All calls share the one array and it keeps the previous
// call's contents: the kernels overwrite every scratch word they read, so
// nothing needs clearing, but calls whose kernels overlap on the GPU (two
// streams, or two host threads) race on it.
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <mutex>

#include "internal.h"

namespace svdq {

namespace {

constexpr size_t kNoallocScratchBytes = size_t(8) << 20;  // 8 MiB per device

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

constexpr int kMaxDev = 64;
std::mutex g_noalloc_mu;
std::atomic<void*> g_noalloc_ptr[kMaxDev] = {};

// Device address of the array on the current device (nullptr on failure). It
// is looked up once per device and process and kept: a context torn down and
// made again (cudaDeviceReset) would leave a stale address, which this entry
// point does not detect. The lock is taken only by a device's first lookup.
void* noalloc_scratch() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return nullptr;
  void* p = g_noalloc_ptr[dev].load(std::memory_order_acquire);
  if (p) return p;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  p = g_noalloc_ptr[dev].load(std::memory_order_relaxed);
  if (!p) {
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
    g_noalloc_ptr[dev].store(p, std::memory_order_release);
  }
  return p;
}

}  // namespace

}  // namespace svdq

using namespace svdq;

extern "C" svdq_status svdq_quantize_act_noalloc(
    const void* x, svdq_dtype x_dtype, int64_t B, int64_t M, int64_t ldx, const float* scale,
    svdq_fmt fmt, const float* act_global_scale, const float* w_global_scale, const void* ld,
    int32_t rank_pad, void* codes, void* sf, float* act_scale, void* down,
    svdq_stream_t stream) {
  const svdq_status st = check_quantize_act_args(x, x_dtype, B, M, ldx, scale, fmt, ld, rank_pad, codes, sf,
                                                 act_scale, down);
  if (st != SVDQ_OK || B == 0) return st;

  // Same launch plan as svdq_quantize_act, with fewer K splits if that is what
  // it takes to fit the fixed array; beyond that the shape is refused. The
  // large-batch flat partition cuts a row block into pieces at CTA boundaries,
  // one partial slot each; when those slots do not fit, the plan goes over to
  // K split units, whose count per row block it can then halve.
  const int32_t rp = (ld != nullptr) ? rank_pad : 0;
  auto to_split = [](ActPlan& q) {
    if (q.small || !q.flat) return;
    q.flat = 0;
    q.ksplit = std::max(1, std::min(q.nsteps, num_sms() / std::max(q.nrb, 1)));
    finish_act_plan(q);
  };
  ActPlan p = plan_act(B, M, rp, x_dtype);
  if (act_scratch_bytes(p) > kNoallocScratchBytes) to_split(p);
  while (act_scratch_bytes(p) > kNoallocScratchBytes && p.ksplit > 1) {
    const int before = p.ksplit;
    p.ksplit = std::max(1, p.ksplit / 2);
    finish_act_plan(p);
    if (!p.small && p.ksplit >= before) break;   // the split cannot shrink further
    // fewer, wider column chunks of the short-batch kernel may outgrow its
    // shared memory: continue with the large-batch plan then
    if (p.small && p.smem > kActSmallSmemMax) {
      p = plan_act(B, M, rp, x_dtype, false);
      if (act_scratch_bytes(p) > kNoallocScratchBytes) to_split(p);
    }
  }
  if (act_scratch_bytes(p) > kNoallocScratchBytes) return SVDQ_EWORKSPACE;

  void* scratch = noalloc_scratch();
  if (!scratch) return SVDQ_ECUDA;
  bool bad = false;
  const cudaError_t e =
      launch_act(p, x, x_dtype, ldx, scale, fmt, act_global_scale,
                 fmt.kind == SVDQ_KIND_NVFP4 ? w_global_scale : nullptr, rp > 0 ? ld : nullptr, codes, sf, act_scale,
                 down, scratch, reinterpret_cast<cudaStream_t>(stream), &bad);
  if (bad) return SVDQ_EUNSUPPORTED;
  return e == cudaSuccess ? SVDQ_OK : SVDQ_ECUDA;
}
