// internal.h - declarations shared by the library's translation units (not part
// of the public C ABI in include/svdq.h).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cstddef>
#include <cstdint>

#include "svdq.h"

namespace svdq {

// Device address of the library's status word (resolved once per device).
unsigned* device_status_word();

// Encode a 2-D tiled tensor map with 128-byte swizzle (or none). Returns false
// if the driver rejects the arguments.
bool make_tmap_2d(CUtensorMap* map, const void* base, CUtensorMapDataType dtype,
                  int elem_bytes, uint64_t inner, uint64_t outer, uint64_t ld_elems,
                  uint32_t box_inner, uint32_t box_outer, bool swizzle128);

inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
inline int64_t round_up(int64_t a, int64_t b) { return ceil_div(a, b) * b; }
inline int32_t rank_pad_of(int32_t rank) { return static_cast<int32_t>(round_up(rank, 16)); }

int num_sms();

// Bump-pointer carving of a caller workspace (256-byte aligned pieces).
struct Carver {
  char* base;
  size_t cap;
  size_t off = 0;
  bool ok = true;
  Carver(void* b, size_t c) : base(static_cast<char*>(b)), cap(c) {}
  void* take(size_t bytes) {
    off = static_cast<size_t>(round_up(static_cast<int64_t>(off), 256));
    void* p = base ? base + off : nullptr;
    off += bytes;
    if (off > cap || base == nullptr) ok = false;
    return p;
  }
};

// ---------------------------------------------------------------- act pass
struct ActPlan {
  int64_t B, M;
  int32_t rank_pad;
  bool bf16;       // x is bf16 (else fp32)
  int tile_k;      // large batch: columns of a 256-byte row segment (128 bf16 / 64 fp32)
  int nrb;         // row blocks of 128
  int nsteps;      // large batch: row segments (the unit of the K split)
  int ksplit;      // K ranges per row block (flat partition: the most pieces a row block is cut into)
  int flat;        // large batch: 1 = flat partition of all segments over qgrid CTAs, 0 = ksplit units
  int qgrid;       // large batch, flat: CTAs asked for (more if a piece would not fit shared memory)
  int nunits;      // nrb * ksplit work units
  int stages;      // large-batch quantise kernel: segment stages in shared memory
  int grid;        // CTAs of the quantise (large batch) or first (short batch) kernel
  int nparts;      // partial maxima written (one per CTA of the first kernel)
  int max_rpc;     // large batch: rows per CTA of the maximum kernel
  int max_nslabs;  // large batch: 2048-byte column slabs of the maximum kernel
  size_t smem;     // dynamic shared memory per CTA
  int small;       // 1: the short-batch kernel (act_small.cu): one column chunk per CTA
  int wc;          // short-batch kernel: columns per chunk (a multiple of 32)
  int chained;     // 1: the first kernel is a programmatic dependent of the work
                   // queued before it (reads x only after griddepcontrol.wait)
};
// Batches up to this many rows take the short-batch kernel.
constexpr int64_t kActSmallMaxB = 128;
// Dynamic shared memory the short-batch kernel may use (else the large-batch plan).
constexpr size_t kActSmallSmemMax = 200 * 1024;
ActPlan plan_act(int64_t B, int64_t M, int32_t rank_pad, svdq_dtype xdt, bool allow_small = true);
// Recompute the derived fields after changing ksplit (for the short-batch
// kernel, ksplit is the number of column chunks).
void finish_act_plan(ActPlan& p);
void finish_act_plan_small(ActPlan& p);
size_t act_scratch_bytes(const ActPlan& p);

// svdq_smooth_scale (smooth.cu): workspace of 2 * M uint32.
cudaError_t launch_smooth_scale(const void* x, svdq_dtype xdt, int64_t B, int64_t M, int64_t ldx, const void* w,
                                svdq_dtype wdt, int64_t N, int64_t ldw, float alpha, float* scale, void* workspace,
                                cudaStream_t st);

// Host checks of svdq_quantize_act's arguments (shared with the allocation-free
// entry point, so both return the same status for the same arguments).
svdq_status check_quantize_act_args(const void* x, svdq_dtype x_dtype, int64_t B, int64_t M, int64_t ldx,
                                    const float* scale, svdq_fmt fmt, const void* ld, int32_t rank_pad,
                                    const void* codes, const void* sf, const float* act_scale,
                                    const void* down);

// svdq_fold_scale (fold.cu)
size_t fold_scratch_bytes(int64_t B, int64_t M);
cudaError_t launch_fold_scale(const void* x, svdq_dtype xdt, int64_t B, int64_t M, int64_t ldx, const void* w,
                              svdq_dtype wdt, int64_t N, int64_t ldw, int bits, float* scale, void* workspace,
                              cudaStream_t st);

cudaError_t launch_act(const ActPlan& p, const void* x, svdq_dtype xdt, int64_t ldx,
                       const float* scale, svdq_fmt fmt, const float* act_global_scale,
                       const float* w_global_scale, const void* ld, void* codes, void* sf,
                       float* act_scale, void* down, void* scratch, cudaStream_t stream,
                       bool* bad_args, unsigned* zero_words = nullptr, int nzero = 0);
cudaError_t launch_act_small(const ActPlan& p, const void* x, svdq_dtype xdt, int64_t ldx,
                             const float* scale, svdq_fmt fmt, const float* act_global_scale,
                             const float* w_global_scale, const void* ld, void* codes, void* sf,
                             float* act_scale, void* down, void* scratch, cudaStream_t stream,
                             bool* bad_args);

// ------------------------------------------------------------ residual GEMM
// split_ws (may be null) holds pair_split_bytes(B, M, N) bytes: the pair kernel
// then splits the tiles of its last, partial round along K.
cudaError_t launch_gemm_int(const svdq_weight* w, const int8_t* act_codes, const float* s_x,
                            const void* down2, int64_t B, const void* bias, void* y,
                            svdq_dtype ydt, int64_t ldy, bool raw_i32, bool pdl, cudaStream_t stream,
                            bool* bad_args, void* split_ws = nullptr);
size_t pair_split_bytes(int64_t B, int64_t M, int64_t N);
// The split's tile counters: pair_split_counters(...) words at that byte offset
// of the split workspace, which must be zero when the GEMM starts.
size_t pair_split_counter_offset(int64_t B, int64_t M, int64_t N);
int pair_split_counters(int64_t B, int64_t M, int64_t N);

// The whole linear for B <= 16 rows with INT weights in one launch (decode.cu);
// false (nothing launched) when the shape or the alignment does not allow it.
bool launch_decode(const svdq_weight* w, const void* x, svdq_dtype xdt, int64_t B, int64_t ldx, const void* bias,
                   void* y, svdq_dtype ydt, int64_t ldy, bool chained, cudaStream_t st, cudaError_t* err);

// NVFP4 or MXFP4, after w->fmt.kind
cudaError_t launch_gemm_fp4(const svdq_weight* w, const uint8_t* act_codes,
                            const uint8_t* act_sf, const float* gs_x, const void* down2,
                            int64_t B, const void* bias, void* y, svdq_dtype ydt,
                            int64_t ldy, bool pdl, cudaStream_t stream, bool* bad_args,
                            void* split_ws = nullptr);

// -------------------------------------------------------------- quantisers
size_t residual_scratch_bytes(int64_t M, int64_t N);
cudaError_t launch_quantize_residual(const float* R, int64_t M, int64_t N, int64_t ldR,
                                     svdq_fmt fmt, void* codes, void* sf, float* w_scale,
                                     void* scratch, cudaStream_t stream);
// INT codes int8 [N, M] -> two per byte [N, M / 2] (element 2j in the low nibble).
cudaError_t launch_pack_int4(const int8_t* codes, int64_t N, int64_t M, uint8_t* packed,
                             cudaStream_t stream);

// ------------------------------------------------------------------ prepare
size_t prepare_scratch_bytes(int64_t M, int64_t N, int32_t rank, int32_t oversample);
svdq_status run_prepare(const void* W, svdq_dtype wdt, int64_t M, int64_t N, int64_t ldW,
                        const float* scale, int32_t rank, svdq_fmt fmt, uint64_t seed,
                        int32_t oversample, int32_t power_iters, void* workspace,
                        size_t ws_bytes, svdq_weight* out, cudaStream_t stream);


}  // namespace svdq
