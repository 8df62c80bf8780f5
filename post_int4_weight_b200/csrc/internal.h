// internal.h -- host-side launchers behind the C ABI of include/awq.h.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <utility>

#include "awq.h"
#include <nvtx3/nvToolsExt.h>

namespace awq {

// A named NVTX range spanning one entry-point call, so that a timeline
// profiler shows each call (and the kernels it enqueued) under its name.
// Without a profiler attached a push or pop costs a pointer check.
struct NvtxRange {
    explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange&) = delete;
    NvtxRange& operator=(const NvtxRange&) = delete;
};


constexpr size_t kWsAlign = 256;

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

inline bool aligned16(const void* p) {
    return (reinterpret_cast<uintptr_t>(p) & 15u) == 0;
}

// Records a failed CUDA runtime call for awq_last_error() (per host thread)
// and passes the error through.
cudaError_t note_cuda(cudaError_t e, const char* where);

struct DeviceInfo {
    int device = 0;
    int num_sms = 0;
    size_t max_smem_optin = 0;    // per block, opt-in
    size_t max_smem_per_sm = 0;
};
cudaError_t query_device(DeviceInfo* info);

// ---- sticky device flags: each device module's accessor (ORs its word into
// *bits, zeroes it if `clear`; the caller has synchronised the device)
cudaError_t stats_unit_flags(unsigned int* bits, bool clear);
cudaError_t search_unit_flags(unsigned int* bits, bool clear);
cudaError_t pack_unit_flags(unsigned int* bits, bool clear);
cudaError_t clip_unit_flags(unsigned int* bits, bool clear);
cudaError_t norm_group_unit_flags(unsigned int* bits, bool clear);
cudaError_t clip_output_unit_flags(unsigned int* bits, bool clear);

// ---- activation statistics
size_t act_stats_workspace(int64_t d_in);
cudaError_t launch_act_stats(const void* X, int64_t T, int64_t d_in, int64_t ld,
                             float* x_mean, void* ws, cudaStream_t stream);

// ---- scale search
size_t scale_search_workspace(int64_t d_in, int group_size, int n_grid);
awq_status launch_scale_search(int n_seg, const void* const* W, const int64_t* d_out,
                               int64_t d_in, const float* x_mean, int group_size,
                               int n_grid, int flags, double* err, int32_t* best_idx,
                               float* s_best, void* ws, cudaStream_t stream);

// ---- quantise + pack
cudaError_t launch_quantize_pack(const void* W, int64_t d_out, int64_t d_in,
                                 const float* s, const uint8_t* clip_idx, int group_size,
                                 int zero_point, int32_t* qweight, void* scales,
                                 int32_t* qzeros, cudaStream_t stream);

// ---- duo scaling (the scale table from x and the weights' row-normalised
// mean); its workspace follows the search workspace
constexpr int kDuoMaxSms = 160;        // weight-mean CTAs (one per SM, at most this many)
constexpr int64_t kDuoMaxDin = 16384;  // the weight-mean pass: at most 4 chunks of 8 per thread
size_t duo_workspace(int64_t d_in, int num_sms, int n_grid);
size_t duo_workspace_bound(int64_t d_in, int n_grid);
cudaError_t launch_duo_table(int n_seg, const void* const* W, const int64_t* d_out, int64_t d_in,
                             const float* x_mean, int n_grid, float* S, float* T,
                             int* dev_words, void* duo_ws, int num_sms, cudaStream_t stream);

// ---- norm-group shared scale
cudaError_t launch_norm_group_scale(int n, const float* const* s, int64_t d_in, float* out,
                                    int num_sms, cudaStream_t stream);

// ---- clip search
size_t clip_search_workspace(int64_t d_in);
cudaError_t launch_clip_search(const void* W, int64_t d_out, int64_t d_in, const float* x_mean,
                               const float* s, int group_size, int n_clip, int flags,
                               uint8_t* clip_idx, double* err, void* ws, cudaStream_t stream);

// ---- output-space clip search (Gram matrices of X's groups, then the
// per (row, group, ratio) quadratic forms)
size_t clip_output_workspace(int64_t d_out, int64_t d_in, int group_size);
cudaError_t launch_clip_search_output(const void* X, int64_t T, int64_t ld, const void* W,
                                      int64_t d_out, int64_t d_in, const float* s,
                                      int group_size, int n_clip, int flags, uint8_t* clip_idx,
                                      double* err, void* ws, cudaStream_t stream);

// ---- output-space scoring
size_t output_error_workspace(int64_t T, int64_t d_out, int64_t d_in, int group_size,
                              int n_grid);
awq_status launch_output_error(const void* X, int64_t T, const void* W, int64_t d_out,
                               int64_t d_in, const float* x_mean, int group_size,
                               int n_grid, int flags, double* err, int32_t* best_idx,
                               float* s_best, void* ws, cudaStream_t stream);

// ---- shared pieces of the search and the output-error mode
// Writes S[i][j] (fp32, [n_grid][d_in]) and a companion table T[i][j] of the
// same shape: (x_mean[j] / S[i][j])^2 for the weight-space search
// (kTableTauSq) or 1 / S[i][j] for the output-space mode (kTableInverse).
// One kernel; clears dev_words[0..1] (error word, CTA-done counter) if
// non-NULL.  Launched as an ordinary launch, so it follows every earlier
// kernel of the stream completely.
enum TableKind { kTableTauSq = 0, kTableInverse = 1 };
constexpr int kMaxTableSlices = 64;
cudaError_t launch_scale_table(const float* x_mean, int64_t d_in, int n_grid, float* S,
                               float* T, int* dev_words, int num_sms, cudaStream_t stream,
                               TableKind kind);

// Launch with the programmatic stream-serialisation attribute (the kernel
// must call pdl_wait() before depending on its predecessor).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}
// Sums partial[c][i] over c in order, picks the first minimum, copies its row
// of S into s_best (if non-NULL).
cudaError_t launch_finalize(const double* partial, int n_parts, int n_grid,
                            const float* S, int64_t d_in, const int* dev_err,
                            double* err, int32_t* best_idx, float* s_best,
                            cudaStream_t stream);

// cuTensorMapEncodeTiled, fetched from the driver once.
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);
EncodeTiledFn encode_tiled_fn();

}  // namespace awq
