// api.cu -- the extern "C" entry points of include/awq.h: host-side argument
// validation, workspace sizing, and dispatch to the launchers.
#include <cstdio>
#include <cstring>

#include "internal.h"

namespace awq {

namespace {
thread_local char g_last_error[256] = "no CUDA error recorded";
}

cudaError_t note_cuda(cudaError_t e, const char* where) {
    if (e != cudaSuccess)
        snprintf(g_last_error, sizeof g_last_error, "%s: %s (%s)", where, cudaGetErrorName(e),
                 cudaGetErrorString(e));
    return e;
}

cudaError_t query_device(DeviceInfo* info) {
    cudaError_t e = cudaGetDevice(&info->device);
    if (e != cudaSuccess) return e;
    e = cudaDeviceGetAttribute(&info->num_sms, cudaDevAttrMultiProcessorCount, info->device);
    if (e != cudaSuccess) return e;
    int v = 0;
    e = cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, info->device);
    if (e != cudaSuccess) return e;
    info->max_smem_optin = (size_t)v;
    e = cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerMultiprocessor, info->device);
    if (e != cudaSuccess) return e;
    info->max_smem_per_sm = (size_t)v;
    return cudaSuccess;
}

EncodeTiledFn encode_tiled_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

static bool valid_group(int g) { return g == 32 || g == 64 || g == 128; }

}  // namespace awq

using namespace awq;

extern "C" {

const char* awq_status_string(int status) {
    switch (status) {
        case AWQ_OK: return "AWQ_OK";
        case AWQ_ERR_INVALID_ARG: return "AWQ_ERR_INVALID_ARG: argument out of range";
        case AWQ_ERR_UNSUPPORTED: return "AWQ_ERR_UNSUPPORTED: valid but not supported";
        case AWQ_ERR_ALIGNMENT: return "AWQ_ERR_ALIGNMENT: pointer or stride misaligned";
        case AWQ_ERR_WORKSPACE: return "AWQ_ERR_WORKSPACE: workspace missing or too small";
        case AWQ_ERR_CUDA: return "AWQ_ERR_CUDA: CUDA runtime or launch failure";
        case AWQ_ERR_NONFINITE: return "AWQ_ERR_NONFINITE: non-finite data met on the device";
        case AWQ_ERR_DEVICE_TIMEOUT:
            return "AWQ_ERR_DEVICE_TIMEOUT: a bounded device-side wait gave up";
        default: return "unknown awq_status";
    }
}

int awq_abi_version(void) { return 101; }

const char* awq_last_error(void) { return g_last_error; }

awq_status awq_last_device_flags(uint32_t* flags, int clear) {
    if (!flags) return AWQ_ERR_INVALID_ARG;
    *flags = 0;
    if (note_cuda(cudaDeviceSynchronize(), "awq_last_device_flags: cudaDeviceSynchronize") !=
        cudaSuccess)
        return AWQ_ERR_CUDA;
    unsigned int bits = 0;
    const bool c = clear != 0;
    cudaError_t (*const units[])(unsigned int*, bool) = {
        stats_unit_flags, search_unit_flags, pack_unit_flags, clip_unit_flags,
        norm_group_unit_flags, clip_output_unit_flags};
    for (auto unit : units)
        if (note_cuda(unit(&bits, c), "awq_last_device_flags: flag word") != cudaSuccess)
            return AWQ_ERR_CUDA;
    *flags = bits;
    if (bits & AWQ_FLAG_WAIT_TIMEOUT) return AWQ_ERR_DEVICE_TIMEOUT;
    if (bits) return AWQ_ERR_NONFINITE;
    return AWQ_OK;
}

awq_status awq_workspace_size(int op, int64_t T, int64_t d_out_total, int64_t d_in,
                              int group_size, int n_grid, size_t* bytes) {
    if (!bytes) return AWQ_ERR_INVALID_ARG;
    if (d_in < 1 || d_in > (int64_t(1) << 24)) return AWQ_ERR_INVALID_ARG;
    switch (op) {
        case AWQ_OP_ACT_STATS:
            *bytes = act_stats_workspace(d_in);
            return AWQ_OK;
        case AWQ_OP_SCALE_SEARCH:
            if (!valid_group(group_size) || n_grid < 1 || n_grid > 32) return AWQ_ERR_INVALID_ARG;
            *bytes = scale_search_workspace(d_in, group_size, n_grid);
            return AWQ_OK;
        case AWQ_OP_SCALE_SEARCH_DUO:
            if (!valid_group(group_size) || n_grid < 1 || n_grid > 32 || d_in > kDuoMaxDin)
                return AWQ_ERR_INVALID_ARG;
            *bytes = scale_search_workspace(d_in, group_size, n_grid) +
                     duo_workspace_bound(d_in, n_grid);
            return AWQ_OK;
        case AWQ_OP_CLIP_SEARCH:
            if (!valid_group(group_size) || d_in < 1 || d_in > (int64_t(1) << 24))
                return AWQ_ERR_INVALID_ARG;
            *bytes = clip_search_workspace(d_in);
            return AWQ_OK;
        case AWQ_OP_CLIP_SEARCH_OUTPUT:
            if (!valid_group(group_size) || d_out_total < 1 || d_out_total > (int64_t(1) << 22) ||
                d_in % group_size || d_in > (int64_t(1) << 20))
                return AWQ_ERR_INVALID_ARG;
            *bytes = clip_output_workspace(d_out_total, d_in, group_size);
            return AWQ_OK;
        case AWQ_OP_OUTPUT_ERROR:
            if (!valid_group(group_size) || n_grid < 1 || n_grid > 32 || T < 1 ||
                d_out_total < 1)
                return AWQ_ERR_INVALID_ARG;
            *bytes = output_error_workspace(T, d_out_total, d_in, group_size, n_grid);
            return AWQ_OK;
        default:
            return AWQ_ERR_INVALID_ARG;
    }
}

awq_status awq_act_stats(const void* X, int64_t T, int64_t d_in, int64_t ld, float* x_mean,
                         void* ws, size_t ws_bytes, void* stream) {
    const NvtxRange nvtx_range("awq_act_stats");
    if (!X || !x_mean) return AWQ_ERR_INVALID_ARG;
    if (T < 1 || T > (int64_t(1) << 23)) return AWQ_ERR_INVALID_ARG;
    if (d_in < 1 || d_in > (int64_t(1) << 24) || ld < d_in) return AWQ_ERR_INVALID_ARG;
    if (d_in % 8 || ld % 8) return AWQ_ERR_ALIGNMENT;
    if (!aligned16(X) || !aligned16(x_mean)) return AWQ_ERR_ALIGNMENT;
    const size_t need = act_stats_workspace(d_in);
    if (need > 0 && (!ws || ws_bytes < need)) return AWQ_ERR_WORKSPACE;
    if (ws && !aligned16(ws)) return AWQ_ERR_ALIGNMENT;
    if (launch_act_stats(X, T, d_in, ld, x_mean, ws, static_cast<cudaStream_t>(stream)) !=
        cudaSuccess)
        return AWQ_ERR_CUDA;
    return AWQ_OK;
}

awq_status awq_scale_search(int n_seg, const void* const* W, const int64_t* d_out,
                            int64_t d_in, const float* x_mean, int group_size, int n_grid,
                            int flags, double* err, int32_t* best_idx, float* s_best,
                            void* ws, size_t ws_bytes, void* stream) {
    const NvtxRange nvtx_range("awq_scale_search");
    if (n_seg < 1 || n_seg > AWQ_MAX_SEGMENTS || !W || !d_out) return AWQ_ERR_INVALID_ARG;
    if (!x_mean || !err || !best_idx || !s_best) return AWQ_ERR_INVALID_ARG;
    if (!valid_group(group_size)) return AWQ_ERR_UNSUPPORTED;
    if (n_grid < 1 || n_grid > 32) return AWQ_ERR_INVALID_ARG;
    if (flags & ~(AWQ_SCALE_FP32 | AWQ_DUO_SCALING | AWQ_ASYMMETRIC | AWQ_TEST_STALL_WAIT))
        return AWQ_ERR_INVALID_ARG;
    const bool duo = (flags & AWQ_DUO_SCALING) != 0;
    if (duo && d_in > kDuoMaxDin) return AWQ_ERR_UNSUPPORTED;
    if (d_in < group_size || d_in % group_size || d_in > (int64_t(1) << 24))
        return AWQ_ERR_INVALID_ARG;
    for (int k = 0; k < n_seg; ++k) {
        if (!W[k]) return AWQ_ERR_INVALID_ARG;
        if (d_out[k] < 1 || d_out[k] > (int64_t(1) << 31)) return AWQ_ERR_INVALID_ARG;
        if (!aligned16(W[k])) return AWQ_ERR_ALIGNMENT;
    }
    if (!aligned16(x_mean) || !aligned16(err) || !aligned16(best_idx) || !aligned16(s_best))
        return AWQ_ERR_ALIGNMENT;
    const size_t need = scale_search_workspace(d_in, group_size, n_grid) +
                        (duo ? duo_workspace_bound(d_in, n_grid) : 0);
    if (!ws || ws_bytes < need) return AWQ_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(ws) & (kWsAlign - 1)) != 0) return AWQ_ERR_ALIGNMENT;
    return launch_scale_search(n_seg, W, d_out, d_in, x_mean, group_size, n_grid, flags, err,
                               best_idx, s_best, ws, static_cast<cudaStream_t>(stream));
}

awq_status awq_quantize_pack(const void* W, int64_t d_out, int64_t d_in, const float* s,
                             const uint8_t* clip_idx, int group_size, int zero_point,
                             int32_t* qweight, void* scales, int32_t* qzeros, void* stream) {
    const NvtxRange nvtx_range("awq_quantize_pack");
    if (!W || !qweight || !scales || !qzeros) return AWQ_ERR_INVALID_ARG;
    if (!valid_group(group_size)) return AWQ_ERR_UNSUPPORTED;
    if (zero_point != 7 && zero_point != 8 && zero_point != AWQ_ZERO_POINT_ASYM)
        return AWQ_ERR_INVALID_ARG;
    if (zero_point == AWQ_ZERO_POINT_ASYM && clip_idx) return AWQ_ERR_UNSUPPORTED;
    if (d_out < 8 || d_out % 8 || d_out > (int64_t(1) << 31)) return AWQ_ERR_INVALID_ARG;
    if (d_in < group_size || d_in % group_size || d_in > (int64_t(1) << 24))
        return AWQ_ERR_INVALID_ARG;
    if (!aligned16(W) || !aligned16(qweight) || !aligned16(scales) || !aligned16(qzeros))
        return AWQ_ERR_ALIGNMENT;
    if (s && !aligned16(s)) return AWQ_ERR_ALIGNMENT;
    if (note_cuda(launch_quantize_pack(W, d_out, d_in, s, clip_idx, group_size, zero_point,
                                       qweight, scales, qzeros,
                                       static_cast<cudaStream_t>(stream)),
                  "quantize_pack launch") != cudaSuccess)
        return AWQ_ERR_CUDA;
    return AWQ_OK;
}

awq_status awq_norm_group_scale(int n, const float* const* s, int64_t d_in, float* s_shared,
                               void* stream) {
    const NvtxRange nvtx_range("awq_norm_group_scale");
    if (n < 1 || n > AWQ_MAX_SEGMENTS || !s || !s_shared) return AWQ_ERR_INVALID_ARG;
    if (d_in < 1 || d_in > (int64_t(1) << 24)) return AWQ_ERR_INVALID_ARG;
    for (int m = 0; m < n; ++m) {
        if (!s[m]) return AWQ_ERR_INVALID_ARG;
        if (!aligned16(s[m])) return AWQ_ERR_ALIGNMENT;
    }
    if (!aligned16(s_shared)) return AWQ_ERR_ALIGNMENT;
    DeviceInfo dev;
    if (note_cuda(query_device(&dev), "device query") != cudaSuccess) return AWQ_ERR_CUDA;
    if (note_cuda(launch_norm_group_scale(n, s, d_in, s_shared, dev.num_sms,
                                          static_cast<cudaStream_t>(stream)),
                  "norm_group_scale launch") != cudaSuccess)
        return AWQ_ERR_CUDA;
    return AWQ_OK;
}

awq_status awq_clip_search(const void* W, int64_t d_out, int64_t d_in, const float* x_mean,
                           const float* s, int group_size, int n_clip, int flags,
                           uint8_t* clip_idx, double* err, void* ws, size_t ws_bytes,
                           void* stream) {
    const NvtxRange nvtx_range("awq_clip_search");
    if (!W || !x_mean || !clip_idx || !err) return AWQ_ERR_INVALID_ARG;
    if (!valid_group(group_size)) return AWQ_ERR_UNSUPPORTED;
    if (n_clip < 1 || n_clip > AWQ_CLIP_MAX) return AWQ_ERR_INVALID_ARG;
    if (flags != AWQ_SCALE_FP16 && flags != AWQ_SCALE_FP32) return AWQ_ERR_INVALID_ARG;
    if (d_out < 1 || d_out > (int64_t(1) << 31)) return AWQ_ERR_INVALID_ARG;
    if (d_in < group_size || d_in % group_size || d_in > (int64_t(1) << 24))
        return AWQ_ERR_INVALID_ARG;
    if (!aligned16(W) || !aligned16(x_mean) || !aligned16(err) || (s && !aligned16(s)))
        return AWQ_ERR_ALIGNMENT;
    if (!ws || ws_bytes < clip_search_workspace(d_in)) return AWQ_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(ws) & (kWsAlign - 1)) != 0) return AWQ_ERR_ALIGNMENT;
    if (note_cuda(launch_clip_search(W, d_out, d_in, x_mean, s, group_size, n_clip, flags,
                                     clip_idx, err, ws, static_cast<cudaStream_t>(stream)),
                  "clip_search launch") != cudaSuccess)
        return AWQ_ERR_CUDA;
    return AWQ_OK;
}

awq_status awq_clip_search_output(const void* X, int64_t T, int64_t ld, const void* W,
                                  int64_t d_out, int64_t d_in, const float* s, int group_size,
                                  int n_clip, int flags, uint8_t* clip_idx, double* err,
                                  void* ws, size_t ws_bytes, void* stream) {
    const NvtxRange nvtx_range("awq_clip_search_output");
    if (!X || !W || !clip_idx || !err) return AWQ_ERR_INVALID_ARG;
    if (!valid_group(group_size)) return AWQ_ERR_UNSUPPORTED;
    if (n_clip < 1 || n_clip > AWQ_CLIP_MAX) return AWQ_ERR_INVALID_ARG;
    if (flags != AWQ_SCALE_FP16 && flags != AWQ_SCALE_FP32) return AWQ_ERR_INVALID_ARG;
    if (T < 1 || T > (int64_t(1) << 24)) return AWQ_ERR_INVALID_ARG;
    if (d_out < 1 || d_out > (int64_t(1) << 22)) return AWQ_ERR_INVALID_ARG;
    if (d_in < group_size || d_in % group_size || d_in > (int64_t(1) << 20) || ld < d_in)
        return AWQ_ERR_INVALID_ARG;
    if (ld % 8) return AWQ_ERR_ALIGNMENT;
    if (!aligned16(X) || !aligned16(W) || !aligned16(err) || (s && !aligned16(s)))
        return AWQ_ERR_ALIGNMENT;
    if (!ws || ws_bytes < clip_output_workspace(d_out, d_in, group_size)) return AWQ_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(ws) & (kWsAlign - 1)) != 0) return AWQ_ERR_ALIGNMENT;
    if (note_cuda(launch_clip_search_output(X, T, ld, W, d_out, d_in, s, group_size, n_clip,
                                            flags, clip_idx, err, ws,
                                            static_cast<cudaStream_t>(stream)),
                  "clip_search_output launch") != cudaSuccess)
        return AWQ_ERR_CUDA;
    return AWQ_OK;
}

awq_status awq_output_error(const void* X, int64_t T, const void* W, int64_t d_out,
                            int64_t d_in, const float* x_mean, int group_size, int n_grid,
                            int flags, double* err, int32_t* best_idx, float* s_best,
                            void* ws, size_t ws_bytes, void* stream) {
    const NvtxRange nvtx_range("awq_output_error");
    if (!X || !W || !x_mean || !err || !best_idx) return AWQ_ERR_INVALID_ARG;
    if (!valid_group(group_size)) return AWQ_ERR_UNSUPPORTED;
    if (n_grid < 1 || n_grid > 32) return AWQ_ERR_INVALID_ARG;
    if (flags & ~(AWQ_SCALE_FP32 | AWQ_ASYMMETRIC)) return AWQ_ERR_INVALID_ARG;
    if (T < 1 || T > (int64_t(1) << 24)) return AWQ_ERR_INVALID_ARG;
    if (d_out < 8 || d_out % 8 || d_out > (int64_t(1) << 24)) return AWQ_ERR_INVALID_ARG;
    if (d_in < group_size || d_in % group_size || d_in % 64 || d_in > (int64_t(1) << 20))
        return AWQ_ERR_INVALID_ARG;
    if (!aligned16(X) || !aligned16(W) || !aligned16(x_mean) || !aligned16(err) ||
        !aligned16(best_idx) || (s_best && !aligned16(s_best)))
        return AWQ_ERR_ALIGNMENT;
    if (!ws || ws_bytes < output_error_workspace(T, d_out, d_in, group_size, n_grid))
        return AWQ_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(ws) & (kWsAlign - 1)) != 0) return AWQ_ERR_ALIGNMENT;
    return launch_output_error(X, T, W, d_out, d_in, x_mean, group_size, n_grid, flags, err,
                               best_idx, s_best, ws, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
