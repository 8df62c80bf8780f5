// output_error.cu -- optional output-space scoring err[i] = ||X (W - W_hat_i)^T||^2
// ("AWQ architecture, in depth", section "The scale search as code";
// "Weight-Only Quantization: GPTQ and AWQ", section 2).
#include "common.cuh"
#include "internal.h"

namespace awq {

size_t output_error_workspace(int64_t T, int64_t d_out, int64_t d_in, int group_size,
                              int n_grid) {
    (void)T;
    (void)group_size;
    const size_t tab = align_up((size_t)n_grid * (size_t)d_in * sizeof(float), kWsAlign);
    return 2 * tab + align_up((size_t)d_out * (size_t)d_in * 2, kWsAlign) +
           align_up((size_t)4096 * 32 * sizeof(double), kWsAlign) + kWsAlign;
}

awq_status launch_output_error(const void*, int64_t, const void*, int64_t, int64_t,
                               const float*, int, int, int, double*, int32_t*, void*,
                               cudaStream_t) {
    return AWQ_ERR_UNSUPPORTED;
}

}  // namespace awq
