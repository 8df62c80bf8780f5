// norm_group.cu -- one shared scale per norm group ("From-Scratch AWQ INT4
// Quantization on Qwen3-8B", section "AutoAWQ / HF-AWQ GEMM on-disk format",
// exporter steps 1-2): the linears that follow one norm (q/k/v; gate/up)
// each have a searched scale s_m, the norm can absorb only one, so they
// share the per-channel geometric mean
//     s_shared[j] = (prod_m s_m[j])^(1/n)
// (fp64 product in member order; sqrt for n = 2, pow(., 1/n) otherwise; one
// rounding to fp32).  The members are then re-quantised with s_shared by
// awq_quantize_pack.  An elementwise pass over n * d_in floats (HBM-bound,
// a few KB to a few hundred KB): one thread per channel.
#include "common.cuh"
#include "internal.h"

namespace awq {
namespace {

struct ScalePtrs {
    const float* s[AWQ_MAX_SEGMENTS];
};

__global__ void __launch_bounds__(256)
geomean_kernel(const __grid_constant__ ScalePtrs p, int n, int64_t d_in, float* out) {
    pdl_wait();   // the member scales may come from the kernels before
    pdl_launch_dependents();
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; j < d_in; j += stride) {
        if (n == 1) {
            const float v = p.s[0][j];
            out[j] = v;
            if (!isfinite(v)) raise_device_flag(AWQ_FLAG_NONFINITE_SCALE);
            continue;
        }
        double prod = 1.0;
        for (int m = 0; m < n; ++m) prod = __dmul_rn(prod, (double)p.s[m][j]);
        const double r = (n == 2) ? __dsqrt_rn(prod) : pow(prod, __drcp_rn((double)n));
        out[j] = __double2float_rn(r);
        if (!isfinite(prod)) raise_device_flag(AWQ_FLAG_NONFINITE_SCALE);
    }
}

}  // namespace

cudaError_t norm_group_unit_flags(unsigned int* bits, bool clear) {
    return unit_device_flags(bits, clear);
}

cudaError_t launch_norm_group_scale(int n, const float* const* s, int64_t d_in, float* out,
                                    int num_sms, cudaStream_t stream) {
    ScalePtrs p;
    for (int m = 0; m < AWQ_MAX_SEGMENTS; ++m) p.s[m] = m < n ? s[m] : nullptr;
    int64_t blocks = (d_in + 255) / 256;
    if (blocks > 4 * (int64_t)num_sms) blocks = 4 * (int64_t)num_sms;
    return launch_pdl(geomean_kernel, dim3((unsigned)blocks), dim3(256), 0, stream, p, n, d_in,
                      out);
}

}  // namespace awq
