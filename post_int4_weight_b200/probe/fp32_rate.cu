// fp32_rate.cu -- measured FP32 FMA-pipe throughput of the current device, the
// denominator beside the derived (SMs x 128 lanes x clock) peak against which
// the bench reports the scale search, an FP32-ALU-bound kernel.
//
// Not part of the method or of the C ABI of include/awq.h: a separate probe
// library (libawq_probe.so) that bench.py loads to time a pure FMA stream.
// Each thread runs 16 independent fused multiply-add chains x <- x * a + b
// (a = 0.5, b = 0.5: every chain converges to 1.0 and never leaves the
// normal range), fully occupying the SM; a lane-op is one fp32 FMA of one
// thread.  Three instruction mixes:
//   mode 0  scalar FFMA only;
//   mode 1  packed fp32x2 FFMA2 only (two lane-ops per instruction);
//   mode 2  half of the chains packed, half scalar (the search kernel's mix).
#include <cuda_runtime.h>
#include <stdint.h>

namespace {

constexpr int kChains = 16;
constexpr int kThreads = 256;
constexpr int kBlocksPerSm = 8;

template <int MODE>
__global__ void __launch_bounds__(kThreads, kBlocksPerSm)
fma_rate_kernel(float* out, int iters) {
    float x[kChains];
#pragma unroll
    for (int i = 0; i < kChains; ++i) x[i] = 1.0f + (float)((threadIdx.x + i) & 7) * 0.125f;
    const float a = 0.5f, b = 0.5f;
    for (int it = 0; it < iters; ++it) {
#pragma unroll
        for (int i = 0; i < kChains; i += 2) {
            if (MODE == 0 || (MODE == 2 && (i & 2))) {
                x[i] = __fmaf_rn(x[i], a, b);
                x[i + 1] = __fmaf_rn(x[i + 1], a, b);
            } else {
                float2 v = __ffma2_rn(make_float2(x[i], x[i + 1]), make_float2(a, a),
                                      make_float2(b, b));
                x[i] = v.x;
                x[i + 1] = v.y;
            }
        }
    }
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < kChains; ++i) s += x[i];
    out[(size_t)blockIdx.x * blockDim.x + threadIdx.x] = s;
}

}  // namespace

// Runs mode's kernel `reps` times with `iters` loop trips on the current
// device and returns the fastest launch: *lane_ops = fp32 FMAs per launch,
// *ms = its duration (CUDA events around the launch on a private stream).
// `out` is a device buffer of at least sms * 8 * 256 floats.  0 on success,
// else the cudaError_t.
extern "C" int awq_probe_fp32_rate(int mode, int iters, int reps, float* out,
                                   double* lane_ops, double* ms) {
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return (int)e;
    cudaStream_t st;
    cudaEvent_t e0, e1;
    if ((e = cudaStreamCreateWithFlags(&st, cudaStreamNonBlocking)) != cudaSuccess) return (int)e;
    cudaEventCreate(&e0);
    cudaEventCreate(&e1);
    const dim3 grid((unsigned)(sms * kBlocksPerSm)), block(kThreads);
    float best = -1.f;
    for (int r = 0; r < reps && e == cudaSuccess; ++r) {
        cudaEventRecord(e0, st);
        if (mode == 0) fma_rate_kernel<0><<<grid, block, 0, st>>>(out, iters);
        else if (mode == 1) fma_rate_kernel<1><<<grid, block, 0, st>>>(out, iters);
        else fma_rate_kernel<2><<<grid, block, 0, st>>>(out, iters);
        cudaEventRecord(e1, st);
        e = cudaEventSynchronize(e1);
        if (e == cudaSuccess) e = cudaGetLastError();
        float t = 0.f;
        if (e == cudaSuccess) cudaEventElapsedTime(&t, e0, e1);
        if (e == cudaSuccess && (best < 0.f || t < best)) best = t;
    }
    cudaEventDestroy(e0);
    cudaEventDestroy(e1);
    cudaStreamDestroy(st);
    if (e != cudaSuccess) return (int)e;
    *lane_ops = (double)grid.x * kThreads * (double)iters * kChains;
    *ms = best;
    return 0;
}
