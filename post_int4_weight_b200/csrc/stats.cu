// stats.cu -- per-input-channel activation magnitude x[j] = mean_t |X[t, j]|
// ("From-Scratch AWQ INT4 Quantization on Qwen3-8B", section "AWQ scaling";
// "AWQ architecture, in depth", section "The scale search as code").
//
// A column reduction over X (fp16 [T, ld]).  It is bound by the HBM read of X
// (2 bytes per element).  Each thread owns one 16-byte chunk (8 channels) of
// a row and walks down the rows of its token slice, so a warp reads 512
// contiguous bytes per row.  The sum is exact: |h| of an fp16 h is an integer
// number of 2^-24 units below 2^40, accumulated in 64-bit integers, so the
// order of the additions (and the integer atomics across CTAs) cannot change
// the result.
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace awq {
namespace {

constexpr int kStatsChunks = 32;   // 16-byte chunks per CTA row (256 channels)
constexpr int kStatsRows = 8;      // rows walked in parallel per CTA

// |h| in units of 2^-24.  A non-finite h adds nothing and sets bit 2*col
// (infinity) or 2*col+1 (NaN) of *flags, col being the channel's place in its
// 16-byte chunk.
__device__ __forceinline__ uint64_t abs_half_units(uint32_t h, int col, uint32_t* flags) {
    const uint32_t e = (h >> 10) & 0x1fu;
    const uint32_t mant = h & 0x3ffu;
    if (e == 0x1fu) {
        *flags |= (mant ? 2u : 1u) << (2 * col);
        return 0;
    }
    return e ? (static_cast<uint64_t>(mant | 0x400u) << (e - 1)) : mant;
}

__global__ void stats_zero_kernel(unsigned long long* sums, uint32_t* flags, int64_t d_in) {
    for (int64_t j = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; j < d_in;
         j += (int64_t)gridDim.x * blockDim.x) {
        sums[j] = 0;
        flags[j] = 0;
    }
}

__global__ void __launch_bounds__(kStatsChunks * kStatsRows)
stats_accumulate_kernel(const uint4* __restrict__ X, int64_t T, int64_t d_in,
                        int64_t ld_chunks, int64_t rows_per_split,
                        unsigned long long* __restrict__ sums,
                        uint32_t* __restrict__ flags) {
    __shared__ unsigned long long red[kStatsRows][kStatsChunks][8];
    __shared__ uint32_t fred[kStatsRows][kStatsChunks];

    const int cx = threadIdx.x % kStatsChunks;
    const int ry = threadIdx.x / kStatsChunks;
    const int64_t chunk = (int64_t)blockIdx.x * kStatsChunks + cx;
    const bool active = chunk * 8 < d_in;
    const int64_t r0 = (int64_t)blockIdx.y * rows_per_split;
    const int64_t r1 = min(T, r0 + rows_per_split);

    unsigned long long acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    uint32_t fl = 0;
    if (active) {
        const uint4* p = X + chunk;
        int64_t r = r0 + ry;
        // two rows in flight per iteration
        for (; r + kStatsRows < r1; r += 2 * kStatsRows) {
            const uint4 a = __ldg(p + r * ld_chunks);
            const uint4 b = __ldg(p + (r + kStatsRows) * ld_chunks);
            const uint32_t wa[4] = {a.x, a.y, a.z, a.w};
            const uint32_t wb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                acc[2 * i] += abs_half_units(wa[i] & 0xffffu, 2 * i, &fl) +
                              abs_half_units(wb[i] & 0xffffu, 2 * i, &fl);
                acc[2 * i + 1] += abs_half_units(wa[i] >> 16, 2 * i + 1, &fl) +
                                  abs_half_units(wb[i] >> 16, 2 * i + 1, &fl);
            }
        }
        if (r < r1) {
            const uint4 a = __ldg(p + r * ld_chunks);
            const uint32_t wa[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                acc[2 * i] += abs_half_units(wa[i] & 0xffffu, 2 * i, &fl);
                acc[2 * i + 1] += abs_half_units(wa[i] >> 16, 2 * i + 1, &fl);
            }
        }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) red[ry][cx][i] = acc[i];
    fred[ry][cx] = fl;
    __syncthreads();
    if (ry == 0 && active) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            unsigned long long s = 0;
            for (int k = 0; k < kStatsRows; ++k) s += red[k][cx][i];
            if (s) atomicAdd(sums + chunk * 8 + i, s);
        }
        uint32_t f = 0;
        for (int k = 0; k < kStatsRows; ++k) f |= fred[k][cx];
        if (f) {
            for (int i = 0; i < 8; ++i) {
                const uint32_t fi = (f >> (2 * i)) & 3u;
                if (fi) atomicOr(flags + chunk * 8 + i, fi);
            }
        }
    }
}

// x[j] = (exact sum * 2^-24) / T in fp64, rounded to fp32; NaN if the column
// held a NaN, +inf if it held an infinity.
__global__ void stats_finalize_kernel(const unsigned long long* __restrict__ sums,
                                      const uint32_t* __restrict__ flags, int64_t T,
                                      int64_t d_in, float* __restrict__ x_mean) {
    for (int64_t j = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; j < d_in;
         j += (int64_t)gridDim.x * blockDim.x) {
        const uint32_t f = flags[j];
        float v;
        if (f & 2u) {
            v = __int_as_float(0x7fc00000);
        } else if (f & 1u) {
            v = __int_as_float(0x7f800000);
        } else {
            const double s = __ll2double_rn(static_cast<long long>(sums[j]));
            v = __double2float_rn(__ddiv_rn(s * 0x1p-24, (double)T));
        }
        x_mean[j] = v;
    }
}

}  // namespace

size_t act_stats_workspace(int64_t d_in) {
    return align_up((size_t)d_in * sizeof(unsigned long long), kWsAlign) +
           align_up((size_t)d_in * sizeof(uint32_t), kWsAlign);
}

cudaError_t launch_act_stats(const void* X, int64_t T, int64_t d_in, int64_t ld,
                             float* x_mean, void* ws, cudaStream_t stream) {
    DeviceInfo dev;
    cudaError_t e = query_device(&dev);
    if (e != cudaSuccess) return e;
    auto* sums = static_cast<unsigned long long*>(ws);
    auto* flags = reinterpret_cast<uint32_t*>(
        static_cast<char*>(ws) + align_up((size_t)d_in * sizeof(unsigned long long), kWsAlign));

    const int zero_blocks = (int)std::min<int64_t>((d_in + 255) / 256, 1024);
    stats_zero_kernel<<<zero_blocks, 256, 0, stream>>>(sums, flags, d_in);

    const int64_t col_blocks = (d_in / 8 + kStatsChunks - 1) / kStatsChunks;
    const int64_t want = 4ll * dev.num_sms;
    int64_t splits = (want + col_blocks - 1) / col_blocks;
    const int64_t max_splits = (T + 2 * kStatsRows - 1) / (2 * kStatsRows);
    if (splits > max_splits) splits = max_splits;
    if (splits < 1) splits = 1;
    if (splits > 65535) splits = 65535;
    const int64_t rows_per_split = (T + splits - 1) / splits;
    splits = (T + rows_per_split - 1) / rows_per_split;
    dim3 grid((unsigned)col_blocks, (unsigned)splits);
    stats_accumulate_kernel<<<grid, kStatsChunks * kStatsRows, 0, stream>>>(
        static_cast<const uint4*>(X), T, d_in, ld / 8, rows_per_split, sums, flags);

    stats_finalize_kernel<<<zero_blocks, 256, 0, stream>>>(sums, flags, T, d_in, x_mean);
    return cudaGetLastError();
}

}  // namespace awq
