// duo.cu -- duo scaling candidates for the scale search ("AWQ architecture,
// in depth", section "The scale search as code": with duo scaling the
// candidate x^r is also divided by the mean normalised weight magnitude
// raised to 1 - r):
//
//   w_mean[j] = (1/R) sum over the R rows of all segments of |W[r,j]| / max_k |W[r,k]|
//   v_i[j]    = max(x[j]^r / (w_mean[j]^(1-r) + 1e-4), 1e-4),   r = i / n_grid
//   S[i][j]   = v_i[j] / sqrt(max_j v_i * min_j v_i)      (fp64, one fp32 rounding)
//   T[i][j]   = (x[j] / S[i][j])^2                         (what the search reads)
//
// Kernels, each a programmatic dependent launch that waits for its
// predecessor before reading and only then lets its dependents launch:
//   wmean_partial_kernel   one CTA of 512 threads per SM, a contiguous range of
//                          rows each; per row a block-wide max of |w|, then
//                          every thread adds |w| / max for its own columns
//                          (at most 4 chunks of 8) into fp64 sums held in
//                          registers (quotients
//                          correctly rounded via ddiv_rn_rcp); the next row is
//                          loaded while the current one is processed.  HBM
//                          reads W once (2 B per weight).
//   wmean_final_kernel     sums the per-CTA column sums in CTA order, / R.
//   duo_minmax_kernel      (slices x alphas): v_i[j] and per-slice min/max.
//   duo_write_kernel       same grid: the normalisation, S and T.
// Column sums are exact row-by-row fp64 additions within a CTA and then in
// CTA order, so the result is the same on every run.
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace awq {
namespace {

constexpr int kWmThreads = 512;
constexpr int kWmWarps = kWmThreads / 32;
constexpr int kWmMaxChunks = 4;        // 16-byte chunks per thread per row: d_in <= 16384
constexpr int kMaxDuoSlices = 64;

struct WmParams {
    const uint4* W[AWQ_MAX_SEGMENTS];
    int64_t row_begin[AWQ_MAX_SEGMENTS + 1];   // prefix sum of rows per segment
    int n_seg;
    int64_t d_in;
    int64_t rows;
    double* partial;                           // [gridDim.x][d_in]
};

// |h| of an fp16 value as fp64 without the conversion pipe: the fp32 value
// has at most 11 significant bits, so its fp64 twin has the high word
// (bits >> 3) + ((1023 - 127) << 20) and a zero low word; 0 stays 0.
__device__ __forceinline__ double abs_half_to_double(uint32_t h16) {
    const uint32_t a = h16 & 0x7fffu;
    if (a == 0) return 0.0;
    const uint32_t f = __float_as_uint(__half2float(__ushort_as_half((unsigned short)a)));
    return __hiloint2double((int)((f >> 3) + 0x38000000u), 0);
}

__device__ __forceinline__ float chunk_absmax(const uint4 v) {
    const uint32_t w[4] = {v.x & 0x7fff7fffu, v.y & 0x7fff7fffu, v.z & 0x7fff7fffu,
                           v.w & 0x7fff7fffu};
    uint32_t m = __vmaxu2(__vmaxu2(w[0], w[1]), __vmaxu2(w[2], w[3]));
    m = max(m & 0xffffu, m >> 16);
    return __half2float(__ushort_as_half((unsigned short)m));
}

__global__ void __launch_bounds__(kWmThreads, 1)
wmean_partial_kernel(const __grid_constant__ WmParams p) {
    __shared__ float red[2][kWmWarps];
    pdl_wait();   // W may come from the kernel before
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t chunks = p.d_in / 8;
    double acc[kWmMaxChunks][8];                    // columns 8 * (tid + c * 512) + 0..7
#pragma unroll
    for (int c = 0; c < kWmMaxChunks; ++c)
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[c][e] = 0.0;
    const int64_t r0 = p.rows * blockIdx.x / gridDim.x;
    const int64_t r1 = p.rows * (blockIdx.x + 1) / gridDim.x;

    auto row_ptr = [&](int64_t r) {
        int k = 0;
        while (k + 1 < p.n_seg && r >= p.row_begin[k + 1]) ++k;
        return p.W[k] + (r - p.row_begin[k]) * chunks;
    };
    uint4 cur[kWmMaxChunks], nxt[kWmMaxChunks];
    const uint4 z = make_uint4(0, 0, 0, 0);
    if (r0 < r1) {
        const uint4* rp = row_ptr(r0);
#pragma unroll
        for (int c = 0; c < kWmMaxChunks; ++c) {
            const int64_t ch = tid + (int64_t)c * kWmThreads;
            cur[c] = ch < chunks ? __ldg(rp + ch) : z;
        }
    }
    for (int64_t r = r0; r < r1; ++r) {
        if (r + 1 < r1) {   // the next row's loads are in flight while this one is summed
            const uint4* rp = row_ptr(r + 1);
#pragma unroll
            for (int c = 0; c < kWmMaxChunks; ++c) {
                const int64_t ch = tid + (int64_t)c * kWmThreads;
                nxt[c] = ch < chunks ? __ldg(rp + ch) : z;
            }
        }
        float m = 0.f;
#pragma unroll
        for (int c = 0; c < kWmMaxChunks; ++c) m = fmaxf(m, chunk_absmax(cur[c]));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        const int slot = (int)(r & 1);   // two slots: one barrier per row suffices
        if (lane == 0) red[slot][warp] = m;
        __syncthreads();
        m = 0.f;
#pragma unroll
        for (int w = 0; w < kWmWarps; ++w) m = fmaxf(m, red[slot][w]);
        if (m > 0.f) {
            const double mx = (double)m;
            const double y = __drcp_rn(mx);
#pragma unroll
            for (int c = 0; c < kWmMaxChunks; ++c) {
                const int64_t ch = tid + (int64_t)c * kWmThreads;
                if (ch < chunks) {
                    const uint32_t w[4] = {cur[c].x, cur[c].y, cur[c].z, cur[c].w};
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const double a0 = abs_half_to_double(w[i] & 0xffffu);
                        const double a1 = abs_half_to_double(w[i] >> 16);
                        acc[c][2 * i] += ddiv_rn_rcp(a0, mx, y);
                        acc[c][2 * i + 1] += ddiv_rn_rcp(a1, mx, y);
                    }
                }
            }
        }
#pragma unroll
        for (int c = 0; c < kWmMaxChunks; ++c) cur[c] = nxt[c];
    }
    pdl_launch_dependents();
    double* out = p.partial + (int64_t)blockIdx.x * p.d_in;
#pragma unroll
    for (int c = 0; c < kWmMaxChunks; ++c) {
        const int64_t ch = tid + (int64_t)c * kWmThreads;
        if (ch < chunks) {
            double2* o2 = reinterpret_cast<double2*>(out + 8 * ch);
#pragma unroll
            for (int e = 0; e < 4; ++e) o2[e] = make_double2(acc[c][2 * e], acc[c][2 * e + 1]);
        }
    }
}

__global__ void __launch_bounds__(256)
wmean_final_kernel(const double* __restrict__ partial, int n_parts, int64_t d_in, int64_t rows,
                   double* __restrict__ w_mean) {
    pdl_wait();
    pdl_launch_dependents();
    for (int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; j < d_in;
         j += (int64_t)gridDim.x * blockDim.x) {
        // CTA order; 16 loads in flight before they are added in that order
        double s = 0.0;
        for (int c0 = 0; c0 < n_parts; c0 += 16) {
            double v[16];
#pragma unroll
            for (int k = 0; k < 16; ++k)
                v[k] = c0 + k < n_parts ? __ldcg(partial + (int64_t)(c0 + k) * d_in + j) : 0.0;
#pragma unroll
            for (int k = 0; k < 16; ++k)
                if (c0 + k < n_parts) s += v[k];
        }
        w_mean[j] = __ddiv_rn(s, (double)rows);
    }
}

__device__ __forceinline__ double duo_value(float xj, double wm, double r) {
    const double v = __ddiv_rn(pow((double)xj, r), pow(wm, 1.0 - r) + 1e-4);
    return v < 1e-4 ? 1e-4 : v;
}

__global__ void __launch_bounds__(256, 1)
duo_minmax_kernel(const float* __restrict__ x, const double* __restrict__ w_mean, int64_t d_in,
                  int n_grid, int64_t slice, double* __restrict__ part,
                  int* __restrict__ dev_words) {
    __shared__ double red_mx[8], red_mn[8];
    pdl_wait();
    pdl_launch_dependents();
    const int a = blockIdx.y, sl = blockIdx.x;
    if (a == 0 && sl == 0 && threadIdx.x == 0) {
        dev_words[0] = 0;
        dev_words[1] = 0;
    }
    const double r = __ddiv_rn((double)a, (double)n_grid);
    double mx = 0.0, mn = __longlong_as_double(0x7ff0000000000000ll);
    const int64_t j0 = (int64_t)sl * slice, j1 = min(d_in, j0 + slice);
    for (int64_t j = j0 + threadIdx.x; j < j1; j += blockDim.x) {
        const double v = duo_value(x[j], w_mean[j], r);
        mx = fmax(mx, v);
        mn = fmin(mn, v);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        mn = fmin(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    }
    if ((threadIdx.x & 31) == 0) {
        red_mx[threadIdx.x >> 5] = mx;
        red_mn[threadIdx.x >> 5] = mn;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int k = 1; k < (int)(blockDim.x >> 5); ++k) {
            mx = fmax(mx, red_mx[k]);
            mn = fmin(mn, red_mn[k]);
        }
        part[((int64_t)a * gridDim.x + sl) * 2 + 0] = mx;
        part[((int64_t)a * gridDim.x + sl) * 2 + 1] = mn;
    }
}

__global__ void __launch_bounds__(256, 1)
duo_write_kernel(const float* __restrict__ x, const double* __restrict__ w_mean, int64_t d_in,
                 int n_grid, int64_t slice, const double* __restrict__ part,
                 float* __restrict__ S, float* __restrict__ T) {
    pdl_wait();
    pdl_launch_dependents();
    const int a = blockIdx.y, sl = blockIdx.x;
    double mx = 0.0, mn = __longlong_as_double(0x7ff0000000000000ll);
    for (int k = 0; k < (int)gridDim.x; ++k) {   // max and min are order-independent
        mx = fmax(mx, __ldcg(part + ((int64_t)a * gridDim.x + k) * 2 + 0));
        mn = fmin(mn, __ldcg(part + ((int64_t)a * gridDim.x + k) * 2 + 1));
    }
    const double norm = __dsqrt_rn(__dmul_rn(mx, mn));
    const double r = __ddiv_rn((double)a, (double)n_grid);
    const int64_t j0 = (int64_t)sl * slice, j1 = min(d_in, j0 + slice);
    for (int64_t j = j0 + threadIdx.x; j < j1; j += blockDim.x) {
        const float xj = x[j];
        const float s = __double2float_rn(__ddiv_rn(duo_value(xj, w_mean[j], r), norm));
        S[(int64_t)a * d_in + j] = s;
        const double q = __ddiv_rn((double)xj, (double)s);
        T[(int64_t)a * d_in + j] = __double2float_rn(q * q);
    }
}

}  // namespace

size_t duo_workspace(int64_t d_in, int num_sms, int n_grid) {
    return align_up((size_t)num_sms * (size_t)d_in * sizeof(double), kWsAlign) +
           align_up((size_t)d_in * sizeof(double), kWsAlign) +
           align_up((size_t)n_grid * kMaxDuoSlices * 2 * sizeof(double), kWsAlign);
}

size_t duo_workspace_bound(int64_t d_in, int n_grid) {
    return duo_workspace(d_in, kDuoMaxSms, n_grid);
}

cudaError_t launch_duo_table(int n_seg, const void* const* W, const int64_t* d_out, int64_t d_in,
                             const float* x_mean, int n_grid, float* S, float* T,
                             int* dev_words, void* duo_ws, int num_sms, cudaStream_t stream) {
    if (d_in > (int64_t)kWmMaxChunks * kWmThreads * 8) return cudaErrorInvalidValue;
    const int grid = std::min(num_sms, kDuoMaxSms);
    char* base = static_cast<char*>(duo_ws);
    double* partial = reinterpret_cast<double*>(base);
    double* w_mean = reinterpret_cast<double*>(
        base + align_up((size_t)grid * (size_t)d_in * sizeof(double), kWsAlign));
    double* part = reinterpret_cast<double*>(
        reinterpret_cast<char*>(w_mean) + align_up((size_t)d_in * sizeof(double), kWsAlign));

    WmParams p;
    int64_t rows = 0;
    for (int k = 0; k < AWQ_MAX_SEGMENTS; ++k) {
        p.W[k] = k < n_seg ? static_cast<const uint4*>(W[k]) : nullptr;
        p.row_begin[k] = rows;
        if (k < n_seg) rows += d_out[k];
    }
    p.row_begin[AWQ_MAX_SEGMENTS] = rows;
    p.n_seg = n_seg;
    p.d_in = d_in;
    p.rows = rows;
    p.partial = partial;
    cudaError_t e = launch_pdl(wmean_partial_kernel, dim3(grid), dim3(kWmThreads), 0, stream, p);
    if (e != cudaSuccess) return e;
    const int fin_blocks = (int)std::min<int64_t>((d_in + 255) / 256, 4 * (int64_t)num_sms);
    e = launch_pdl(wmean_final_kernel, dim3(fin_blocks), dim3(256), 0, stream,
                   (const double*)partial, grid, d_in, rows, w_mean);
    if (e != cudaSuccess) return e;

    int64_t slices = (2 * (int64_t)num_sms + n_grid - 1) / n_grid;
    slices = std::min<int64_t>(slices, (d_in + 63) / 64);
    slices = std::max<int64_t>(1, std::min<int64_t>(slices, kMaxDuoSlices));
    const int64_t slice = (d_in + slices - 1) / slices;
    slices = (d_in + slice - 1) / slice;
    const dim3 tg((unsigned)slices, (unsigned)n_grid);
    e = launch_pdl(duo_minmax_kernel, tg, dim3(256), 0, stream, x_mean, (const double*)w_mean,
                   d_in, n_grid, slice, part, dev_words);
    if (e != cudaSuccess) return e;
    return launch_pdl(duo_write_kernel, tg, dim3(256), 0, stream, x_mean, (const double*)w_mean,
                      d_in, n_grid, slice, (const double*)part, S, T);
}

}  // namespace awq
