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
//                          rows each, streamed by bulk copies (TMA) into a
//                          shared ring 6-16 rows deep.  Per batch of rows the
//                          block-wide maxima of |w|; every thread adds |w| / max
//                          for its columns (at most 4 chunks of 8) into fp64
//                          sums held in registers (quotients correctly rounded
//                          via ddiv_rn_rcp).  HBM reads W once (2 B per weight).
//   duo_candidates_kernel  one CTA per 32 columns: w_mean from the per-CTA
//                          column sums, then v_i[j] for every alpha (stored in
//                          fp64) and its max and min over the CTA's columns.
//   duo_write_kernel       (slices x alphas): the alpha's max and min over the
//                          candidates CTAs, the normalisation, S and T.
// Column sums are fp64 additions in a fixed order (rows in order within a
// weight-mean CTA; those CTAs' sums in eight interleaved running sums, added
// in order), so the result is the same on every run.
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace awq {
namespace {

constexpr int kWmThreads = 512;
constexpr int kWmWarps = kWmThreads / 32;
constexpr int kWmMaxChunks = 4;        // 16-byte chunks per thread per row: d_in <= 16384
constexpr int kMaxDuoSlices = 64;

// Shape of the weight-mean copy ring for CPT 16-byte chunks per thread and
// row: RB rows per batch (one block barrier per batch for the row maxima),
// NB batches in flight.  NB * RB * CPT * 8 KB of shared memory: 128 KB for
// d_in <= 4096, 192 KB above, i.e. 6-16 rows of 8-32 KB in flight per SM.
template <int CPT> struct WmShape;
template <> struct WmShape<1> { static constexpr int RB = 4, NB = 4; };
template <> struct WmShape<2> { static constexpr int RB = 2, NB = 6; };
template <> struct WmShape<3> { static constexpr int RB = 1, NB = 8; };
template <> struct WmShape<4> { static constexpr int RB = 1, NB = 6; };

template <int CPT>
constexpr size_t wm_ring_bytes() {
    return (size_t)WmShape<CPT>::NB * WmShape<CPT>::RB * CPT * kWmThreads * 16;
}

struct WmParams {
    const uint4* W[AWQ_MAX_SEGMENTS];
    int64_t row_begin[AWQ_MAX_SEGMENTS + 1];   // prefix sum of rows per segment
    int n_seg;
    int64_t d_in;
    int64_t rows;
    double* partial;                           // [gridDim.x][d_in]
    int* status;                               // [gridDim.x]: 0, or kDevErrWaitTimeout
};

// Largest |w| of a chunk of eight fp16 values as fp16 bits compared as
// integers: a NaN ranks above inf, inf above every finite value.
__device__ __forceinline__ uint32_t chunk_maxbits(const uint4 v) {
    uint32_t m = __vmaxu2(__vmaxu2(v.x & 0x7fff7fffu, v.y & 0x7fff7fffu),
                          __vmaxu2(v.z & 0x7fff7fffu, v.w & 0x7fff7fffu));
    return max(m & 0xffffu, m >> 16);
}

// The same without NaN (a NaN half counts as 0): the row maximum the method
// takes when a row holds a NaN.
__device__ __forceinline__ uint32_t chunk_maxbits_nonan(const uint4 v) {
    const uint32_t w[4] = {v.x & 0x7fff7fffu, v.y & 0x7fff7fffu, v.z & 0x7fff7fffu,
                           v.w & 0x7fff7fffu};
    uint32_t m = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t keep = ~__vcmpgtu2(w[i], 0x7c007c00u);   // 0 where the half is NaN
        m = __vmaxu2(m, w[i] & keep);
    }
    return max(m & 0xffffu, m >> 16);
}

__device__ __forceinline__ float half_bits_to_float(uint32_t h) {
    return __half2float(__ushort_as_half((unsigned short)h));
}

// 1-D bulk copy global -> shared (the TMA engine), completion counted on bar.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes,
                                          uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        :: "r"(smem_addr(dst)), "l"(src), "r"(bytes), "r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// One CTA of 512 threads per SM over a contiguous range of rows.  Thread 0
// streams the rows into a shared ring of NB stages of RB rows (one bulk copy
// per row, one mbarrier per stage); thread t reads the 8-column chunks t,
// t + 512, ... of every row, takes their |w| maxima and, after the batch's
// block-wide row maxima, adds |w| / rowmax (fp64, correctly rounded via
// ddiv_rn_rcp) into fp64 sums held in registers, rows in order.  A stage is
// refilled after the batch's block barrier, when every thread has its chunks
// in registers.  A wait that runs out of time ends the CTA's loop (the flag
// is read after the barrier, so every thread leaves together), thread 0
// waits (bounded) for the copies still in flight, and the CTA's status word
// records the timeout.
template <int CPT>
__global__ void __launch_bounds__(kWmThreads, 1)
wmean_partial_kernel(const __grid_constant__ WmParams p) {
    constexpr int RB = WmShape<CPT>::RB, NB = WmShape<CPT>::NB;
    extern __shared__ __align__(128) uint4 ring[];   // [NB][RB] rows of d_in fp16
    __shared__ uint64_t full[NB];
    __shared__ uint32_t red[2][RB][kWmWarps];
    __shared__ uint32_t red_nan[kWmWarps];
    __shared__ int failed_s;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t chunks = p.d_in / 8;
    const uint32_t row_bytes = (uint32_t)(p.d_in * 2);
    const int64_t r0 = p.rows * blockIdx.x / gridDim.x;
    const int64_t r1 = p.rows * (blockIdx.x + 1) / gridDim.x;
    const int64_t n_batches = (r1 - r0 + RB - 1) / RB;
    bool mine[CPT];
#pragma unroll
    for (int c = 0; c < CPT; ++c) mine[c] = tid + (int64_t)c * kWmThreads < chunks;
    if (tid == 0) {
        for (int s = 0; s < NB; ++s) mbar_init(&full[s], 1);
        mbar_fence_init();
        failed_s = 0;
    }
    __syncthreads();
    pdl_wait();   // W may come from the kernel before

    auto row_ptr = [&](int64_t r) {
        int k = 0;
        while (k + 1 < p.n_seg && r >= p.row_begin[k + 1]) ++k;
        return p.W[k] + (r - p.row_begin[k]) * chunks;
    };
    // Batch b into ring stage b % NB (thread 0).
    auto issue = [&](int64_t b) {
        if (b >= n_batches) return;
        const int st = (int)(b % NB);
        const int64_t rb0 = r0 + b * RB;
        const int n_rows = (int)(r1 - rb0 < RB ? r1 - rb0 : RB);
        mbar_arrive_expect_tx(&full[st], (uint32_t)n_rows * row_bytes);
        for (int k = 0; k < n_rows; ++k)
            bulk_load(ring + ((int64_t)st * RB + k) * chunks, row_ptr(rb0 + k), row_bytes,
                      &full[st]);
    };
    if (tid == 0)
        for (int b = 0; b < NB; ++b) issue(b);

    double acc[CPT][8];
#pragma unroll
    for (int c = 0; c < CPT; ++c)
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[c][e] = 0.0;
    const uint4 z = make_uint4(0, 0, 0, 0);
    bool failed = false;
    int64_t b = 0;
    for (; b < n_batches; ++b) {
        const int st = (int)(b % NB);
        if (!mbar_wait_bounded(&full[st], (uint32_t)(b / NB) & 1u))
            *(volatile int*)&failed_s = 1;
        const uint4* rs = ring + (int64_t)st * RB * chunks;
        uint4 v[RB][CPT];
#pragma unroll
        for (int k = 0; k < RB; ++k) {
            const bool row_ok = r0 + b * RB + k < r1;   // the last batch may be short
#pragma unroll
            for (int c = 0; c < CPT; ++c)
                v[k][c] = (row_ok && mine[c]) ? rs[k * chunks + tid + c * kWmThreads] : z;
        }
        uint32_t m[RB];
#pragma unroll
        for (int k = 0; k < RB; ++k) {
            m[k] = 0;
#pragma unroll
            for (int c = 0; c < CPT; ++c) m[k] = max(m[k], chunk_maxbits(v[k][c]));
        }
#pragma unroll
        for (int k = 0; k < RB; ++k) m[k] = __reduce_max_sync(0xffffffffu, m[k]);
        const int slot = (int)(b & 1);   // two slots: one barrier per batch suffices
        if (lane == 0)
#pragma unroll
            for (int k = 0; k < RB; ++k) red[slot][k][warp] = m[k];
        __syncthreads();
        if (*(volatile int*)&failed_s) {   // the same value in every thread
            failed = true;
            break;
        }
        if (tid == 0) {   // every thread holds its chunks of the stage: refill it
            fence_proxy_async_smem();
            issue(b + NB);
        }
#pragma unroll
        for (int k = 0; k < RB; ++k) {
            uint32_t mk = 0;
#pragma unroll
            for (int w = 0; w < kWmWarps; ++w) mk = max(mk, red[slot][k][w]);
            m[k] = mk;
        }
        // One reciprocal per warp and batch: lane k takes row k's.  Rows whose
        // maximum is finite and positive take the scaled quotient (both
        // operands times 2^-896, exact; see f32_scaled_f64).
        uint32_t m_l = m[0];
#pragma unroll
        for (int k = 1; k < RB; ++k)
            if (lane == k) m_l = m[k];
        const double ys_l = __drcp_rn(f32_scaled_f64(half_bits_to_float(m_l)));
#pragma unroll
        for (int k = 0; k < RB; ++k) {
            const uint32_t mb = m[k];        // the same in every thread of the CTA
            const double ys = __shfl_sync(0xffffffffu, ys_l, k);
            if (mb - 1u < 0x7bffu) {         // 0 < max <= 65504
                const double ms = f32_scaled_f64(half_bits_to_float(mb));
#pragma unroll
                for (int c = 0; c < CPT; ++c) {
                    if (mine[c]) {
                        const uint32_t w[4] = {v[k][c].x & 0x7fff7fffu, v[k][c].y & 0x7fff7fffu,
                                               v[k][c].z & 0x7fff7fffu, v[k][c].w & 0x7fff7fffu};
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[i]));
                            acc[c][2 * i] += ddiv_rn_rcp(f32_scaled_f64(f.x), ms, ys);
                            acc[c][2 * i + 1] += ddiv_rn_rcp(f32_scaled_f64(f.y), ms, ys);
                        }
                    }
                }
            } else if (mb != 0) {
                // A non-finite weight in the row (uniform branch): the maximum
                // skips NaN, each term is the IEEE quotient (inf / inf and
                // NaN / max give NaN), and a zero maximum adds nothing.
                uint32_t mn = 0;
#pragma unroll
                for (int c = 0; c < CPT; ++c) mn = max(mn, chunk_maxbits_nonan(v[k][c]));
                mn = __reduce_max_sync(0xffffffffu, mn);
                if (lane == 0) red_nan[warp] = mn;
                __syncthreads();
                mn = 0;
#pragma unroll
                for (int w = 0; w < kWmWarps; ++w) mn = max(mn, red_nan[w]);
                __syncthreads();   // red_nan is free for the next such row
                const double mx = (double)half_bits_to_float(mn);
                if (mn != 0) {
#pragma unroll
                    for (int c = 0; c < CPT; ++c) {
                        if (mine[c]) {
                            const uint32_t w[4] = {v[k][c].x, v[k][c].y, v[k][c].z, v[k][c].w};
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                const double a0 = fabs((double)half_bits_to_float(w[i] & 0xffffu));
                                const double a1 = fabs((double)half_bits_to_float(w[i] >> 16));
                                acc[c][2 * i] += __ddiv_rn(a0, mx);
                                acc[c][2 * i + 1] += __ddiv_rn(a1, mx);
                            }
                        }
                    }
                }
            }
        }
    }
    if (failed && tid == 0) {
        // batches b .. b + NB - 1 may still have copies in flight
        for (int64_t bb = b; bb < b + NB && bb < n_batches; ++bb)
            if (!mbar_wait_drain(&full[bb % NB], (uint32_t)(bb / NB) & 1u)) failed = true;
    }
    if (tid == 0) p.status[blockIdx.x] = failed ? kDevErrWaitTimeout : 0;
    pdl_launch_dependents();
    double* out = p.partial + (int64_t)blockIdx.x * p.d_in;
#pragma unroll
    for (int c = 0; c < CPT; ++c) {
        const int64_t ch = tid + (int64_t)c * kWmThreads;
        if (mine[c]) {
            double2* o2 = reinterpret_cast<double2*>(out + 8 * ch);
#pragma unroll
            for (int e = 0; e < 4; ++e) o2[e] = make_double2(acc[c][2 * e], acc[c][2 * e + 1]);
        }
    }
}

template <int CPT>
cudaError_t launch_wmean_partial(const WmParams& p, int grid, cudaStream_t stream) {
    constexpr size_t smem = wm_ring_bytes<CPT>();
    static int configured[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64 || !configured[dev]) {
        cudaError_t e = cudaFuncSetAttribute(wmean_partial_kernel<CPT>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) configured[dev] = 1;
    }
    return launch_pdl(wmean_partial_kernel<CPT>, dim3(grid), dim3(kWmThreads), smem, stream, p);
}

__device__ __forceinline__ double duo_value(float xj, double wm, double r) {
    const double v = __ddiv_rn(pow((double)xj, r), pow(wm, 1.0 - r) + 1e-4);
    return v < 1e-4 ? 1e-4 : v;
}

constexpr int kCandCols = 32;    // columns per candidates CTA: one per lane
constexpr int kCandWarps = 8;

// One CTA per 32 columns.  Warp w adds the per-CTA column sums w, w + 8,
// w + 16, ... in that order and the eight warp sums are then added in warp
// order (a fixed order, so every run gives the same w_mean), / R.  Then for
// every alpha (warp w takes alphas w, w + 8, ...; lane = column) the
// candidate v in fp64, stored for the write kernel, and its max and min over
// the CTA's columns.  Block 0 also sets the search's error word from the
// weight-mean CTAs' status words and clears its done counter.
__global__ void __launch_bounds__(kCandWarps * 32)
duo_candidates_kernel(const double* __restrict__ partial, const int* __restrict__ wm_status,
                      int n_parts, int64_t d_in, int64_t rows, const float* __restrict__ x,
                      int n_grid,
                      double* __restrict__ V, double* __restrict__ part,
                      int* __restrict__ dev_words) {
    __shared__ double colsum[kCandWarps][kCandCols];
    __shared__ double wm_s[kCandCols];
    pdl_wait();
    pdl_launch_dependents();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (blockIdx.x == 0 && warp == 0) {
        int st = 0;   // a weight-mean CTA's wait that ran out of time
        for (int k = lane; k < n_parts; k += 32) st |= __ldcg(wm_status + k);
        st = (int)__reduce_or_sync(0xffffffffu, (unsigned)st);
        if (lane == 0) {
            dev_words[0] = st;
            dev_words[1] = 0;
        }
    }
    const int64_t j = (int64_t)blockIdx.x * kCandCols + lane;
    const bool col_ok = j < d_in;
    double s = 0.0;
    if (col_ok) {
        constexpr int kBatch = 8;   // loads in flight per lane before they are added in order
        for (int p0 = warp; p0 < n_parts; p0 += kBatch * kCandWarps) {
            double v[kBatch];
#pragma unroll
            for (int k = 0; k < kBatch; ++k) {
                const int pp = p0 + k * kCandWarps;
                v[k] = pp < n_parts ? __ldcg(partial + (int64_t)pp * d_in + j) : 0.0;
            }
#pragma unroll
            for (int k = 0; k < kBatch; ++k)
                if (p0 + k * kCandWarps < n_parts) s += v[k];
        }
    }
    colsum[warp][lane] = s;
    __syncthreads();
    if (warp == 0) {
        double tot = 0.0;
#pragma unroll
        for (int w = 0; w < kCandWarps; ++w) tot += colsum[w][lane];
        wm_s[lane] = __ddiv_rn(tot, (double)rows);
    }
    __syncthreads();
    const float xj = col_ok ? x[j] : 0.f;
    const double wmj = wm_s[lane];
    for (int a = warp; a < n_grid; a += kCandWarps) {
        const double r = __ddiv_rn((double)a, (double)n_grid);
        double mx = 0.0, mn = __longlong_as_double(0x7ff0000000000000ll);
        if (col_ok) {
            const double v = duo_value(xj, wmj, r);
            V[(int64_t)a * d_in + j] = v;
            mx = v;
            mn = v;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            mn = fmin(mn, __shfl_xor_sync(0xffffffffu, mn, o));
        }
        if (lane == 0) {
            part[((int64_t)a * gridDim.x + blockIdx.x) * 2 + 0] = mx;
            part[((int64_t)a * gridDim.x + blockIdx.x) * 2 + 1] = mn;
        }
    }
}

// grid (slices, alphas).  Each CTA takes its alpha's max and min over the
// candidates CTAs' (max, min) pairs (order-independent), then writes the
// slice's S = fp32(v / sqrt(max min)) and T = fp32((x / S)^2).
__global__ void __launch_bounds__(256, 1)
duo_write_kernel(const float* __restrict__ x, const double* __restrict__ V, int64_t d_in,
                 int64_t slice, const double* __restrict__ part, int n_part,
                 float* __restrict__ S, float* __restrict__ T) {
    __shared__ double red_mx[8], red_mn[8];
    pdl_wait();
    pdl_launch_dependents();
    const int a = blockIdx.y, sl = blockIdx.x;
    double mx = 0.0, mn = __longlong_as_double(0x7ff0000000000000ll);
    for (int k = threadIdx.x; k < n_part; k += blockDim.x) {
        mx = fmax(mx, __ldcg(part + ((int64_t)a * n_part + k) * 2 + 0));
        mn = fmin(mn, __ldcg(part + ((int64_t)a * n_part + k) * 2 + 1));
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
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        mx = fmax(mx, red_mx[k]);
        mn = fmin(mn, red_mn[k]);
    }
    const double norm = __dsqrt_rn(__dmul_rn(mx, mn));
    const int64_t j0 = (int64_t)sl * slice, j1 = min(d_in, j0 + slice);
    for (int64_t j = j0 + threadIdx.x; j < j1; j += blockDim.x) {
        const float xj = x[j];
        const float s = __double2float_rn(__ddiv_rn(__ldcg(V + (int64_t)a * d_in + j), norm));
        S[(int64_t)a * d_in + j] = s;
        const double q = __ddiv_rn((double)xj, (double)s);
        T[(int64_t)a * d_in + j] = __double2float_rn(q * q);
    }
}

}  // namespace

size_t duo_workspace(int64_t d_in, int num_sms, int n_grid) {
    const size_t n_cand = (size_t)((d_in + kCandCols - 1) / kCandCols);
    return align_up((size_t)num_sms * (size_t)d_in * sizeof(double), kWsAlign) +
           align_up((size_t)n_grid * (size_t)d_in * sizeof(double), kWsAlign) +
           align_up((size_t)n_grid * n_cand * 2 * sizeof(double), kWsAlign) +
           align_up((size_t)num_sms * sizeof(int), kWsAlign);
}

size_t duo_workspace_bound(int64_t d_in, int n_grid) {
    return duo_workspace(d_in, kDuoMaxSms, n_grid);
}

cudaError_t launch_duo_table(int n_seg, const void* const* W, const int64_t* d_out, int64_t d_in,
                             const float* x_mean, int n_grid, float* S, float* T,
                             int* dev_words, void* duo_ws, int num_sms, cudaStream_t stream) {
    if (d_in > (int64_t)kWmMaxChunks * kWmThreads * 8) return cudaErrorInvalidValue;
    const int grid = std::min(num_sms, kDuoMaxSms);
    const int n_cand = (int)((d_in + kCandCols - 1) / kCandCols);
    char* base = static_cast<char*>(duo_ws);
    double* partial = reinterpret_cast<double*>(base);
    double* V = reinterpret_cast<double*>(
        base + align_up((size_t)grid * (size_t)d_in * sizeof(double), kWsAlign));
    double* part = reinterpret_cast<double*>(
        reinterpret_cast<char*>(V) + align_up((size_t)n_grid * (size_t)d_in * sizeof(double),
                                              kWsAlign));
    int* wm_status = reinterpret_cast<int*>(
        reinterpret_cast<char*>(part) +
        align_up((size_t)n_grid * (size_t)n_cand * 2 * sizeof(double), kWsAlign));

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
    p.status = wm_status;
    const int64_t cpt = (d_in / 8 + kWmThreads - 1) / kWmThreads;
    cudaError_t e = cpt <= 1 ? launch_wmean_partial<1>(p, grid, stream)
                  : cpt == 2 ? launch_wmean_partial<2>(p, grid, stream)
                  : cpt == 3 ? launch_wmean_partial<3>(p, grid, stream)
                             : launch_wmean_partial<4>(p, grid, stream);
    if (e != cudaSuccess) return e;
    e = launch_pdl(duo_candidates_kernel, dim3(n_cand), dim3(kCandWarps * 32), 0, stream,
                   (const double*)partial, (const int*)wm_status, grid, d_in, rows, x_mean,
                   n_grid, V, part, dev_words);
    if (e != cudaSuccess) return e;

    int64_t slices = (2 * (int64_t)num_sms + n_grid - 1) / n_grid;
    slices = std::min<int64_t>(slices, (d_in + 63) / 64);
    slices = std::max<int64_t>(1, std::min<int64_t>(slices, kMaxDuoSlices));
    const int64_t slice = (d_in + slices - 1) / slices;
    slices = (d_in + slice - 1) / slice;
    const dim3 tg((unsigned)slices, (unsigned)n_grid);
    return launch_pdl(duo_write_kernel, tg, dim3(256), 0, stream, x_mean, (const double*)V, d_in,
                      slice, (const double*)part, n_cand, S, T);
}

}  // namespace awq
