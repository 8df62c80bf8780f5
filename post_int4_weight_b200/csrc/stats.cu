// stats.cu -- per-input-channel activation magnitude x[j] = mean_t |X[t, j]|
// ("From-Scratch AWQ INT4 Quantization on Qwen3-8B", section "AWQ scaling";
// "AWQ architecture, in depth", section "The scale search as code").
//
// A column reduction over X (fp16 [T, ld]), bound by the HBM read of X
// (2 bytes per element).  One launch, no workspace:
//   * a CTA owns 64 channels (8 chunks of 16 bytes) and one eighth of the
//     tokens; the 8 CTAs of a thread-block cluster (1 x 8 x 1) cover all
//     tokens of the same channels;
//   * each thread walks its chunk down every 32nd row of its slice in
//     batches of four 16-byte loads, the next batch issued before the
//     current one is summed, and adds |h| in fp64.  Every |fp16| is an
//     integer multiple of 2^-24 below 2^16, so a sum of up to 4096 of them is
//     an integer multiple of 2^-24 below 2^28: exact in fp64.  Every 4096
//     rows the fp64 sums are moved, exactly, into 64-bit integer counts of
//     2^-24;
//   * the integer sums are added across the warp's row lanes with shuffles
//     into the warp's own shared slots, the warps' slots are added in warp
//     order, and the CTAs' sums meet in CTA 0 of the cluster
//     through distributed shared memory atomics; integer addition makes the
//     result independent of order.  CTA 0 writes x[j] = (sum * 2^-24) / T
//     (fp64 division, rounded to fp32).
// A NaN makes its column's fp64 sum NaN and an infinity makes it +inf; they
// are carried as flag bits (NaN wins).
#include <cooperative_groups.h>

#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace cg = cooperative_groups;

namespace awq {
namespace {

constexpr int kCluster = 8;        // CTAs per cluster, splitting the tokens
constexpr int kChunks = 8;         // 16-byte chunks per CTA (64 channels)
constexpr int kRowLanes = 32;      // rows walked in parallel per CTA
constexpr int kBatch = 4;          // 16-byte loads per batch; the next batch is in flight
                                   // while the current one is summed
constexpr int kFlushRows = 4096;   // rows per thread between exact flushes

// |h| as an fp64 value without the (slow-pipe) fp32 -> fp64 conversion: the
// fp16 -> fp32 conversion is exact, and an fp32 value f with at most 11
// significant bits is the fp64 value whose high word is (bits(f) >> 3) +
// ((1023 - 127) << 20) and whose low word is 0.  Zero maps to 2^-127 instead
// of 0; a sum of integers multiples of 2^-24 is unaffected by such terms once
// it is scaled by 2^24 and rounded to an integer, which is what flush()
// does.  Non-finite inputs are caught separately by the lane's running
// maximum of |h| bit patterns (hmax).
__device__ __forceinline__ void add_halves(const uint4& v, double* acc, uint32_t* hmax) {
    const uint32_t wv[4] = {v.x & 0x7fff7fffu, v.y & 0x7fff7fffu, v.z & 0x7fff7fffu,
                            v.w & 0x7fff7fffu};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        hmax[i] = __vmaxu2(hmax[i], wv[i]);
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&wv[i]));
        const uint32_t hx = (__float_as_uint(f.x) >> 3) + 0x38000000u;
        const uint32_t hy = (__float_as_uint(f.y) >> 3) + 0x38000000u;
        acc[2 * i] += __hiloint2double((int)hx, 0);
        acc[2 * i + 1] += __hiloint2double((int)hy, 0);
    }
}

// Moves the exact fp64 partial sums into integer counts of 2^-24 (or flag
// bits for a column that held a non-finite value: bit 0 infinity, bit 1
// NaN, from the largest |h| bit patterns seen), adds them over the warp's
// row lanes (lanes with the same chunk) and into the warp's own shared
// slots (lanes 0..7 own disjoint entries: no atomics), and clears them.
// Called by every lane of a warp together.  A thread's sum covers at most
// kFlushRows rows of values of at most 65504 (the main loop flushes once it
// reaches kFlushRows; at most kBatch tail rows follow its last flush and
// leave it at most kFlushRows), so sum * 2^24 is an integer below
// 4096 * 65504 * 2^24 < 2^52 (plus the zeros' 2^-127 terms, far below 1/2):
// adding 2^52 rounds it to that integer exactly and leaves it in the low 52
// bits.
__device__ __forceinline__ void flush(double* acc, const uint32_t* hmax, int cx,
                                      unsigned long long* wred, uint32_t* wfred) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const uint32_t hm = (hmax[i >> 1] >> (16 * (i & 1))) & 0xffffu;
        unsigned long long u =
            (unsigned long long)__double_as_longlong(__fma_rn(acc[i], 0x1p24, 0x1p52)) -
            0x4330000000000000ull;
        uint32_t f = 0;
        if (hm > 0x7c00u) {
            f = 2u;
            u = 0;
        } else if (hm == 0x7c00u) {
            f = 1u;
            u = 0;
        }
#pragma unroll
        for (int o = kChunks; o < 32; o <<= 1) {
            u += __shfl_xor_sync(0xffffffffu, u, o);
            f |= __shfl_xor_sync(0xffffffffu, f, o);
        }
        if (lane < kChunks) {
            wred[cx * 8 + i] += u;
            wfred[cx * 8 + i] |= f;
        }
        acc[i] = 0.0;
    }
}

__global__ void __cluster_dims__(1, kCluster, 1) __launch_bounds__(kChunks * kRowLanes, 4)
stats_kernel(const uint4* __restrict__ X, int64_t T, int64_t d_in, int64_t ld_chunks,
             float* __restrict__ x_mean) {
    constexpr int kWarps = kChunks * kRowLanes / 32;
    __shared__ unsigned long long red[kChunks * 8];
    __shared__ uint32_t fred[kChunks * 8];
    __shared__ unsigned long long red_w[kWarps][kChunks * 8];   // per-warp sums
    __shared__ uint32_t fred_w[kWarps][kChunks * 8];
    cg::cluster_group cluster = cg::this_cluster();
    const int rank = (int)cluster.block_rank();

    // a programmatic dependent launch: X may be written by the kernel before
    pdl_wait();
    const int tid = threadIdx.x;
    const int cx = tid % kChunks;
    const int ry = tid / kChunks;
    if (tid < kChunks * 8) {
        red[tid] = 0;
        fred[tid] = 0;
    }
    {   // each warp clears its own slots (only it writes them, in flush)
        const int w = tid >> 5, l = tid & 31;
        for (int i = l; i < kChunks * 8; i += 32) {
            red_w[w][i] = 0;
            fred_w[w][i] = 0;
        }
        __syncwarp();
    }
    // every CTA's accumulators must be cleared before other CTAs add into
    // them: arrive now, wait just before the remote adds (after the loads)
    cluster.barrier_arrive();

    const int64_t chunk = (int64_t)blockIdx.x * kChunks + cx;
    const bool active = chunk * 8 < d_in;
    const int64_t per = (T + kCluster - 1) / kCluster;
    const int64_t r0 = rank * per;
    const int64_t r1 = min(T, r0 + per);

    double acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    uint32_t hmax[4] = {0, 0, 0, 0};   // per word: max |h| bits of its two channels
    const uint4* p = X + (active ? chunk : 0);
    // The 32 lanes of a warp hold row offsets 4w .. 4w+3 (and 8 chunks each):
    // the main loop's trip count depends only on the warp's first row, so
    // every lane of a warp runs it (and the shuffles in flush) together.
    const int64_t warp_row = r0 + (ry & ~3);
    const int sub = ry & 3;
    int64_t base = warp_row;
    int since_flush = 0;
    // software-pipelined batches: the loop's trip count depends only on the
    // warp's first row (every lane of a warp runs it and the flush together)
    uint4 cur[kBatch];
    bool have = base + 3 + (kBatch - 1) * kRowLanes < r1;
    if (have) {
#pragma unroll
        for (int k = 0; k < kBatch; ++k)
            cur[k] = active ? __ldg(p + (base + sub + k * kRowLanes) * ld_chunks)
                            : make_uint4(0, 0, 0, 0);
    }
    while (have) {
        const int64_t nb = base + kBatch * kRowLanes;
        const bool have_next = nb + 3 + (kBatch - 1) * kRowLanes < r1;
        uint4 nxt[kBatch];
        if (have_next) {
#pragma unroll
            for (int k = 0; k < kBatch; ++k)
                nxt[k] = active ? __ldg(p + (nb + sub + k * kRowLanes) * ld_chunks)
                                : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int k = 0; k < kBatch; ++k) add_halves(cur[k], acc, hmax);
        since_flush += kBatch;
        if (since_flush >= kFlushRows) {
            flush(acc, hmax, cx, red_w[tid >> 5], fred_w[tid >> 5]);
            since_flush = 0;
        }
        base = nb;
        have = have_next;
#pragma unroll
        for (int k = 0; k < kBatch; ++k) cur[k] = nxt[k];
    }
    for (int64_t r = base + sub; r < r1; r += kRowLanes)
        if (active) add_halves(__ldg(p + r * ld_chunks), acc, hmax);
    pdl_launch_dependents();   // X is read; the next kernel may start launching
    flush(acc, hmax, cx, red_w[tid >> 5], fred_w[tid >> 5]);
    __syncthreads();
    if (tid < kChunks * 8) {   // the warps' sums, in warp order (integers: exact)
        unsigned long long s = 0;
        uint32_t f = 0;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
            s += red_w[w][tid];
            f |= fred_w[w][tid];
        }
        // other CTAs of the cluster may already be adding into rank 0's red
        if (s) atomicAdd(&red[tid], s);
        if (f) atomicOr(&fred[tid], f);
    }
    __syncthreads();
    cluster.barrier_wait();
    if (rank != 0 && tid < kChunks * 8) {
        unsigned long long* red0 = cluster.map_shared_rank(red, 0);
        uint32_t* fred0 = cluster.map_shared_rank(fred, 0);
        if (red[tid]) atomicAdd(&red0[tid], red[tid]);
        if (fred[tid]) atomicOr(&fred0[tid], fred[tid]);
    }
    cluster.sync();
    if (rank == 0 && tid < kChunks * 8) {
        const int64_t j = (int64_t)blockIdx.x * kChunks * 8 + tid;
        if (j < d_in) {
            const uint32_t f = fred[tid];
            float v;
            if (f & 2u) {
                v = __int_as_float(0x7fc00000);
                raise_device_flag(AWQ_FLAG_NONFINITE_X);
            } else if (f & 1u) {
                v = __int_as_float(0x7f800000);
                raise_device_flag(AWQ_FLAG_NONFINITE_X);
            } else {
                const double s = __ull2double_rn(red[tid]);
                v = __double2float_rn(__ddiv_rn(s * 0x1p-24, (double)T));
            }
            x_mean[j] = v;
        }
    }
}

}  // namespace

cudaError_t stats_unit_flags(unsigned int* bits, bool clear) {
    return unit_device_flags(bits, clear);
}

size_t act_stats_workspace(int64_t d_in) {
    (void)d_in;
    return 0;
}

cudaError_t launch_act_stats(const void* X, int64_t T, int64_t d_in, int64_t ld,
                             float* x_mean, void* ws, cudaStream_t stream) {
    (void)ws;
    const int64_t col_blocks = (d_in / 8 + kChunks - 1) / kChunks;
    dim3 grid((unsigned)col_blocks, kCluster);
    return launch_pdl(stats_kernel, grid, dim3(kChunks * kRowLanes), 0, stream,
                      static_cast<const uint4*>(X), T, d_in, ld / 8, x_mean);
}

}  // namespace awq
