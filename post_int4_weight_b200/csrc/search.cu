// search.cu -- the fused AWQ alpha-grid scale search.
//
// Method ("From-Scratch AWQ INT4 Quantization on Qwen3-8B", sections "AWQ
// scaling" and "Group-wise symmetric INT4"; "AWQ architecture, in depth",
// section "The scale search as code"): for every grid point alpha_i the
// candidate scale s_i = max(x,1e-4)^alpha_i / sqrt(max*min) is applied to W,
// W*s_i is fake-quantised group-wise to symmetric INT4 with an fp16 group
// scale, and scored by sum(((W - Q(W s_i)/s_i) * x)^2).
//
// Kernels (all on the caller's stream):
//   scale_table_kernel  one CTA per alpha: s_i in fp64 (pow, max, min, sqrt),
//                       rounded to fp32, and tau_i = x / s_i;
//   search_kernel       persistent, 2 CTAs per SM.  A work unit is one group
//                       of g input channels x R rows of one weight segment.
//                       Thread 0 streams units into a 2-stage shared-memory
//                       ring with TMA (cp.async.bulk.tensor, mbarrier
//                       completion); W is read from HBM exactly once and kept
//                       in registers as fp32 while all grid points are
//                       evaluated;
//   finalize_kernel     sums the per-CTA partials in a fixed order (fp64),
//                       picks the first minimum and copies s_best.
//
// Register-level formulation of one (weight, alpha) pair, 6 FMA-pipe ops plus
// one max, issued as packed fp32x2 instructions (sm_100):
//   ws = w * s                         (exact fp32 product, as the method)
//   m  = max(m, |ws|)                  (then shuffled across the L lanes)
//   t  = ws * (1/q_scale) + 1.5*2^23   (rounds to the nearest code, ties even)
//   q  = t - 1.5*2^23
//   d  = ws - q * q_scale              (= (w - w_hat) * s)
//   e  = d * tau,  tau = x / s         (= (w - w_hat) * x)
//   acc += e * e
// q_scale itself is computed exactly as the method states (IEEE fp32 quotient
// by 7, fp16 round-to-nearest-even).  The code decision uses the reciprocal of
// q_scale instead of the IEEE quotient; the two differ only when ws/q_scale
// lies within an ulp of a half-integer, where either code's error is the same
// to ~1e-7 of a step.  The exact quotient is used where codes are stored
// (pack.cu).
#include <algorithm>
#include <cstring>

#include "common.cuh"
#include "internal.h"

namespace awq {
namespace {

constexpr int kConsumerWarps = 8;
constexpr int kThreads = kConsumerWarps * 32;
constexpr int kStages = 2;
constexpr int kElemsPerLane = 32;          // weights of one row held per lane
constexpr int kUnitBytes = 16384;          // R * g * 2 for every group size
constexpr int kMaxGrid = 32;

struct SearchParams {
    CUtensorMap tmap[AWQ_MAX_SEGMENTS];    // fp16 [d_out_k, d_in], box [g, R]
    int64_t unit_begin[AWQ_MAX_SEGMENTS + 1];  // prefix sum of units per segment
    int32_t row_blocks[AWQ_MAX_SEGMENTS];  // ceil(d_out_k / R)
    int32_t n_seg;
    int32_t group_size;
    int32_t n_grid;
    int32_t flags;
    int64_t n_units;
    int64_t d_in;
    const float* S;        // [n_grid][d_in]
    const float* tau;      // [n_grid][d_in]
    double* partial;       // [gridDim.x][n_grid]
    int* dev_err;
};

__device__ __forceinline__ float2 f2(float a, float b) { return make_float2(a, b); }

// Shared-memory layout of one alpha's table slice for a group of g = 32*L
// channels: float4 index (k4*2 + h)*L + l holds channels 8*(l + L*k4) + 4*h
// + 0..3, so the L lanes of a row read L consecutive 16-byte words (all rows
// of the warp read the same words: a broadcast).
template <int L>
__device__ __forceinline__ int table_slot(int c) {
    const int chunk = c >> 3;
    const int l = chunk % L, k4 = chunk / L, h = (c >> 2) & 1, e = c & 3;
    return (((k4 * 2 + h) * L + l) << 2) + e;
}

template <int L>
__global__ void __launch_bounds__(kThreads, 2)
search_kernel(const __grid_constant__ SearchParams p) {
    constexpr int G = 32 * L;                    // group size
    constexpr int R = kConsumerWarps * 32 / L;   // rows per unit
    static_assert(R * G * 2 == kUnitBytes, "unit size");

    extern __shared__ __align__(1024) unsigned char smem[];
    unsigned char* stage_base = smem;                                   // kStages * 16 KB
    float* tab = reinterpret_cast<float*>(smem + kStages * kUnitBytes); // n_grid * 2 * G
    double* acc = reinterpret_cast<double*>(tab + p.n_grid * 2 * G);    // n_grid * kThreads
    uint64_t* full = reinterpret_cast<uint64_t*>(acc + p.n_grid * kThreads);
    uint64_t* empty = full + kStages;
    int* abort_flag = reinterpret_cast<int*>(empty + kStages);

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int row = warp * (32 / L) + lane / L;   // row within the unit
    const int l = lane % L;                       // sub-lane within the row

    // contiguous, balanced range of units for this CTA
    const int64_t u0 = p.n_units * blockIdx.x / gridDim.x;
    const int64_t u1 = p.n_units * (blockIdx.x + 1) / gridDim.x;

    for (int i = tid; i < p.n_grid * kThreads; i += kThreads) acc[i] = 0.0;
    if (tid == 0) {
        *abort_flag = 0;
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kConsumerWarps);
        }
        mbar_fence_init();
        for (int k = 0; k < p.n_seg; ++k) tma_prefetch_desc(&p.tmap[k]);
    }
    __syncthreads();

    // unit -> (segment, group, row block)
    auto decode = [&](int64_t u, int* seg, int* grp, int* rb) {
        int k = 0;
        while (k + 1 < p.n_seg && u >= p.unit_begin[k + 1]) ++k;
        const int64_t lu = u - p.unit_begin[k];
        *seg = k;
        *grp = (int)(lu / p.row_blocks[k]);
        *rb = (int)(lu % p.row_blocks[k]);
    };
    int issued[kStages] = {};   // loads issued into each stage (thread 0 only)
    auto issue = [&](int64_t u, int stage) {
        int seg, grp, rb;
        decode(u, &seg, &grp, &rb);
        mbar_arrive_expect_tx(&full[stage], kUnitBytes);
        tma_load_2d(stage_base + stage * kUnitBytes, &p.tmap[seg], grp * G, rb * R,
                    &full[stage]);
        ++issued[stage];
    };

    if (tid == 0) {
        for (int s = 0; s < kStages && u0 + s < u1; ++s) issue(u0 + s, s);
    }

    const bool fp32_scale = (p.flags & AWQ_SCALE_FP32) != 0;
    const float2 magic2 = f2(kRoundMagic, kRoundMagic);
    const float2 nmagic2 = f2(-kRoundMagic, -kRoundMagic);
    int cur_grp = -1;
    // Once any bounded wait gives up, the CTA stops computing but keeps the
    // same barrier sequence (no thread leaves a __syncthreads behind).
    bool failed = false;

    for (int64_t u = u0; u < u1; ++u) {
        const int it = (int)(u - u0);
        const int stage = it % kStages;
        const uint32_t parity = (uint32_t)(it / kStages) & 1u;

        // the load of unit u+1 goes into the stage unit u-1 used, once every
        // consumer warp has read unit u-1 out of it
        if (tid == 0 && it >= 1 && u + 1 < u1 && !failed) {
            const int ps = (it - 1) % kStages;
            const uint32_t pp = (uint32_t)((it - 1) / kStages) & 1u;
            if (*(volatile int*)abort_flag == 0 && mbar_wait_bounded(&empty[ps], pp)) {
                issue(u + 1, ps);
            } else {
                atomicOr(p.dev_err, kDevErrWaitTimeout);
                *(volatile int*)abort_flag = 1;
                failed = true;
            }
        }

        int seg, grp, rb;
        decode(u, &seg, &grp, &rb);
        if (grp != cur_grp) {   // uniform: every thread walks the same units
            __syncthreads();
            const float* Sg = p.S + (int64_t)grp * G;
            const float* Tg = p.tau + (int64_t)grp * G;
            for (int i = tid; i < p.n_grid * G; i += kThreads) {
                const int a = i / G, c = i % G;
                const int slot = table_slot<L>(c);
                tab[a * 2 * G + slot] = Sg[(int64_t)a * p.d_in + c];
                tab[a * 2 * G + G + slot] = Tg[(int64_t)a * p.d_in + c];
            }
            cur_grp = grp;
            __syncthreads();
        }

        bool ok = !failed && *(volatile int*)abort_flag == 0;
        if (ok) ok = mbar_wait_bounded(&full[stage], parity);
        if (!failed && !ok) {
            if (lane == 0) {
                atomicOr(p.dev_err, kDevErrWaitTimeout);
                *(volatile int*)abort_flag = 1;
            }
        }
        failed = __any_sync(0xffffffffu, !ok) || failed;
        if (failed) {
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[stage]);
            continue;
        }
        // this lane's 32 weights: chunks l + L*k4 (8 channels each) of its row
        float2 w[kElemsPerLane / 2];
        {
            const uint4* src = reinterpret_cast<const uint4*>(
                stage_base + stage * kUnitBytes + row * G * 2);
#pragma unroll
            for (int k4 = 0; k4 < 4; ++k4) {
                const uint4 v = src[l + L * k4];
                const uint32_t hw[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    w[k4 * 4 + i] = __half22float2(*reinterpret_cast<const __half2*>(&hw[i]));
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[stage]);

        for (int a = 0; a < p.n_grid; ++a) {
            const float4* Sa = reinterpret_cast<const float4*>(tab + a * 2 * G);
            const float4* Ta = reinterpret_cast<const float4*>(tab + a * 2 * G + G);
            float2 ws[kElemsPerLane / 2];
            float m0 = 0.f, m1 = 0.f;
#pragma unroll
            for (int k4 = 0; k4 < 4; ++k4) {
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const float4 s4 = Sa[(k4 * 2 + h) * L + l];
                    const int i0 = k4 * 4 + h * 2;
                    ws[i0] = __fmul2_rn(w[i0], f2(s4.x, s4.y));
                    ws[i0 + 1] = __fmul2_rn(w[i0 + 1], f2(s4.z, s4.w));
                    m0 = fmaxf(m0, fmaxf(fabsf(ws[i0].x), fabsf(ws[i0].y)));
                    m1 = fmaxf(m1, fmaxf(fabsf(ws[i0 + 1].x), fabsf(ws[i0 + 1].y)));
                }
            }
            float m = fmaxf(m0, m1);
#pragma unroll
            for (int o = 1; o < L; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));

            bool in_range;
            const float qs = group_scale(m, fp32_scale, &in_range);
            const float rq = (qs > 0.f) ? __frcp_rn(qs) : 0.f;
            const float2 rq2 = f2(rq, rq);
            const float2 nqs2 = f2(-qs, -qs);
            float2 acc2 = f2(0.f, 0.f);
            if (in_range) {
#pragma unroll
                for (int k4 = 0; k4 < 4; ++k4) {
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const float4 t4 = Ta[(k4 * 2 + h) * L + l];
                        const int i0 = k4 * 4 + h * 2;
#pragma unroll
                        for (int j = 0; j < 2; ++j) {
                            const float2 tau = j ? f2(t4.z, t4.w) : f2(t4.x, t4.y);
                            const float2 t = __ffma2_rn(ws[i0 + j], rq2, magic2);
                            const float2 q = __fadd2_rn(t, nmagic2);
                            const float2 d = __ffma2_rn(q, nqs2, ws[i0 + j]);
                            const float2 e = __fmul2_rn(d, tau);
                            acc2 = __ffma2_rn(e, e, acc2);
                        }
                    }
                }
            } else {   // fp16-subnormal, overflowing, zero or NaN scale: clamp codes
#pragma unroll
                for (int k4 = 0; k4 < 4; ++k4) {
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const float4 t4 = Ta[(k4 * 2 + h) * L + l];
                        const int i0 = k4 * 4 + h * 2;
#pragma unroll
                        for (int j = 0; j < 2; ++j) {
                            const float2 tau = j ? f2(t4.z, t4.w) : f2(t4.x, t4.y);
                            float2 t = __ffma2_rn(ws[i0 + j], rq2, magic2);
                            t.x = fminf(fmaxf(t.x, kRoundMagic - 7.f), kRoundMagic + 7.f);
                            t.y = fminf(fmaxf(t.y, kRoundMagic - 7.f), kRoundMagic + 7.f);
                            const float2 q = __fadd2_rn(t, nmagic2);
                            const float2 d = __ffma2_rn(q, nqs2, ws[i0 + j]);
                            const float2 e = __fmul2_rn(d, tau);
                            acc2 = __ffma2_rn(e, e, acc2);
                        }
                    }
                }
            }
            acc[a * kThreads + tid] += (double)(acc2.x + acc2.y);
        }
    }

    // drain: never leave the CTA while a TMA copy may still write its smem.
    // The n-th load into a stage completes that barrier's phase n.
    if (tid == 0) {
        for (int s = 0; s < kStages; ++s)
            if (issued[s] > 0) (void)mbar_wait_bounded(&full[s], (uint32_t)(issued[s] - 1) & 1u);
    }
    __syncthreads();

    // fixed-order reduction of the per-thread partials: warp w reduces
    // grid points a = w, w + 8, ...
    for (int a = warp; a < p.n_grid; a += kConsumerWarps) {
        double s = 0.0;
        for (int i = lane; i < kThreads; i += 32) s += acc[a * kThreads + i];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if (lane == 0) p.partial[(int64_t)blockIdx.x * p.n_grid + a] = s;
    }
}

__global__ void __launch_bounds__(256)
scale_table_kernel(const float* __restrict__ x, int64_t d_in, int n_grid,
                   float* __restrict__ S, float* __restrict__ tau, int* __restrict__ dev_err) {
    __shared__ double red_mx[32], red_mn[32];
    const int a = blockIdx.x;
    if (dev_err && a == 0 && threadIdx.x == 0) *dev_err = 0;
    const double alpha = __ddiv_rn((double)a, (double)n_grid);
    double mx = -__longlong_as_double(0x7ff0000000000000ll);
    double mn = __longlong_as_double(0x7ff0000000000000ll);
    for (int64_t j = threadIdx.x; j < d_in; j += blockDim.x) {
        const double sd = pow((double)fmaxf(x[j], 1e-4f), alpha);
        mx = fmax(mx, sd);
        mn = fmin(mn, sd);
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
    if (threadIdx.x < 32) {
        const int nw = blockDim.x >> 5;
        mx = threadIdx.x < nw ? red_mx[threadIdx.x] : red_mx[0];
        mn = threadIdx.x < nw ? red_mn[threadIdx.x] : red_mn[0];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            mn = fmin(mn, __shfl_xor_sync(0xffffffffu, mn, o));
        }
        if (threadIdx.x == 0) {
            red_mx[0] = mx;
            red_mn[0] = mn;
        }
    }
    __syncthreads();
    const double norm = __dsqrt_rn(__dmul_rn(red_mx[0], red_mn[0]));
    for (int64_t j = threadIdx.x; j < d_in; j += blockDim.x) {
        const double sd = pow((double)fmaxf(x[j], 1e-4f), alpha);
        const float s = __double2float_rn(__ddiv_rn(sd, norm));
        S[(int64_t)a * d_in + j] = s;
        tau[(int64_t)a * d_in + j] = __fdiv_rn(x[j], s);
    }
}

__global__ void __launch_bounds__(256)
finalize_kernel(const double* __restrict__ partial, int n_parts, int n_grid,
                const float* __restrict__ S, int64_t d_in, const int* __restrict__ dev_err,
                double* __restrict__ err, int32_t* __restrict__ best_idx,
                float* __restrict__ s_best) {
    __shared__ double e_s[kMaxGrid];
    __shared__ int best_s;
    const int t = threadIdx.x;
    if (t < n_grid) {
        double s = 0.0;
        for (int c = 0; c < n_parts; ++c) s += partial[(int64_t)c * n_grid + t];
        e_s[t] = s;
        err[t] = s;
    }
    __syncthreads();
    if (t == 0) {
        int b = 0;
        bool finite = true;
        for (int i = 0; i < n_grid; ++i) {
            if (!isfinite(e_s[i])) finite = false;
            if (e_s[i] < e_s[b]) b = i;
        }
        if (!finite) b = -1;
        if (dev_err && *dev_err) b = -2;
        best_s = b;
        *best_idx = b;
    }
    __syncthreads();
    if (s_best) {
        const int b = best_s;
        for (int64_t j = t; j < d_in; j += blockDim.x)
            s_best[j] = b >= 0 ? S[(int64_t)b * d_in + j] : __int_as_float(0x7fc00000);
    }
}

struct SearchWs {
    float* S;
    float* tau;
    double* partial;
    int* dev_err;
};

size_t max_search_ctas() { return 1024; }

SearchWs carve_search_ws(void* ws, int64_t d_in, int n_grid) {
    char* p = static_cast<char*>(ws);
    SearchWs w;
    const size_t tab = align_up((size_t)n_grid * (size_t)d_in * sizeof(float), kWsAlign);
    w.S = reinterpret_cast<float*>(p);
    w.tau = reinterpret_cast<float*>(p + tab);
    w.partial = reinterpret_cast<double*>(p + 2 * tab);
    w.dev_err = reinterpret_cast<int*>(
        p + 2 * tab + align_up(max_search_ctas() * kMaxGrid * sizeof(double), kWsAlign));
    return w;
}

size_t search_smem_bytes(int group_size, int n_grid) {
    return (size_t)kStages * kUnitBytes + (size_t)n_grid * 2 * group_size * sizeof(float) +
           (size_t)n_grid * kThreads * sizeof(double) + 2 * kStages * sizeof(uint64_t) + 16;
}

template <int L>
cudaError_t launch_search_L(const SearchParams& p, int grid, size_t smem, cudaStream_t st) {
    cudaError_t e = cudaFuncSetAttribute(search_kernel<L>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    search_kernel<L><<<grid, kThreads, smem, st>>>(p);
    return cudaGetLastError();
}

}  // namespace

size_t scale_search_workspace(int64_t d_in, int group_size, int n_grid) {
    (void)group_size;
    const size_t tab = align_up((size_t)n_grid * (size_t)d_in * sizeof(float), kWsAlign);
    return 2 * tab + align_up(max_search_ctas() * kMaxGrid * sizeof(double), kWsAlign) +
           kWsAlign;
}

cudaError_t launch_scale_table(const float* x_mean, int64_t d_in, int n_grid, float* S,
                               float* tau, int* dev_err, cudaStream_t stream) {
    scale_table_kernel<<<n_grid, 256, 0, stream>>>(x_mean, d_in, n_grid, S, tau, dev_err);
    return cudaGetLastError();
}

cudaError_t launch_finalize(const double* partial, int n_parts, int n_grid, const float* S,
                            int64_t d_in, const int* dev_err, double* err,
                            int32_t* best_idx, float* s_best, cudaStream_t stream) {
    finalize_kernel<<<1, 256, 0, stream>>>(partial, n_parts, n_grid, S, d_in, dev_err, err,
                                           best_idx, s_best);
    return cudaGetLastError();
}

awq_status launch_scale_search(int n_seg, const void* const* W, const int64_t* d_out,
                               int64_t d_in, const float* x_mean, int group_size,
                               int n_grid, int flags, double* err, int32_t* best_idx,
                               float* s_best, void* ws, cudaStream_t stream) {
    DeviceInfo dev;
    if (query_device(&dev) != cudaSuccess) return AWQ_ERR_CUDA;
    EncodeTiledFn encode = encode_tiled_fn();
    if (!encode) return AWQ_ERR_CUDA;

    const int L = group_size / 32;
    const int R = kConsumerWarps * 32 / L;
    SearchWs w = carve_search_ws(ws, d_in, n_grid);

    SearchParams p;
    std::memset(&p, 0, sizeof(p));
    p.n_seg = n_seg;
    p.group_size = group_size;
    p.n_grid = n_grid;
    p.flags = flags;
    p.d_in = d_in;
    p.S = w.S;
    p.tau = w.tau;
    p.partial = w.partial;
    p.dev_err = w.dev_err;
    const int64_t G = d_in / group_size;
    int64_t units = 0;
    for (int k = 0; k < n_seg; ++k) {
        const cuuint64_t gdim[2] = {(cuuint64_t)d_in, (cuuint64_t)d_out[k]};
        const cuuint64_t gstride[1] = {(cuuint64_t)d_in * 2};
        const cuuint32_t box[2] = {(cuuint32_t)group_size, (cuuint32_t)R};
        const cuuint32_t estride[2] = {1, 1};
        CUresult r = encode(&p.tmap[k], CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2,
                            const_cast<void*>(W[k]), gdim, gstride, box, estride,
                            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return AWQ_ERR_CUDA;
        p.row_blocks[k] = (int32_t)((d_out[k] + R - 1) / R);
        p.unit_begin[k] = units;
        units += G * p.row_blocks[k];
    }
    p.unit_begin[n_seg] = units;
    p.n_units = units;

    const size_t smem = search_smem_bytes(group_size, n_grid);
    const int per_sm = (2 * (smem + 1024) <= dev.max_smem_per_sm) ? 2 : 1;
    int64_t grid = (int64_t)dev.num_sms * per_sm;
    if (grid > units) grid = units;
    if (grid > (int64_t)max_search_ctas()) grid = (int64_t)max_search_ctas();

    if (launch_scale_table(x_mean, d_in, n_grid, w.S, w.tau, w.dev_err, stream) != cudaSuccess)
        return AWQ_ERR_CUDA;
    cudaError_t e;
    switch (L) {
        case 1: e = launch_search_L<1>(p, (int)grid, smem, stream); break;
        case 2: e = launch_search_L<2>(p, (int)grid, smem, stream); break;
        case 4: e = launch_search_L<4>(p, (int)grid, smem, stream); break;
        default: return AWQ_ERR_UNSUPPORTED;
    }
    if (e != cudaSuccess) return AWQ_ERR_CUDA;
    if (launch_finalize(w.partial, (int)grid, n_grid, w.S, d_in, w.dev_err, err, best_idx,
                        s_best, stream) != cudaSuccess)
        return AWQ_ERR_CUDA;
    return AWQ_OK;
}

}  // namespace awq
