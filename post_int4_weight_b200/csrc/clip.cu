// clip.cu -- per (row, group) search of a shrunk quantisation range at a
// fixed scale s ("AWQ architecture, in depth", section "The pipeline end to
// end", step 5: an optional search of a clipping range per output channel
// that shrinks the quantisation range to cut rounding error on outliers;
// "AWQ, Reproduced": the paper also clips the weight range).
//
// For every row r and group k and every ratio index i < n_clip, with
// c_i = RN((20 - i) / 20):
//   m     = max_j |fl32(w_j s_j)|            over the group
//   q_s   = fp16_rne(fl32(fl32(c_i m) / 7))  (exactly as awq_quantize_pack)
//   q_j   = clamp(rint(ws_j / q_s), -7, 7)
//   e_i   = sum_j (ws_j - q_j q_s)^2 (x_j / s_j)^2
// and the first i with the smallest e_i is stored.  The totals at i = 0 and
// at the chosen indices are reduced in a fixed order (deterministic).
//
// Work and roofline: n_clip x (the scale search's per-pair arithmetic) per
// weight with W read once (2 B), so it is FP32-ALU-bound like the search.
// One warp task = one group of g channels x 2 * 32 / L rows (L = g / 16
// lanes per row, 16 weights of two rows per lane, the search's layout);
// tasks are dealt to warps in a fixed order by a persistent grid, so every
// CTA's partial, and the final sums, are the same on every run.
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace awq {
namespace {

constexpr int kClipWarps = 8;
constexpr int kClipThreads = kClipWarps * 32;
constexpr int kClipCtasPerSm = 2;
constexpr int kMaxClipCtas = 1024;
constexpr int kClipDen = 20;

struct ClipParams {
    const uint4* W;        // fp16 [d_out, d_in], rows of d_in / 8 chunks
    int64_t d_out;
    int64_t d_in;
    const float* tau2;     // [d_in] (x / s)^2, from clip_tau_kernel
    const float* s;        // [d_in] or NULL (s = 1)
    int64_t groups;        // d_in / g
    int64_t n_tasks;       // row blocks x groups
    int n_clip;
    int fp32_scale;
    uint8_t* idx;          // [d_out, groups]
    double* partial;       // [gridDim.x][2]
    int* counter;          // CTAs done (zeroed before the launch)
    double* err;           // [2]
};

__device__ __forceinline__ float2 f2(float a, float b) { return make_float2(a, b); }

// 16 channels of one lane: chunks (8 channels) l and l + L of the group
__device__ __forceinline__ void load_chunk_f32(const float* p, float* v) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(p));
    const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

__device__ __forceinline__ void unpack8(const uint4 v, float2* w) {
    const uint32_t hw[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) w[i] = __half22float2(*reinterpret_cast<const __half2*>(&hw[i]));
}

// Error of the lane's 16 weights of one row at group scale qs (reciprocal
// rq; 0 for a zero group): codes by the rounding addition, clamped to +-7.
__device__ __forceinline__ float lane_error(const float2* ws, const float2* t2, float qs,
                                            float rq) {
    const float2 nqs = f2(-qs, -qs), rq2 = f2(rq, rq);
    const float2 magic2 = f2(kRoundMagic, kRoundMagic), nmagic2 = f2(-kRoundMagic, -kRoundMagic);
    float2 acc = f2(0.f, 0.f);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        float2 t = __ffma2_rn(ws[i], rq2, magic2);
        t = f2(fminf(fmaxf(t.x, kRoundMagic - 7.f), kRoundMagic + 7.f),
               fminf(fmaxf(t.y, kRoundMagic - 7.f), kRoundMagic + 7.f));
        const float2 q = __fadd2_rn(t, nmagic2);
        const float2 d = __ffma2_rn(q, nqs, ws[i]);
        acc = __ffma2_rn(__fmul2_rn(d, d), t2[i], acc);
    }
    return acc.x + acc.y;
}

template <int L>
__device__ __forceinline__ float row_max(float v) {
#pragma unroll
    for (int o = 1; o < L; o <<= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

template <int L>
__global__ void __launch_bounds__(kClipThreads, kClipCtasPerSm)
clip_kernel(const ClipParams p) {
    constexpr int G = 16 * L;               // group size
    constexpr int kSlots = 32 / L;          // row pairs per warp task
    constexpr int RPT = 2 * kSlots;         // rows per task
    __shared__ double red[kClipWarps][2];
    __shared__ int last;
    __shared__ float ratio[AWQ_CLIP_MAX];   // c_i = RN((20 - i) / 20), once per CTA

    if (threadIdx.x < AWQ_CLIP_MAX)
        ratio[threadIdx.x] = __fdiv_rn((float)(kClipDen - (int)threadIdx.x), (float)kClipDen);
    __syncthreads();
    pdl_wait();   // W, x and s may come from the kernel before
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int l = lane % L, slot = lane / L;
    const int64_t ld = p.d_in / 8;
    double tot0 = 0.0, tot1 = 0.0;   // rows this lane reports (l == 0: row 0, l == 1: row 1)

    const int64_t n_warps = (int64_t)gridDim.x * kClipWarps;
    for (int64_t t = (int64_t)blockIdx.x * kClipWarps + warp; t < p.n_tasks; t += n_warps) {
        const int64_t rb = t / p.groups;
        const int64_t k = t % p.groups;
        const int64_t r0 = rb * RPT + slot, r1 = r0 + kSlots;
        const bool v0 = r0 < p.d_out, v1 = r1 < p.d_out;
        const int64_t ch0 = k * G + 8 * l, ch1 = ch0 + 8 * L;   // first channels of the chunks

        float2 ws0[8], ws1[8], t2[8];
        {
            float sv[16], tv[16];
            if (p.s) {
                load_chunk_f32(p.s + ch0, sv);
                load_chunk_f32(p.s + ch1, sv + 8);
            } else {
#pragma unroll
                for (int i = 0; i < 16; ++i) sv[i] = 1.f;
            }
            load_chunk_f32(p.tau2 + ch0, tv);
            load_chunk_f32(p.tau2 + ch1, tv + 8);
            const uint4 z = make_uint4(0, 0, 0, 0);
            const uint4 a0 = v0 ? __ldg(p.W + r0 * ld + ch0 / 8) : z;
            const uint4 b0 = v0 ? __ldg(p.W + r0 * ld + ch1 / 8) : z;
            const uint4 a1 = v1 ? __ldg(p.W + r1 * ld + ch0 / 8) : z;
            const uint4 b1 = v1 ? __ldg(p.W + r1 * ld + ch1 / 8) : z;
            float2 w0[8], w1[8];
            unpack8(a0, w0);
            unpack8(b0, w0 + 4);
            unpack8(a1, w1);
            unpack8(b1, w1 + 4);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float2 s2 = f2(sv[2 * i], sv[2 * i + 1]);
                ws0[i] = __fmul2_rn(w0[i], s2);
                ws1[i] = __fmul2_rn(w1[i], s2);
                t2[i] = f2(tv[2 * i], tv[2 * i + 1]);
            }
        }
        // group maxima; fmaxf drops NaN, so a NaN product is tracked apart and
        // makes the whole row group's maximum NaN
        float m0 = 0.f, m1 = 0.f;
        bool nan0 = false, nan1 = false;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            m0 = fmaxf(m0, fmaxf(fabsf(ws0[i].x), fabsf(ws0[i].y)));
            m1 = fmaxf(m1, fmaxf(fabsf(ws1[i].x), fabsf(ws1[i].y)));
            nan0 |= (ws0[i].x != ws0[i].x) | (ws0[i].y != ws0[i].y);
            nan1 |= (ws1[i].x != ws1[i].x) | (ws1[i].y != ws1[i].y);
        }
        m0 = row_max<L>(m0);
        m1 = row_max<L>(m1);
#pragma unroll
        for (int o = 1; o < L; o <<= 1) {
            nan0 |= __shfl_xor_sync(0xffffffffu, (int)nan0, o) != 0;
            nan1 |= __shfl_xor_sync(0xffffffffu, (int)nan1, o) != 0;
        }
        if (nan0) m0 = __int_as_float(0x7fc00000);
        if (nan1) m1 = __int_as_float(0x7fc00000);

        // Each lane pair splits the two rows: even lanes finish row 0's group
        // scale, error sum and best ratio, odd lanes row 1's.  The error sum
        // is the same pairwise tree as a butterfly over the row's lanes.
        const bool odd = (lane & 1) != 0;
        const int even = lane & ~1;
        const float m_own = odd ? m1 : m0;
        float e_first = 0.f, best = 0.f;
        int b_own = 0;
        for (int i = 0; i < p.n_clip; ++i) {
            const float c = ratio[i];
            bool unused;
            const float qs = group_scale(__fmul_rn(m_own, c), p.fp32_scale != 0, &unused);
            const float rq = qs > 0.f ? rcp_approx(qs) : (qs == 0.f ? 0.f : qs);
            const float qs0 = __shfl_sync(0xffffffffu, qs, even);
            const float qs1 = __shfl_sync(0xffffffffu, qs, even | 1);
            const float rq0 = __shfl_sync(0xffffffffu, rq, even);
            const float rq1 = __shfl_sync(0xffffffffu, rq, even | 1);
            const float ea = lane_error(ws0, t2, qs0, rq0);
            const float eb = lane_error(ws1, t2, qs1, rq1);
            float e = (odd ? eb : ea) + __shfl_xor_sync(0xffffffffu, odd ? ea : eb, 1);
#pragma unroll
            for (int o = 2; o < L; o <<= 1) e += __shfl_xor_sync(0xffffffffu, e, o);
            if (i == 0) {
                e_first = best = e;
            } else if (e < best) {
                best = e;
                b_own = i;
            }
        }
        if (l < 2 && (odd ? v1 : v0)) {   // l == 0 reports row 0, l == 1 row 1
            p.idx[(odd ? r1 : r0) * p.groups + k] = (uint8_t)b_own;
            tot0 += (double)e_first;
            tot1 += (double)best;
        }
    }
    pdl_launch_dependents();

    // fixed-order reduction: warp tree, then warps in order, then (last CTA)
    // the CTAs' partials in a fixed order
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        tot0 += __shfl_xor_sync(0xffffffffu, tot0, o);
        tot1 += __shfl_xor_sync(0xffffffffu, tot1, o);
    }
    if (lane == 0) {
        red[warp][0] = tot0;
        red[warp][1] = tot1;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        double a = 0.0, b = 0.0;
        for (int w = 0; w < kClipWarps; ++w) {
            a += red[w][0];
            b += red[w][1];
        }
        p.partial[2 * blockIdx.x] = a;
        p.partial[2 * blockIdx.x + 1] = b;
        __threadfence();
        last = (atomicAdd(p.counter, 1) == (int)gridDim.x - 1);
    }
    __syncthreads();
    if (last && warp == 0) {
        __threadfence();
        // lane k adds the CTAs k, k + 32, k + 64, ... in that order (every
        // load of a batch in flight before its adds), then a fixed shuffle
        // tree: the same order on every run
        constexpr int kB = 8;
        const int n = (int)gridDim.x;
        double a = 0.0, b = 0.0;
        for (int c0 = 0; c0 < n; c0 += 32 * kB) {
            double va[kB], vb[kB];
#pragma unroll
            for (int k = 0; k < kB; ++k) {
                const int c = c0 + lane + 32 * k;
                va[k] = c < n ? __ldcg(p.partial + 2 * c) : 0.0;
                vb[k] = c < n ? __ldcg(p.partial + 2 * c + 1) : 0.0;
            }
#pragma unroll
            for (int k = 0; k < kB; ++k) {
                a += va[k];
                b += vb[k];
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            a += __shfl_xor_sync(0xffffffffu, a, o);
            b += __shfl_xor_sync(0xffffffffu, b, o);
        }
        if (lane == 0) {
            p.err[0] = a;
            p.err[1] = b;
            if (!isfinite(a) || !isfinite(b)) raise_device_flag(AWQ_FLAG_NONFINITE_SCORE);
        }
    }
}

// tau2[j] = (RN(x_j / s_j))^2 in fp32, once per call (every task of a
// column's group reads it)
__global__ void __launch_bounds__(256)
clip_tau_kernel(const float* __restrict__ x, const float* __restrict__ s, int64_t d_in,
                float* __restrict__ tau2) {
    pdl_wait();   // x and s may come from the kernel before
    pdl_launch_dependents();
    for (int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; j < d_in;
         j += (int64_t)gridDim.x * blockDim.x) {
        const float t = s ? __fdiv_rn(x[j], s[j]) : x[j];
        tau2[j] = __fmul_rn(t, t);
    }
}

template <int L>
cudaError_t launch_clip_L(const ClipParams& p, int grid, cudaStream_t st) {
    return launch_pdl(clip_kernel<L>, dim3(grid), dim3(kClipThreads), 0, st, p);
}

}  // namespace

cudaError_t clip_unit_flags(unsigned int* bits, bool clear) {
    return unit_device_flags(bits, clear);
}

size_t clip_search_workspace(int64_t d_in) {
    return align_up((size_t)kMaxClipCtas * 2 * sizeof(double), kWsAlign) + kWsAlign +
           align_up((size_t)d_in * sizeof(float), kWsAlign);
}

cudaError_t launch_clip_search(const void* W, int64_t d_out, int64_t d_in, const float* x_mean,
                               const float* s, int group_size, int n_clip, int flags,
                               uint8_t* clip_idx, double* err, void* ws, cudaStream_t stream) {
    DeviceInfo dev;
    cudaError_t e = query_device(&dev);
    if (e != cudaSuccess) return e;
    const int L = group_size / 16;
    const int64_t rows_per_task = 2 * 32 / L;
    ClipParams p;
    p.W = static_cast<const uint4*>(W);
    p.d_out = d_out;
    p.d_in = d_in;
    p.s = s;
    p.groups = d_in / group_size;
    p.n_tasks = (d_out + rows_per_task - 1) / rows_per_task * p.groups;
    p.n_clip = n_clip;
    p.fp32_scale = (flags & AWQ_SCALE_FP32) ? 1 : 0;
    p.idx = clip_idx;
    char* base = static_cast<char*>(ws);
    p.partial = reinterpret_cast<double*>(base);
    p.counter = reinterpret_cast<int*>(
        base + align_up((size_t)kMaxClipCtas * 2 * sizeof(double), kWsAlign));
    float* tau2 = reinterpret_cast<float*>(
        base + align_up((size_t)kMaxClipCtas * 2 * sizeof(double), kWsAlign) + kWsAlign);
    p.tau2 = tau2;
    p.err = err;
    int64_t grid = (int64_t)dev.num_sms * kClipCtasPerSm;
    const int64_t need = (p.n_tasks + kClipWarps - 1) / kClipWarps;
    if (grid > need) grid = need;
    if (grid > kMaxClipCtas) grid = kMaxClipCtas;
    if (grid < 1) grid = 1;
    e = cudaMemsetAsync(p.counter, 0, sizeof(int), stream);
    if (e != cudaSuccess) return e;
    const int tau_blocks = (int)std::min<int64_t>((d_in + 255) / 256, 4 * (int64_t)dev.num_sms);
    e = launch_pdl(clip_tau_kernel, dim3(tau_blocks), dim3(256), 0, stream, x_mean, s, d_in, tau2);
    if (e != cudaSuccess) return e;
    switch (L) {
        case 2: return launch_clip_L<2>(p, (int)grid, stream);
        case 4: return launch_clip_L<4>(p, (int)grid, stream);
        case 8: return launch_clip_L<8>(p, (int)grid, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace awq
