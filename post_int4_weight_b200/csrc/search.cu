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
//   table_kernel   (slices x alphas) CTAs.  pow is monotonic in x, so
//                  max_j s_i[j] and min_j s_i[j] come from the largest and
//                  smallest max(x_j, 1e-4), which every CTA finds by itself;
//                  then s_i[j] = pow(max(x_j,1e-4), alpha_i) / sqrt(max*min)
//                  (fp64, rounded once to fp32) and tau2_i[j] = (x_j/s_i[j])^2
//                  for the CTA's slice of channels.
//   search_kernel  persistent, one CTA of 16 warps per SM (a programmatic
//                  dependent launch of the table kernel).  A work unit is one
//                  group of g input channels x R rows of one weight segment.
//                  Thread 0 streams units into a 2-stage shared-memory ring
//                  with TMA (cp.async.bulk.tensor, mbarrier completion),
//                  starting before the scale table is ready; W is read from
//                  HBM exactly once and kept in registers as fp32 while all
//                  grid points are evaluated.  The last CTA to finish sums
//                  the per-CTA partials in a fixed order (fp64), picks the
//                  first minimum and copies s_best.
// One CTA per SM (rather than two of 8 warps) keeps the SM's warps on one
// range of units: two co-resident CTAs drift apart under the scheduler's
// age priority and the later one ends alone on its SM.
//
// Register-level formulation of one (weight, alpha) pair: 5.5 FMA-pipe lane
// operations and one max, every FMA-pipe operation a packed fp32x2
// instruction (sm_100): a packed instruction does two lane operations in one
// issue slot, and a measured FMA stream reaches the same lane-op rate packed
// or scalar, so packing leaves issue slots for the maxima, shuffles and
// shared-memory reads.  Each lane holds the same 16 channels of two rows
// r0, r1:
//   ws = w * s                         (exact fp32 product, as the method)
//   m  = max(m, |ws|)                  (then shuffled across the L lanes)
//   t  = ws * (1/q_scale) + 1.5*2^23   (rounds to the nearest code, ties even)
//   q  = t - 1.5*2^23
//   d  = ws - q * q_scale              (= (w - w_hat) * s)
//   acc += tau2 * (d_r0^2 + d_r1^2),   tau2 = (x / s)^2
// so that ((w - w_hat) * x)^2 = d^2 * tau2 is summed without forming each
// product d * tau.  The error pass of one alpha is fused with the products
// and row maxima of the next (rows_errors_next), so the two kinds of work
// interleave in one instruction stream.  q_scale itself is computed exactly as the method states
// (IEEE fp32 quotient by 7, fp16 round-to-nearest-even).  The code decision
// uses the reciprocal of q_scale instead of the IEEE quotient; the two differ
// only when ws/q_scale lies within an ulp of a half-integer, where either
// code's error is the same to ~1e-7 of a step.  The exact quotient is used
// where codes are stored (pack.cu).
#include <algorithm>
#include <cstring>

#include "common.cuh"
#include "internal.h"

namespace awq {
namespace {

constexpr int kConsumerWarps = 16;
constexpr int kThreads = kConsumerWarps * 32;
constexpr int kStages = 2;
constexpr int kElemsPerRow = 16;           // weights of each of a lane's two rows
constexpr int kUnitBytes = 32768;          // R * g * 2 for every group size
constexpr int kMaxBoxRows = 256;           // TMA box limit: R is loaded in boxes of <= 256 rows
constexpr int kMaxGrid = 32;
constexpr int kMaxParts = 1024;            // per-CTA partials (grid size bound)

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
    const float* tau2;     // [n_grid][d_in], (x / s)^2
    double* partial;       // [gridDim.x][n_grid]
    int* dev_words;        // [0] error bits, [1] CTAs done
    double* err;           // [n_grid] output
    int32_t* best_idx;     // [1] output
    float* s_best;         // [d_in] output
};

__device__ __forceinline__ float2 f2(float a, float b) { return make_float2(a, b); }

// Shared-memory layout of one alpha's table slice for a group of g = 16*L
// channels: float4 index (k2*2 + h)*L + l holds channels 8*(l + L*k2) + 4*h
// + 0..3, so the L lanes of a row read L consecutive 16-byte words (all rows
// of the warp read the same words: a broadcast).
template <int L>
__device__ __forceinline__ int table_slot(int c) {
    const int chunk = c >> 3;
    const int l = chunk % L, k2 = chunk / L, h = (c >> 2) & 1, e = c & 3;
    return (((k2 * 2 + h) * L + l) << 2) + e;
}

// Sum of the CTAs' partial errors in a fixed order (for every alpha, lane k
// adds the partials k, k + 32, k + 64, ... in that order, then a fixed
// shuffle tree), the first minimum, and s_best.  Run by one CTA of kThreads
// threads after every partial is visible.  All loads of a batch are issued
// before any add, so the pass costs a few L2 round trips.
__device__ void finalize_cta(const double* partial, int n_parts, int n_grid,
                             const float* S, int64_t d_in, int dev_err, double* err,
                             int32_t* best_idx, float* s_best, double* e_s, int* best_s) {
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    constexpr int kWarps = kThreads / 32;
    constexpr int kA = (kMaxGrid + kWarps - 1) / kWarps;   // alphas per warp
    constexpr int kBatch = 8;                              // partials per lane per batch
    double sums[kA];
#pragma unroll
    for (int i = 0; i < kA; ++i) sums[i] = 0.0;
    for (int c0 = 0; c0 * 32 < n_parts; c0 += kBatch) {
        double v[kA][kBatch];
#pragma unroll
        for (int i = 0; i < kA; ++i) {
            const int a = warp + i * kWarps;
#pragma unroll
            for (int k = 0; k < kBatch; ++k) {
                const int c = lane + 32 * (c0 + k);
                v[i][k] = (a < n_grid && c < n_parts)
                              ? __ldcg(partial + (int64_t)c * n_grid + a) : 0.0;
            }
        }
#pragma unroll
        for (int i = 0; i < kA; ++i)
#pragma unroll
            for (int k = 0; k < kBatch; ++k)
                if (lane + 32 * (c0 + k) < n_parts) sums[i] += v[i][k];
    }
#pragma unroll
    for (int i = 0; i < kA; ++i) {
        const int a = warp + i * kWarps;
        double t = sums[i];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
        if (lane == 0 && a < n_grid) {
            e_s[a] = t;
            err[a] = t;
        }
    }
    __syncthreads();
    if (tid == 0) {
        int b = 0;
        bool finite = true;
        for (int i = 0; i < n_grid; ++i) {
            if (!isfinite(e_s[i])) finite = false;
            if (e_s[i] < e_s[b]) b = i;
        }
        if (!finite) {
            b = -1;
            raise_device_flag(AWQ_FLAG_NONFINITE_SCORE);
        }
        if (dev_err) {
            b = -2;
            raise_device_flag(AWQ_FLAG_WAIT_TIMEOUT);
        }
        *best_s = b;
        *best_idx = b;
    }
    __syncthreads();
    if (s_best) {
        // S rows and s_best are 16-byte aligned (d_in % 32 == 0)
        const int b = *best_s;
        const float4* src = reinterpret_cast<const float4*>(S + (int64_t)(b >= 0 ? b : 0) * d_in);
        float4* dst = reinterpret_cast<float4*>(s_best);
        const int64_t n4 = d_in / 4;
        const float nan = __int_as_float(0x7fc00000);
        for (int64_t j0 = tid; j0 < n4; j0 += 4 * kThreads) {
            float4 v[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int64_t j = j0 + (int64_t)k * kThreads;
                v[k] = (j < n4 && b >= 0) ? __ldcg(src + j) : make_float4(nan, nan, nan, nan);
            }
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int64_t j = j0 + (int64_t)k * kThreads;
                if (j < n4) dst[j] = v[k];
            }
        }
    }
}

// Pass 1 of one row: ws = w * s (exact fp32 products, packed fp32x2) and the
// lane's largest |ws|.
__device__ __forceinline__ float row_products(const float2* w, const float4* s4, float2* ws) {
    float mx[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        ws[2 * k] = __fmul2_rn(w[2 * k], f2(s4[k].x, s4[k].y));
        ws[2 * k + 1] = __fmul2_rn(w[2 * k + 1], f2(s4[k].z, s4[k].w));
        mx[k] = fmaxf(fmaxf(fabsf(ws[2 * k].x), fabsf(ws[2 * k].y)),
                      fmaxf(fabsf(ws[2 * k + 1].x), fabsf(ws[2 * k + 1].y)));
    }
    return fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
}

// q_scale of each of a lane's two rows from its largest |ws| (the lane-local
// maxima combined over the row's L lanes), its approximate reciprocal, and
// whether every |ws| / q_scale of the row is known to stay below 7.5 (then
// the code needs no clamp and the reciprocal is finite).  Non-finite ws need
// no flag here: they make the row's error non-finite on their own.  Even
// lanes finish row 0 and odd lanes row 1 (one exchange with the neighbour,
// then the butterfly over the row's remaining lanes), each lane computes one
// q_scale, and the pair shares the results; *in_range covers the row this
// lane computed, and every row of the warp is computed by some lane.
template <int L, bool kFp32>
__device__ __forceinline__ void rows_scale(float m0, float m1, int lane, float* qs0, float* rq0,
                                           float* qs1, float* rq1, bool* in_range) {
    const bool odd = (lane & 1) != 0;
    float m = fmaxf(odd ? m1 : m0, __shfl_xor_sync(0xffffffffu, odd ? m0 : m1, 1));
#pragma unroll
    for (int o = 2; o < L; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float q;
    if (kFp32) {
        q = div7_rn(m);
        *in_range = q >= kFloatMinNormal && q <= 3.402823466e38f;
    } else {
        const float h = __half2float(__float2half_rn(div7_rn_for_fp16(m)));
        *in_range = (h >= kHalfMinNormal) & (h <= kHalfMax);
        q = fminf(h, kHalfMax);
    }
    const float r = rcp_approx(q);
    const int even = lane & ~1;
    *qs0 = __shfl_sync(0xffffffffu, q, even);
    *qs1 = __shfl_sync(0xffffffffu, q, even | 1);
    *rq0 = __shfl_sync(0xffffffffu, r, even);
    *rq1 = __shfl_sync(0xffffffffu, r, even | 1);
}

// ---- asymmetric grid (16 levels, per-group zero point)
// Pass 1: ws = w * s and the lane's largest and smallest ws.
__device__ __forceinline__ float2 row_products_minmax(const float2* w, const float4* s4,
                                                      float2* ws) {
    float mx = __int_as_float(0xff800000), mn = __int_as_float(0x7f800000);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        ws[2 * k] = __fmul2_rn(w[2 * k], f2(s4[k].x, s4[k].y));
        ws[2 * k + 1] = __fmul2_rn(w[2 * k + 1], f2(s4[k].z, s4[k].w));
        mx = fmaxf(fmaxf(mx, fmaxf(ws[2 * k].x, ws[2 * k].y)),
                   fmaxf(ws[2 * k + 1].x, ws[2 * k + 1].y));
        mn = fminf(fminf(mn, fminf(ws[2 * k].x, ws[2 * k].y)),
                   fminf(ws[2 * k + 1].x, ws[2 * k + 1].y));
    }
    return f2(mx, mn);
}

// For each of a lane's two rows: the scale fp16(max(max - min, 1e-5) / 15)
// (exact quotient), the zero point clamp(rint(-min / q_scale), 0, 15) (exact
// quotient), the rounding constant 1.5*2^23 + zero and an approximate
// reciprocal for the codes, split between the lanes of each pair as in
// rows_scale.  *in_range: the codes of the row's smallest and largest ws,
// taken by the same FMA as the codes pass, lie in 0..15; that FMA is
// monotonic in ws, so then no code of the row needs the clamp.  A non-finite
// ws makes the row's error non-finite by itself: its residual is NaN with or
// without the clamp (an inf also makes in_range false; a NaN is skipped by
// the row's min and max).
template <int L, bool kFp32>
__device__ __forceinline__ void rows_scale_asym(float2 mm0, float2 mm1, int lane, float* qs0,
                                                float* rq0, float* mz0, float* qs1, float* rq1,
                                                float* mz1, bool* in_range) {
    const bool odd = (lane & 1) != 0;
    const float2 own = odd ? mm1 : mm0, other = odd ? mm0 : mm1;
    float mx = fmaxf(own.x, __shfl_xor_sync(0xffffffffu, other.x, 1));
    float mn = fminf(own.y, __shfl_xor_sync(0xffffffffu, other.y, 1));
#pragma unroll
    for (int o = 2; o < L; o <<= 1) {
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    }
    const float range = fmaxf(__fsub_rn(mx, mn), 1e-5f);
    float q = div15_rn(range);
    if (!kFp32) q = fminf(__half2float(__float2half_rn(q)), kHalfMax);
    const float z = fminf(fmaxf(rintf(div_rn_rcp(-mn, q, __frcp_rn(q))), 0.f), 15.f);
    const float r = rcp_approx(q);
    const float mz = kRoundMagic + z;
    *in_range = (__fmaf_rn(mn, r, mz) >= kRoundMagic) & (__fmaf_rn(mx, r, mz) <= kRoundMagic + 15.f);
    const int even = lane & ~1;
    *qs0 = __shfl_sync(0xffffffffu, q, even);
    *qs1 = __shfl_sync(0xffffffffu, q, even | 1);
    *rq0 = __shfl_sync(0xffffffffu, r, even);
    *rq1 = __shfl_sync(0xffffffffu, r, even | 1);
    *mz0 = __shfl_sync(0xffffffffu, mz, even);
    *mz1 = __shfl_sync(0xffffffffu, mz, even | 1);
}

// The error pass of one alpha fused with the products pass of the next one
// (software pipelining within the warp, in place): for every element pair
// the terms of this alpha are taken from ws (as in rows_errors), then ws is
// overwritten with w * s_next and the running row maxima |ws| (symmetric)
// or max / min (asymmetric) of the next alpha are updated.  The next
// alpha's group-scale chain (shuffles, division, reciprocal) therefore runs
// after a loop that mixes FMA-pipe and ALU work, instead of the ALU-only max
// tree and the FMA-only error loop running as separate phases in every
// warp at once.  kNext = false for the last alpha (no next products).
template <bool kClamp, bool kNext, int L>
__device__ __forceinline__ float2 rows_errors_next(float2* ws0, float2* ws1, const float2* w0,
                                                   const float2* w1, const float4* T2,
                                                   const float4* Sn, int l, float qs0, float rq0,
                                                   float qs1, float rq1, float* m0, float* m1) {
    if (kClamp && !(qs0 > 0.f)) rq0 = 0.f;
    if (kClamp && !(qs1 > 0.f)) rq1 = 0.f;
    const float2 nqs0 = f2(-qs0, -qs0), nqs1 = f2(-qs1, -qs1);
    const float2 rq02 = f2(rq0, rq0), rq12 = f2(rq1, rq1);
    const float2 magic2 = f2(kRoundMagic, kRoundMagic), nmagic2 = f2(-kRoundMagic, -kRoundMagic);
    float2 acc2[2] = {f2(0.f, 0.f), f2(0.f, 0.f)};
    float mx0[2] = {0.f, 0.f}, mx1[2] = {0.f, 0.f};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const float4 tv = T2[k * L + l];
        float4 sv;
        if (kNext) sv = Sn[k * L + l];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const int i = 2 * k + j;
            float2 t0 = __ffma2_rn(ws0[i], rq02, magic2);
            float2 t1 = __ffma2_rn(ws1[i], rq12, magic2);
            if (kClamp) {
                t0 = f2(fminf(fmaxf(t0.x, kRoundMagic - 7.f), kRoundMagic + 7.f),
                        fminf(fmaxf(t0.y, kRoundMagic - 7.f), kRoundMagic + 7.f));
                t1 = f2(fminf(fmaxf(t1.x, kRoundMagic - 7.f), kRoundMagic + 7.f),
                        fminf(fmaxf(t1.y, kRoundMagic - 7.f), kRoundMagic + 7.f));
            }
            const float2 q0 = __fadd2_rn(t0, nmagic2);
            const float2 q1 = __fadd2_rn(t1, nmagic2);
            const float2 d0 = __ffma2_rn(q0, nqs0, ws0[i]);
            const float2 d1 = __ffma2_rn(q1, nqs1, ws1[i]);
            float2 sq = __fmul2_rn(d0, d0);
            sq = __ffma2_rn(d1, d1, sq);
            acc2[j] = __ffma2_rn(j ? f2(tv.z, tv.w) : f2(tv.x, tv.y), sq, acc2[j]);
            if (kNext) {
                const float2 s2 = j ? f2(sv.z, sv.w) : f2(sv.x, sv.y);
                ws0[i] = __fmul2_rn(w0[i], s2);
                ws1[i] = __fmul2_rn(w1[i], s2);
                mx0[j] = fmaxf(mx0[j], fmaxf(fabsf(ws0[i].x), fabsf(ws0[i].y)));
                mx1[j] = fmaxf(mx1[j], fmaxf(fabsf(ws1[i].x), fabsf(ws1[i].y)));
            }
        }
    }
    if (kNext) {
        *m0 = fmaxf(mx0[0], mx0[1]);
        *m1 = fmaxf(mx1[0], mx1[1]);
    }
    return __fadd2_rn(acc2[0], acc2[1]);
}

// The asymmetric counterpart: rows_errors_asym for this alpha, then the
// next alpha's products and their running max and min per row.
template <bool kClamp, bool kNext, int L>
__device__ __forceinline__ float2 rows_errors_asym_next(float2* ws0, float2* ws1,
                                                        const float2* w0, const float2* w1,
                                                        const float4* T2, const float4* Sn,
                                                        int l, float qs0, float rq0, float mz0,
                                                        float qs1, float rq1, float mz1,
                                                        float2* mm0, float2* mm1) {
    const float2 nqs0 = f2(-qs0, -qs0), nqs1 = f2(-qs1, -qs1);
    const float2 rq02 = f2(rq0, rq0), mz02 = f2(mz0, mz0), nmz02 = f2(-mz0, -mz0);
    const float2 rq12 = f2(rq1, rq1), mz12 = f2(mz1, mz1), nmz12 = f2(-mz1, -mz1);
    constexpr float lo = kRoundMagic, hi = kRoundMagic + 15.f;
    float2 acc2[2] = {f2(0.f, 0.f), f2(0.f, 0.f)};
    float mx0 = __int_as_float(0xff800000), mn0 = __int_as_float(0x7f800000);
    float mx1 = mx0, mn1 = mn0;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const float4 tv = T2[k * L + l];
        float4 sv;
        if (kNext) sv = Sn[k * L + l];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const int i = 2 * k + j;
            float2 t0 = __ffma2_rn(ws0[i], rq02, mz02);
            float2 t1 = __ffma2_rn(ws1[i], rq12, mz12);
            if (kClamp) {
                t0 = f2(fminf(fmaxf(t0.x, lo), hi), fminf(fmaxf(t0.y, lo), hi));
                t1 = f2(fminf(fmaxf(t1.x, lo), hi), fminf(fmaxf(t1.y, lo), hi));
            }
            const float2 q0 = __fadd2_rn(t0, nmz02);
            const float2 q1 = __fadd2_rn(t1, nmz12);
            const float2 d0 = __ffma2_rn(q0, nqs0, ws0[i]);
            const float2 d1 = __ffma2_rn(q1, nqs1, ws1[i]);
            float2 sq = __fmul2_rn(d0, d0);
            sq = __ffma2_rn(d1, d1, sq);
            acc2[j] = __ffma2_rn(j ? f2(tv.z, tv.w) : f2(tv.x, tv.y), sq, acc2[j]);
            if (kNext) {
                const float2 s2 = j ? f2(sv.z, sv.w) : f2(sv.x, sv.y);
                ws0[i] = __fmul2_rn(w0[i], s2);
                ws1[i] = __fmul2_rn(w1[i], s2);
                mx0 = fmaxf(mx0, fmaxf(ws0[i].x, ws0[i].y));
                mn0 = fminf(mn0, fminf(ws0[i].x, ws0[i].y));
                mx1 = fmaxf(mx1, fmaxf(ws1[i].x, ws1[i].y));
                mn1 = fminf(mn1, fminf(ws1[i].x, ws1[i].y));
            }
        }
    }
    if (kNext) {
        *mm0 = f2(mx0, mn0);
        *mm1 = f2(mx1, mn1);
    }
    return __fadd2_rn(acc2[0], acc2[1]);
}

template <int L, bool kFp32, bool kAsym>
__global__ void __launch_bounds__(kThreads, 1)
search_kernel(const __grid_constant__ SearchParams p) {
    constexpr int G = 16 * L;                    // group size
    constexpr int RPW = 2 * 32 / L;              // rows per warp (two per lane)
    constexpr int R = kConsumerWarps * RPW;      // rows per unit
    static_assert(R * G * 2 == kUnitBytes, "unit size");

    extern __shared__ __align__(1024) unsigned char smem[];
    unsigned char* stage_base = smem;                                   // kStages * 16 KB
    float* tab = reinterpret_cast<float*>(smem + kStages * kUnitBytes); // (n_grid+1) * 2 * G
    double* wacc = reinterpret_cast<double*>(tab + (p.n_grid + 1) * 2 * G);  // n_grid * warps
    float* acc = reinterpret_cast<float*>(wacc + p.n_grid * kConsumerWarps);   // n_grid * kThreads
    uint64_t* full = reinterpret_cast<uint64_t*>(acc + p.n_grid * kThreads);
    uint64_t* empty = full + kStages;
    int* flags_s = reinterpret_cast<int*>(empty + kStages);   // [0] abort, [1] last, [2] best
    double* e_s = wacc;                                       // reused by the last CTA

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int row = warp * RPW + lane / L;        // first row within the unit
    const int l = lane % L;                       // sub-lane within the row
    // the lane's second row is row + 32 / L

    // contiguous, balanced range of units for this CTA
    const int64_t u0 = p.n_units * blockIdx.x / gridDim.x;
    const int64_t u1 = p.n_units * (blockIdx.x + 1) / gridDim.x;

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
        // the test hook: CTA 0's first load is armed for 16 bytes that never
        // come, so its phase never completes (the copy itself lands)
        const bool stall = (p.flags & AWQ_TEST_STALL_WAIT) && blockIdx.x == 0 && u == u0;
        mbar_arrive_expect_tx(&full[stage], kUnitBytes + (stall ? 16u : 0u));
        // R rows in boxes of at most kMaxBoxRows (R = 512 for g = 32)
#pragma unroll
        for (int b = 0; b * kMaxBoxRows < R; ++b)
            tma_load_2d(stage_base + stage * kUnitBytes + b * kMaxBoxRows * G * 2, &p.tmap[seg],
                        grp * G, rb * R + b * kMaxBoxRows, &full[stage]);
        ++issued[stage];
    };

    // prologue, overlapping the scale-table kernels: W does not depend on them
    if (tid == 0) {
        flags_s[0] = 0;
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kConsumerWarps);
        }
        mbar_fence_init();
        for (int k = 0; k < p.n_seg; ++k) tma_prefetch_desc(&p.tmap[k]);
        for (int s = 0; s < kStages && u0 + s < u1; ++s) issue(u0 + s, s);
    }
    for (int i = tid; i < p.n_grid * kThreads; i += kThreads) acc[i] = 0.f;
    for (int i = tid; i < p.n_grid * kConsumerWarps; i += kThreads) wacc[i] = 0.0;
    pdl_wait();          // the scale table (and the cleared counters) are ready
    __syncthreads();

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
            if (*(volatile int*)&flags_s[0] == 0 && mbar_wait_bounded(&empty[ps], pp)) {
                issue(u + 1, ps);
            } else {
                atomicOr(&p.dev_words[0], kDevErrWaitTimeout);
                *(volatile int*)&flags_s[0] = 1;
                failed = true;
            }
        }

        int seg, grp, rb;
        decode(u, &seg, &grp, &rb);
        if (grp != cur_grp) {   // uniform: every thread walks the same units
            __syncthreads();
            // The group's S and tau2 columns, 16 bytes at a time (rows are
            // 16-byte aligned: d_in % 32 == 0; table_slot keeps each run of
            // four channels together), every load issued before any store.
            constexpr int kC4 = G / 4;                                   // float4 per row
            constexpr int kPer = (kMaxGrid * kC4 + kThreads - 1) / kThreads;
            const float4* Sg = reinterpret_cast<const float4*>(p.S + (int64_t)grp * G);
            const float4* Tg = reinterpret_cast<const float4*>(p.tau2 + (int64_t)grp * G);
            const int64_t ld4 = p.d_in / 4;
            const int n4 = p.n_grid * kC4;
            float4 sv[kPer], tv[kPer];
#pragma unroll
            for (int k = 0; k < kPer; ++k) {
                const int i = tid + k * kThreads;
                if (i < n4) {
                    sv[k] = __ldcg(Sg + (int64_t)(i / kC4) * ld4 + i % kC4);
                    tv[k] = __ldcg(Tg + (int64_t)(i / kC4) * ld4 + i % kC4);
                }
            }
#pragma unroll
            for (int k = 0; k < kPer; ++k) {
                const int i = tid + k * kThreads;
                if (i < n4) {
                    const int a = i / kC4, slot = table_slot<L>(4 * (i % kC4));
                    *reinterpret_cast<float4*>(&tab[a * 2 * G + slot]) = sv[k];
                    *reinterpret_cast<float4*>(&tab[a * 2 * G + G + slot]) = tv[k];
                }
            }
            for (int i = tid; i < 2 * G; i += kThreads) tab[p.n_grid * 2 * G + i] = 0.f;
            cur_grp = grp;
            __syncthreads();
        }

        bool ok = !failed && *(volatile int*)&flags_s[0] == 0;
        if (ok) ok = mbar_wait_bounded(&full[stage], parity);
        if (!failed && !ok && lane == 0) {
            atomicOr(&p.dev_words[0], kDevErrWaitTimeout);
            *(volatile int*)&flags_s[0] = 1;
        }
        failed = __any_sync(0xffffffffu, !ok) || failed;
        if (failed) {
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[stage]);
            continue;
        }
        // this lane's weights: chunks l and l + L (8 channels each) of its two rows
        float2 w[2][kElemsPerRow / 2];
        {
#pragma unroll
            for (int rr = 0; rr < 2; ++rr) {
                const uint4* src = reinterpret_cast<const uint4*>(
                    stage_base + stage * kUnitBytes + (row + rr * (32 / L)) * G * 2);
#pragma unroll
                for (int k2 = 0; k2 < 2; ++k2) {
                    const uint4 v = src[l + L * k2];
                    const uint32_t hw[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        w[rr][k2 * 4 + i] =
                            __half22float2(*reinterpret_cast<const __half2*>(&hw[i]));
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[stage]);

        // alpha 0's products and row extremes; then each alpha's group-scale
        // chain, and its error pass fused with the next alpha's products
        float2 ws[2][kElemsPerRow / 2];
        {
            const float4* S0 = reinterpret_cast<const float4*>(tab);
            float4 s4[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) s4[k] = S0[k * L + l];
            if (kAsym) {
                float2 mm0 = row_products_minmax(w[0], s4, ws[0]);
                float2 mm1 = row_products_minmax(w[1], s4, ws[1]);
                for (int a = 0; a < p.n_grid; ++a) {
                    const float4* Ta = reinterpret_cast<const float4*>(tab + a * 2 * G + G);
                    const float4* Sn = reinterpret_cast<const float4*>(tab + (a + 1) * 2 * G);
                    float qs0, rq0, mz0, qs1, rq1, mz1;
                    bool in;
                    rows_scale_asym<L, kFp32>(mm0, mm1, lane, &qs0, &rq0, &mz0, &qs1, &rq1,
                                              &mz1, &in);
                    const bool all_in = __all_sync(0xffffffffu, in);
                    float2 e;
                    if (a + 1 < p.n_grid) {
                        e = all_in ? rows_errors_asym_next<false, true, L>(
                                         ws[0], ws[1], w[0], w[1], Ta, Sn, l, qs0, rq0, mz0,
                                         qs1, rq1, mz1, &mm0, &mm1)
                                   : rows_errors_asym_next<true, true, L>(
                                         ws[0], ws[1], w[0], w[1], Ta, Sn, l, qs0, rq0, mz0,
                                         qs1, rq1, mz1, &mm0, &mm1);
                    } else {
                        e = all_in ? rows_errors_asym_next<false, false, L>(
                                         ws[0], ws[1], w[0], w[1], Ta, Sn, l, qs0, rq0, mz0,
                                         qs1, rq1, mz1, &mm0, &mm1)
                                   : rows_errors_asym_next<true, false, L>(
                                         ws[0], ws[1], w[0], w[1], Ta, Sn, l, qs0, rq0, mz0,
                                         qs1, rq1, mz1, &mm0, &mm1);
                    }
                    acc[a * kThreads + tid] += e.x + e.y;
                }
            } else {
                float m0 = row_products(w[0], s4, ws[0]);
                float m1 = row_products(w[1], s4, ws[1]);
                for (int a = 0; a < p.n_grid; ++a) {
                    const float4* Ta = reinterpret_cast<const float4*>(tab + a * 2 * G + G);
                    const float4* Sn = reinterpret_cast<const float4*>(tab + (a + 1) * 2 * G);
                    float qs0, rq0, qs1, rq1;
                    bool in;
                    rows_scale<L, kFp32>(m0, m1, lane, &qs0, &rq0, &qs1, &rq1, &in);
                    const bool all_in = __all_sync(0xffffffffu, in);
                    float2 e;
                    // some row has an fp16-subnormal, overflowing, zero or NaN
                    // scale: the clamping variant
                    if (a + 1 < p.n_grid) {
                        e = all_in ? rows_errors_next<false, true, L>(ws[0], ws[1], w[0], w[1],
                                                                      Ta, Sn, l, qs0, rq0, qs1,
                                                                      rq1, &m0, &m1)
                                   : rows_errors_next<true, true, L>(ws[0], ws[1], w[0], w[1],
                                                                     Ta, Sn, l, qs0, rq0, qs1,
                                                                     rq1, &m0, &m1);
                    } else {
                        e = all_in ? rows_errors_next<false, false, L>(ws[0], ws[1], w[0], w[1],
                                                                       Ta, Sn, l, qs0, rq0, qs1,
                                                                       rq1, &m0, &m1)
                                   : rows_errors_next<true, false, L>(ws[0], ws[1], w[0], w[1],
                                                                      Ta, Sn, l, qs0, rq0, qs1,
                                                                      rq1, &m0, &m1);
                    }
                    acc[a * kThreads + tid] += e.x + e.y;
                }
            }
        }
        // every 8 units the per-thread fp32 partials move into the warp's fp64
        // accumulators (fixed order), bounding fp32 accumulation to 8 units
        if (((it + 1) & 7) == 0 || u + 1 == u1) {
            for (int a = 0; a < p.n_grid; ++a) {
                double v = (double)acc[a * kThreads + tid];
                acc[a * kThreads + tid] = 0.f;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
                if (lane == 0) wacc[a * kConsumerWarps + warp] += v;
            }
        }
    }

    // the next kernel (e.g. the pack, which waits for this grid to finish)
    // may start launching while the partials are reduced
    pdl_launch_dependents();

    // drain: never leave the CTA while a TMA copy may still write its smem.
    // The n-th load into a stage completes that barrier's phase n.  On the
    // normal path every load was consumed and these waits return at once; a
    // drain that gives up (kDrainLimitNs) marks the result invalid.
    if (tid == 0) {
        for (int s = 0; s < kStages; ++s)
            if (issued[s] > 0 && !mbar_wait_drain(&full[s], (uint32_t)(issued[s] - 1) & 1u))
                atomicOr(&p.dev_words[0], kDevErrWaitTimeout);
    }
    __syncthreads();

    // fixed-order reduction of the per-warp partials
    if (tid < p.n_grid) {
        double v = 0.0;
        for (int w8 = 0; w8 < kConsumerWarps; ++w8) v += wacc[tid * kConsumerWarps + w8];
        p.partial[(int64_t)blockIdx.x * p.n_grid + tid] = v;
    }

    // the last CTA to arrive reduces every partial
    __threadfence();
    __syncthreads();
    if (tid == 0) {
        const int done = atomicAdd(&p.dev_words[1], 1);
        flags_s[1] = (done == (int)gridDim.x - 1);
    }
    __syncthreads();
    if (flags_s[1]) {
        __threadfence();
        finalize_cta(p.partial, gridDim.x, p.n_grid, p.S, p.d_in,
                     *(volatile int*)&p.dev_words[0], p.err, p.best_idx, p.s_best, e_s,
                     &flags_s[2]);
    }
}

// ---- scale table: s_i[j] = max(x_j, 1e-4)^alpha_i / sqrt(max_j * min_j)

__device__ __forceinline__ double table_pow(float xj, double alpha) {
    return pow((double)fmaxf(xj, 1e-4f), alpha);
}

// Every CTA reduces max_j and min_j of max(x_j, 1e-4) over all channels (x
// is at most a few tens of KB and stays in L2): pow(., alpha) is monotonic
// for alpha >= 0 and its fp64 error is far below the spacing of pow at
// distinct fp32 arguments, so pow(x_max, alpha) and pow(x_min, alpha) are
// exactly the largest and smallest entries of the row.  The CTA then writes
// its slice of channels for its alpha.
__global__ void __launch_bounds__(256)
table_kernel(const float* __restrict__ x, int64_t d_in, int n_grid, int64_t slice,
             float* __restrict__ S, float* __restrict__ T, int kind,
             int* __restrict__ dev_words) {
    __shared__ float red_mx[8], red_mn[8];
    // Wait for the kernel before (x may come from it) before letting the
    // search kernel launch: the search reads W before its own wait, so W
    // must already be final when it starts.
    pdl_wait();
    pdl_launch_dependents();
    const int a = blockIdx.y;
    const int sl = blockIdx.x;
    if (dev_words && a == 0 && sl == 0 && threadIdx.x == 0) {
        dev_words[0] = 0;
        dev_words[1] = 0;
    }
    // The thread's first channel: its pow does not depend on the reduction
    // below, so it is taken first and its latency overlaps the reduction's.
    const double alpha = __ddiv_rn((double)a, (double)n_grid);
    const int64_t j0 = (int64_t)sl * slice, j1 = min(d_in, j0 + slice);
    const int64_t jf = j0 + threadIdx.x;
    float xf = 1.f;
    double pf = 1.0;
    if (jf < j1) {
        xf = x[jf];
        pf = table_pow(xf, alpha);
    }
    // x is 16-byte aligned and d_in % 32 == 0: 16-byte loads, eight in
    // flight per thread (max and min are order-independent)
    float mx = 0.f, mn = __int_as_float(0x7f800000);
    const float4* x4 = reinterpret_cast<const float4*>(x);
    const int64_t n4 = d_in / 4;
    for (int64_t j0 = threadIdx.x; j0 < n4; j0 += 8 * (int64_t)blockDim.x) {
        float4 v[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const int64_t j = j0 + (int64_t)k * blockDim.x;
            v[k] = j < n4 ? __ldg(x4 + j) : make_float4(1.f, 1.f, 1.f, 1.f);
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            if (j0 + (int64_t)k * blockDim.x < n4) {
                const float a = fmaxf(v[k].x, 1e-4f), b = fmaxf(v[k].y, 1e-4f);
                const float c = fmaxf(v[k].z, 1e-4f), d = fmaxf(v[k].w, 1e-4f);
                mx = fmaxf(mx, fmaxf(fmaxf(a, b), fmaxf(c, d)));
                mn = fminf(mn, fminf(fminf(a, b), fminf(c, d)));
            }
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    }
    if ((threadIdx.x & 31) == 0) {
        red_mx[threadIdx.x >> 5] = mx;
        red_mn[threadIdx.x >> 5] = mn;
    }
    __syncthreads();
    for (int k = 0; k < (int)(blockDim.x >> 5); ++k) {
        mx = fmaxf(mx, red_mx[k]);
        mn = fminf(mn, red_mn[k]);
    }
    const double norm = __dsqrt_rn(__dmul_rn(table_pow(mx, alpha), table_pow(mn, alpha)));
    for (int64_t j = jf; j < j1; j += blockDim.x) {
        const float xj = j == jf ? xf : x[j];
        const double pj = j == jf ? pf : table_pow(xj, alpha);
        const float s = __double2float_rn(__ddiv_rn(pj, norm));
        S[(int64_t)a * d_in + j] = s;
        float t;
        if (kind == kTableInverse) {
            t = __frcp_rn(s);
        } else {
            const double q = __ddiv_rn((double)xj, (double)s);
            t = __double2float_rn(q * q);
        }
        T[(int64_t)a * d_in + j] = t;
    }
}

__global__ void __launch_bounds__(kThreads)
finalize_kernel(const double* __restrict__ partial, int n_parts, int n_grid,
                const float* __restrict__ S, int64_t d_in, const int* __restrict__ dev_err,
                double* __restrict__ err, int32_t* __restrict__ best_idx,
                float* __restrict__ s_best) {
    __shared__ double e_s[kMaxGrid];
    __shared__ int best_s;
    pdl_wait();
    finalize_cta(partial, n_parts, n_grid, S, d_in, dev_err ? *dev_err : 0, err, best_idx,
                 s_best, e_s, &best_s);
}

struct SearchWs {
    float* S;
    float* tau2;
    double* partial;
    int* dev_words;
};

size_t max_search_ctas() { return kMaxParts; }

SearchWs carve_search_ws(void* ws, int64_t d_in, int n_grid) {
    char* p = static_cast<char*>(ws);
    SearchWs w;
    const size_t tab = align_up((size_t)n_grid * (size_t)d_in * sizeof(float), kWsAlign);
    w.S = reinterpret_cast<float*>(p);
    w.tau2 = reinterpret_cast<float*>(p + tab);
    w.partial = reinterpret_cast<double*>(p + 2 * tab);
    w.dev_words = reinterpret_cast<int*>(
        p + 2 * tab + align_up(max_search_ctas() * kMaxGrid * sizeof(double), kWsAlign));
    return w;
}

size_t search_smem_bytes(int group_size, int n_grid) {
    return (size_t)kStages * kUnitBytes + (size_t)(n_grid + 1) * 2 * group_size * sizeof(float) +
           (size_t)n_grid * kConsumerWarps * sizeof(double) +
           (size_t)n_grid * kThreads * sizeof(float) + 2 * kStages * sizeof(uint64_t) + 16;
}

template <int L, bool kFp32, bool kAsym>
cudaError_t launch_search_L(const SearchParams& p, int grid, size_t smem, cudaStream_t st) {
    static int configured_smem[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64 || configured_smem[dev] < (int)smem) {
        cudaError_t e = cudaFuncSetAttribute(search_kernel<L, kFp32, kAsym>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) configured_smem[dev] = (int)smem;
    }
    return launch_pdl(search_kernel<L, kFp32, kAsym>, dim3(grid), dim3(kThreads), smem, st, p);
}

template <bool kFp32, bool kAsym>
cudaError_t launch_search(int L, const SearchParams& p, int grid, size_t smem,
                          cudaStream_t st) {
    switch (L) {
        case 2: return launch_search_L<2, kFp32, kAsym>(p, grid, smem, st);
        case 4: return launch_search_L<4, kFp32, kAsym>(p, grid, smem, st);
        case 8: return launch_search_L<8, kFp32, kAsym>(p, grid, smem, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t search_unit_flags(unsigned int* bits, bool clear) {
    return unit_device_flags(bits, clear);
}

size_t scale_search_workspace(int64_t d_in, int group_size, int n_grid) {
    (void)group_size;
    const size_t tab = align_up((size_t)n_grid * (size_t)d_in * sizeof(float), kWsAlign);
    return 2 * tab + align_up(max_search_ctas() * kMaxGrid * sizeof(double), kWsAlign) +
           kWsAlign;
}

cudaError_t launch_scale_table(const float* x_mean, int64_t d_in, int n_grid, float* S,
                               float* T, int* dev_words, int num_sms, cudaStream_t stream,
                               TableKind kind) {
    (void)num_sms;
    // one channel per thread where d_in allows (every CTA also reads all of x
    // for the row's max and min, so the slice count stays bounded)
    int64_t slices = std::max<int64_t>(1, std::min<int64_t>((d_in + 255) / 256, kMaxTableSlices));
    const int64_t slice = (d_in + slices - 1) / slices;
    slices = (d_in + slice - 1) / slice;
    const dim3 grid((unsigned)slices, (unsigned)n_grid);
    return launch_pdl(table_kernel, grid, dim3(256), 0, stream, x_mean, d_in, n_grid, slice, S,
                      T, (int)kind, dev_words);
}

cudaError_t launch_finalize(const double* partial, int n_parts, int n_grid, const float* S,
                            int64_t d_in, const int* dev_err, double* err,
                            int32_t* best_idx, float* s_best, cudaStream_t stream) {
    return launch_pdl(finalize_kernel, dim3(1), dim3(kThreads), 0, stream, partial, n_parts,
                      n_grid, S, d_in, dev_err, err, best_idx, s_best);
}

awq_status launch_scale_search(int n_seg, const void* const* W, const int64_t* d_out,
                               int64_t d_in, const float* x_mean, int group_size,
                               int n_grid, int flags, double* err, int32_t* best_idx,
                               float* s_best, void* ws, cudaStream_t stream) {
    DeviceInfo dev;
    if (query_device(&dev) != cudaSuccess) return AWQ_ERR_CUDA;
    EncodeTiledFn encode = encode_tiled_fn();
    if (!encode) return AWQ_ERR_CUDA;

    const int L = group_size / 16;
    const int R = kConsumerWarps * 2 * 32 / L;
    SearchWs w = carve_search_ws(ws, d_in, n_grid);

    SearchParams p;
    std::memset(&p, 0, sizeof(p));
    p.n_seg = n_seg;
    p.group_size = group_size;
    p.n_grid = n_grid;
    p.flags = flags;
    p.d_in = d_in;
    p.S = w.S;
    p.tau2 = w.tau2;
    p.partial = w.partial;
    p.dev_words = w.dev_words;
    p.err = err;
    p.best_idx = best_idx;
    p.s_best = s_best;
    const int64_t G = d_in / group_size;
    int64_t units = 0;
    for (int k = 0; k < n_seg; ++k) {
        const cuuint64_t gdim[2] = {(cuuint64_t)d_in, (cuuint64_t)d_out[k]};
        const cuuint64_t gstride[1] = {(cuuint64_t)d_in * 2};
        const cuuint32_t box[2] = {(cuuint32_t)group_size,
                                   (cuuint32_t)std::min(R, kMaxBoxRows)};
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
    int per_sm = 1;
    while (per_sm > 1 && (size_t)per_sm * (smem + 1024) > dev.max_smem_per_sm) --per_sm;
    int64_t grid = (int64_t)dev.num_sms * per_sm;
    if (grid > units) grid = units;
    if (grid > (int64_t)max_search_ctas()) grid = (int64_t)max_search_ctas();

    cudaError_t te;
    if (flags & AWQ_DUO_SCALING) {
        char* duo_ws = static_cast<char*>(ws) + scale_search_workspace(d_in, group_size, n_grid);
        te = launch_duo_table(n_seg, W, d_out, d_in, x_mean, n_grid, w.S, w.tau2, w.dev_words,
                              duo_ws, dev.num_sms, stream);
    } else {
        te = launch_scale_table(x_mean, d_in, n_grid, w.S, w.tau2, w.dev_words, dev.num_sms,
                                stream, kTableTauSq);
    }
    if (note_cuda(te, "scale table launch") != cudaSuccess) return AWQ_ERR_CUDA;
    const bool fp32 = (flags & AWQ_SCALE_FP32) != 0, asym = (flags & AWQ_ASYMMETRIC) != 0;
    const cudaError_t e =
        fp32 ? (asym ? launch_search<true, true>(L, p, (int)grid, smem, stream)
                     : launch_search<true, false>(L, p, (int)grid, smem, stream))
             : (asym ? launch_search<false, true>(L, p, (int)grid, smem, stream)
                     : launch_search<false, false>(L, p, (int)grid, smem, stream));
    if (e != cudaSuccess) return AWQ_ERR_CUDA;
    return AWQ_OK;
}

}  // namespace awq
