// clip_output.cu -- output-space clip search at a fixed scale s
// ("AWQ architecture, in depth", section "The pipeline end to end", step 5:
// an optional search of a clipping range that shrinks the quantisation
// range; section "The scale search as code": candidates are scored on the
// output).  For every row r, group k and ratio index i < n_clip, with
// c_i = RN((20 - i) / 20) and the clipped fake quantisation of awq_clip_search
// (q_scale = fp16(fl32(fl32(c_i max|ws|) / 7)), codes saturating at +-7):
//
//   e[r,k,i] = sum_t ( sum_{j in k} X[t,j] (W[r,j] - W_hat_i[r,j]) )^2
//            = v^T H_k v,   v = W[r,k] - W_hat_i[r,k],   H_k = X_k^T X_k,
//
// the group's share of the output error; clip_idx[r,k] = the first i with
// the smallest e, err[0] / err[1] the totals without clipping / with the
// chosen ratios.
//
//   gram_kernel         partial H_k for every group over up to 4 token slices,
//                       in fp64 (fp16 products are exact in fp64); X staged
//                       two halves per thread and step, so a warp's shared-
//                       memory stores are one contiguous run, and each lane
//                       reads tile columns tx + (tile width / 4) r
//                       (consecutive lanes, consecutive doubles); one
//                       CTA per (group, tile of H on or above the diagonal,
//                       slice), so the grid covers the SMs even for 32
//                       groups.  HBM: X read once per tile row of H.  2 T g
//                       d_in flop (3/4 of it at g = 128: H_k is symmetric).
//   gram_reduce_kernel  H_k = fp32(sum of the slices in order): deterministic.
//   clip_output_kernel  one CTA per (group, 64 rows): H_k staged in shared
//                       memory; warp w takes 8 rows; per ratio each lane forms
//                       its g/32 entries of every row's v exactly (the IEEE
//                       quotient decides the codes, as awq_quantize_pack), then
//                       H v for its entries against the 8 rows at once (H read
//                       once per 8 rows) and e = v . H v by a warp sum.
//                       2 g^2 flop per (row, group, ratio).  Fixed task order
//                       and a last-CTA sum of the per-CTA partials in a fixed
//                       order: deterministic.
#include <algorithm>
#include <cstring>

#include "common.cuh"
#include "internal.h"

namespace awq {
namespace {

constexpr int kCoWarps = 8;
constexpr int kCoThreads = kCoWarps * 32;
constexpr int kCoRowsPerWarp = 8;
constexpr int kCoRows = kCoWarps * kCoRowsPerWarp;     // 64 rows per CTA
constexpr int kClipDen = 20;
constexpr int kMaxCoCtas = 1 << 20;

// ---------------------------------------------------------------- Gram
// Partial H_k[a][b] = sum_t X[t, k g + a] X[t, k g + b] over one slice of the
// tokens (blockIdx.y; slices of t_per tokens) for a 64 x 64 (g >= 64) or
// 32 x 32 tile of H_k; each thread accumulates a 4 x 4 block in fp64, tokens
// in order, and writes it unrounded.  X arrives in 16-byte loads (8 halves).
constexpr int kMaxGramSlices = 4;
template <int TILE>
__global__ void __launch_bounds__((TILE / 4) * (TILE / 4))
gram_kernel(const __half* __restrict__ X, int64_t T, int64_t ld, int g, int64_t t_per,
            double* __restrict__ Hpart) {
    constexpr int kT = 32;                      // tokens per staged chunk
    constexpr int kN = (TILE / 4) * (TILE / 4);
    __shared__ __align__(16) double sa[kT][TILE];   // 16-byte pairs are stored into it
    __shared__ __align__(16) double sb[kT][TILE];
    pdl_wait();
    // H_k is symmetric: only tiles ti <= tj are computed (tiles (tiles + 1) / 2
    // per group), an off-diagonal one also written transposed
    const int tiles = g / TILE;
    const int pairs = tiles * (tiles + 1) / 2;
    const int k = blockIdx.x / pairs;
    int ti = 0, tj = blockIdx.x % pairs;
    while (tj >= tiles - ti) {
        tj -= tiles - ti;
        ++ti;
    }
    tj += ti;
    const int64_t ca = (int64_t)k * g + ti * TILE, cb = (int64_t)k * g + tj * TILE;
    const int tx = threadIdx.x % (TILE / 4), ty = threadIdx.x / (TILE / 4);
    const int64_t t_begin = (int64_t)blockIdx.y * t_per;
    const int64_t t_end = min(T, t_begin + t_per);
    double acc[4][4] = {};
    for (int64_t t0 = t_begin; t0 < t_end; t0 += kT) {
        // one half2 per thread and step: a warp stores one contiguous run of
        // 16-byte pairs (no bank conflicts)
        for (int e = threadIdx.x; e < kT * (TILE / 2); e += kN) {
            const int tt = e / (TILE / 2), c2 = e % (TILE / 2);
            const bool in = t0 + tt < t_end;
            const uint32_t ha = in ? __ldg(reinterpret_cast<const unsigned int*>(
                                             X + (t0 + tt) * ld + ca) + c2)
                                   : 0u;
            const uint32_t hb = in ? __ldg(reinterpret_cast<const unsigned int*>(
                                             X + (t0 + tt) * ld + cb) + c2)
                                   : 0u;
            const float2 fa = __half22float2(*reinterpret_cast<const __half2*>(&ha));
            const float2 fb = __half22float2(*reinterpret_cast<const __half2*>(&hb));
            *reinterpret_cast<double2*>(&sa[tt][2 * c2]) = make_double2(fa.x, fa.y);
            *reinterpret_cast<double2*>(&sb[tt][2 * c2]) = make_double2(fb.x, fb.y);
        }
        __syncthreads();
#pragma unroll 4
        for (int tt = 0; tt < kT; ++tt) {
            // rows 4 ty + q (two per warp: broadcasts) against columns
            // tx + (TILE / 4) r (consecutive lanes, consecutive doubles)
            double a[4], b[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                a[q] = sa[tt][4 * ty + q];
                b[q] = sb[tt][tx + (TILE / 4) * q];
            }
#pragma unroll
            for (int q = 0; q < 4; ++q)
#pragma unroll
                for (int r = 0; r < 4; ++r) acc[q][r] = __fma_rn(a[q], b[r], acc[q][r]);
        }
        __syncthreads();
    }
    pdl_launch_dependents();
    // slice blockIdx.y of [slices][G][g][g]; gridDim.x / pairs = G
    double* Hk = Hpart + ((int64_t)blockIdx.y * (gridDim.x / pairs) + k) * g * g;
#pragma unroll
    for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const int a_ = ti * TILE + 4 * ty + q, b_ = tj * TILE + tx + (TILE / 4) * r;
            Hk[(int64_t)a_ * g + b_] = acc[q][r];
            if (ti != tj) Hk[(int64_t)b_ * g + a_] = acc[q][r];
        }
}

// H = fp32(sum of the slices' partials, slices in order): deterministic.
__global__ void __launch_bounds__(256)
gram_reduce_kernel(const double* __restrict__ Hpart, int slices, int64_t n,
                   float* __restrict__ H) {
    pdl_wait();
    pdl_launch_dependents();
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x) {
        double v = Hpart[i];
        for (int s = 1; s < slices; ++s) v += Hpart[(int64_t)s * n + i];
        H[i] = __double2float_rn(v);
    }
}

// ---------------------------------------------------------- clip scoring
struct CoParams {
    const __half* W;       // fp16 [d_out, d_in]
    int64_t d_out, d_in;
    const float* s;        // [d_in] or NULL
    const float* H;        // [G][g][g] fp32
    int n_clip;
    int fp32_scale;
    uint8_t* idx;          // [d_out, G]
    double* partial;       // [gridDim.x * gridDim.y][2]
    int* counter;
    double* err;           // [2]
};

// kE = g / 32 entries of a group per lane (lane l holds entries kE*l ..).
// Two CTAs per SM (128 registers; for g = 128 a few values spill): 1.86 ->
// 1.76 ms on q_proj against one CTA of 207 registers, which left 8 warps per
// SM to hide the shared-memory and FMA latencies.
template <int kE>
__global__ void __launch_bounds__(kCoThreads, 2)
clip_output_kernel(const CoParams p) {
    constexpr int G = 32 * kE;
    extern __shared__ __align__(16) float co_smem[];
    float* Hs = co_smem;                                    // [G][G]
    float* vbuf = Hs + G * G;                               // [warps][8][G]
    __shared__ double red[kCoWarps][2];
    __shared__ int last;

    pdl_wait();   // H (and W, s) may come from the kernels before
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int k = blockIdx.x;                               // group
    const int64_t groups = p.d_in / G;
    const int64_t rbase = (int64_t)blockIdx.y * kCoRows + warp * kCoRowsPerWarp;
    {   // stage H_k (symmetric: row j holds H[j][i] for all i)
        const float4* src = reinterpret_cast<const float4*>(p.H + (int64_t)k * G * G);
        float4* dst = reinterpret_cast<float4*>(Hs);
        for (int i = tid; i < G * G / 4; i += kCoThreads) dst[i] = __ldg(src + i);
    }
    // this lane's s entries and their fp64 reciprocals
    float sv[kE];
    double isd[kE];
#pragma unroll
    for (int e = 0; e < kE; ++e) {
        sv[e] = p.s ? __ldg(p.s + (int64_t)k * G + kE * lane + e) : 1.0f;
        isd[e] = __drcp_rn((double)sv[e]);
    }
    __syncthreads();

    // the rows' weights and the group maxima of |w s| (exact fp32 products)
    float wv[kCoRowsPerWarp][kE];
    float mrow[kCoRowsPerWarp];
    bool bad[kCoRowsPerWarp];
#pragma unroll
    for (int rr = 0; rr < kCoRowsPerWarp; ++rr) {
        const int64_t r = rbase + rr;
        float m = 0.f;
        bool nf = false;
#pragma unroll
        for (int e = 0; e < kE; ++e) {
            wv[rr][e] = r < p.d_out
                            ? __half2float(p.W[r * p.d_in + (int64_t)k * G + kE * lane + e])
                            : 0.f;
            const float ws = __fmul_rn(wv[rr][e], sv[e]);
            nf |= !(fabsf(ws) <= 3.402823466e38f);
            m = fmaxf(m, fabsf(ws));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
            nf |= __shfl_xor_sync(0xffffffffu, (int)nf, o) != 0;
        }
        mrow[rr] = m;
        bad[rr] = nf;
    }

    float* vb = vbuf + warp * kCoRowsPerWarp * G;
    double e0[kCoRowsPerWarp], best[kCoRowsPerWarp];
    int bi[kCoRowsPerWarp];
    for (int i = 0; i < p.n_clip; ++i) {
        const float c = __fdiv_rn((float)(kClipDen - i), (float)kClipDen);
        // v = w - q q_scale / s for every row of the warp (codes from the
        // IEEE quotient of fl32(w s); v in fp64, rounded once), into shared memory
#pragma unroll
        for (int rr = 0; rr < kCoRowsPerWarp; ++rr) {
            bool in_range;
            const float qs = group_scale(__fmul_rn(c, mrow[rr]), p.fp32_scale != 0, &in_range);
            const float rq = (qs > 0.f) ? __frcp_rn(qs) : 0.f;
#pragma unroll
            for (int e = 0; e < kE; ++e) {
                const float a = __fmul_rn(wv[rr][e], sv[e]);
                const float y = (qs > 0.f) ? div_rn_rcp(a, qs, rq) : 0.f;
                float t = __fadd_rn(y, kRoundMagic);
                t = fminf(fmaxf(t, kRoundMagic - 7.f), kRoundMagic + 7.f);
                const double qq = (double)__fadd_rn(t, -kRoundMagic) * (double)qs;
                vb[rr * G + kE * lane + e] =
                    __double2float_rn(__fma_rn(-qq, isd[e], (double)wv[rr][e]));
            }
        }
        __syncwarp();
        // (H v)[a] for this lane's entries a = kE*lane + e, all rows at once:
        // v read four j at a time (one 16-byte broadcast per row), the lane's
        // entries in pairs (packed fp32x2 FMAs); every entry still adds its
        // terms in j order, one rounding each, as the scalar loop would
        float hv[kCoRowsPerWarp][kE];
#pragma unroll
        for (int rr = 0; rr < kCoRowsPerWarp; ++rr)
#pragma unroll
            for (int e = 0; e < kE; ++e) hv[rr][e] = 0.f;
#pragma unroll 2
        for (int j0 = 0; j0 < G; j0 += 4) {
            float h[4][kE];
#pragma unroll
            for (int q = 0; q < 4; ++q)
#pragma unroll
                for (int e = 0; e < kE; ++e) h[q][e] = Hs[(j0 + q) * G + kE * lane + e];
#pragma unroll
            for (int rr = 0; rr < kCoRowsPerWarp; ++rr) {
                const float4 v4 = *reinterpret_cast<const float4*>(&vb[rr * G + j0]);
                const float vq[4] = {v4.x, v4.y, v4.z, v4.w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    if constexpr (kE >= 2) {
#pragma unroll
                        for (int e = 0; e < kE; e += 2) {
                            const float2 r2 = __ffma2_rn(make_float2(h[q][e], h[q][e + 1]),
                                                         make_float2(vq[q], vq[q]),
                                                         make_float2(hv[rr][e], hv[rr][e + 1]));
                            hv[rr][e] = r2.x;
                            hv[rr][e + 1] = r2.y;
                        }
                    } else {
                        hv[rr][0] = __fmaf_rn(h[q][0], vq[q], hv[rr][0]);
                    }
                }
            }
        }
#pragma unroll
        for (int rr = 0; rr < kCoRowsPerWarp; ++rr) {
            float part = 0.f;
#pragma unroll
            for (int e = 0; e < kE; ++e) part = __fmaf_rn(vb[rr * G + kE * lane + e], hv[rr][e], part);
            double d = (double)part;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
            if (i == 0) {
                e0[rr] = d;
                best[rr] = d;
                bi[rr] = 0;
            } else if (d < best[rr]) {
                best[rr] = d;
                bi[rr] = i;
            }
        }
        __syncwarp();   // every lane has read vb before the next ratio rewrites it
    }

    // store the indices; the warp's totals
    double t0 = 0.0, t1 = 0.0;
#pragma unroll
    for (int rr = 0; rr < kCoRowsPerWarp; ++rr) {
        const int64_t r = rbase + rr;
        if (r < p.d_out) {
            if (lane == 0) p.idx[r * groups + k] = (uint8_t)(bad[rr] ? 0 : bi[rr]);
            const double nan = __longlong_as_double(0x7ff8000000000000ll);
            t0 += bad[rr] ? nan : e0[rr];
            t1 += bad[rr] ? nan : best[rr];
        }
    }
    pdl_launch_dependents();
    if (lane == 0) {
        red[warp][0] = t0;
        red[warp][1] = t1;
    }
    __syncthreads();
    const int cta = blockIdx.y * gridDim.x + blockIdx.x;
    const int n_cta = gridDim.x * gridDim.y;
    if (tid == 0) {
        double a = 0.0, b = 0.0;
        for (int w = 0; w < kCoWarps; ++w) {
            a += red[w][0];
            b += red[w][1];
        }
        p.partial[2 * cta] = a;
        p.partial[2 * cta + 1] = b;
        __threadfence();
        last = (atomicAdd(p.counter, 1) == n_cta - 1);
    }
    __syncthreads();
    if (last && warp == 0) {
        __threadfence();
        // lane l adds the CTAs l, l + 32, ... in order, then a fixed shuffle tree
        double a = 0.0, b = 0.0;
        for (int c0 = lane; c0 < n_cta; c0 += 32) {
            a += __ldcg(p.partial + 2 * c0);
            b += __ldcg(p.partial + 2 * c0 + 1);
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

template <int kE>
size_t co_smem_bytes() {
    constexpr int G = 32 * kE;
    return (size_t)G * G * sizeof(float) + (size_t)kCoWarps * kCoRowsPerWarp * G * sizeof(float);
}

template <int kE>
cudaError_t launch_co(const CoParams& p, int64_t row_blocks, cudaStream_t st) {
    const size_t smem = co_smem_bytes<kE>();
    static int configured[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64 || !configured[dev]) {
        cudaError_t e = cudaFuncSetAttribute(clip_output_kernel<kE>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) configured[dev] = 1;
    }
    const dim3 grid((unsigned)(p.d_in / (32 * kE)), (unsigned)row_blocks);
    return launch_pdl(clip_output_kernel<kE>, grid, dim3(kCoThreads), smem, st, p);
}

}  // namespace

size_t clip_output_workspace(int64_t d_out, int64_t d_in, int group_size) {
    const int64_t ctas = (d_in / group_size) * ((d_out + kCoRows - 1) / kCoRows);
    return align_up((size_t)d_in * (size_t)group_size * sizeof(float), kWsAlign) +
           align_up((size_t)ctas * 2 * sizeof(double), kWsAlign) + kWsAlign +
           align_up((size_t)kMaxGramSlices * d_in * group_size * sizeof(double), kWsAlign);
}

cudaError_t clip_output_unit_flags(unsigned int* bits, bool clear) {
    return unit_device_flags(bits, clear);
}

cudaError_t launch_clip_search_output(const void* X, int64_t T, int64_t ld, const void* W,
                                      int64_t d_out, int64_t d_in, const float* s,
                                      int group_size, int n_clip, int flags, uint8_t* clip_idx,
                                      double* err, void* ws, cudaStream_t stream) {
    const int64_t G = d_in / group_size;
    const int64_t row_blocks = (d_out + kCoRows - 1) / kCoRows;
    if (G * row_blocks > kMaxCoCtas || row_blocks > 65535) return cudaErrorInvalidValue;
    char* base = static_cast<char*>(ws);
    float* H = reinterpret_cast<float*>(base);
    base += align_up((size_t)d_in * (size_t)group_size * sizeof(float), kWsAlign);
    double* partial = reinterpret_cast<double*>(base);
    base += align_up((size_t)G * row_blocks * 2 * sizeof(double), kWsAlign);
    int* counter = reinterpret_cast<int*>(base);
    base += kWsAlign;
    double* Hpart = reinterpret_cast<double*>(base);

    DeviceInfo dev;
    cudaError_t e = query_device(&dev);
    if (e != cudaSuccess) return e;
    e = cudaMemsetAsync(counter, 0, sizeof(int), stream);
    if (e != cudaSuccess) return e;
    const __half* Xh = static_cast<const __half*>(X);
    // token slices: about two CTAs per SM in all, at least 64 tokens a slice
    const int tiles = group_size == 32 ? 1 : group_size / 64;
    const int64_t gram_ctas = G * (tiles * (tiles + 1) / 2);
    int64_t slices = (2 * (int64_t)dev.num_sms + gram_ctas - 1) / gram_ctas;
    slices = std::max<int64_t>(1, std::min<int64_t>({slices, (int64_t)kMaxGramSlices, T / 64}));
    const int64_t t_per = ((T + slices - 1) / slices + 31) / 32 * 32;
    slices = (T + t_per - 1) / t_per;
    if (slices < 1) slices = 1;
    if (group_size == 32) {
        e = launch_pdl(gram_kernel<32>, dim3((unsigned)G, (unsigned)slices), dim3(64), 0, stream,
                       Xh, T, ld, group_size, t_per, Hpart);
    } else {
        e = launch_pdl(gram_kernel<64>, dim3((unsigned)gram_ctas, (unsigned)slices), dim3(256), 0,
                       stream, Xh, T, ld, group_size, t_per, Hpart);
    }
    if (e != cudaSuccess) return e;
    const int64_t n_h = d_in * (int64_t)group_size;
    e = launch_pdl(gram_reduce_kernel, dim3((unsigned)std::min<int64_t>((n_h + 255) / 256,
                                                                          4 * (int64_t)dev.num_sms)),
                   dim3(256), 0, stream, static_cast<const double*>(Hpart), (int)slices, n_h, H);
    if (e != cudaSuccess) return e;
    CoParams p;
    std::memset(&p, 0, sizeof(p));
    p.W = static_cast<const __half*>(W);
    p.d_out = d_out;
    p.d_in = d_in;
    p.s = s;
    p.H = H;
    p.n_clip = n_clip;
    p.fp32_scale = (flags & AWQ_SCALE_FP32) ? 1 : 0;
    p.idx = clip_idx;
    p.partial = partial;
    p.counter = counter;
    p.err = err;
    switch (group_size) {
        case 32: return launch_co<1>(p, row_blocks, stream);
        case 64: return launch_co<2>(p, row_blocks, stream);
        case 128: return launch_co<4>(p, row_blocks, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace awq
