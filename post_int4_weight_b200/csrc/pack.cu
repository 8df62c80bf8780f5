// pack.cu -- group-wise symmetric INT4 quantisation of W*s and packing into
// the AutoAWQ GEMM layout ("From-Scratch AWQ INT4 Quantization on Qwen3-8B",
// sections "Group-wise symmetric INT4", "AutoAWQ / HF-AWQ GEMM on-disk
// format" and exporter step 4; "AWQ architecture, in depth", section
// "Quantization, storage and packing").
//
//   u[r, j]       = clamp(rint(RN(fl32(w*s) / q_scale)), -7, 7) + zero_point
//   qweight[j, c] = nibble p holds u[8c + order[p], j], order {0,2,4,6,1,3,5,7}
//   scales[k, r]  = fp16 q_scale;   qzeros[k, c] = zero_point in every nibble
//
// HBM-bound: each weight is read once (2 B); 0.5 B of codes plus the group
// scale (2/g B) and zero word (0.5/g B) are written.  One CTA handles a
// 128-row x 128-column tile (one to four whole groups):
//   phase 1  coalesced 16-byte loads of the tile into shared memory, the
//            16-byte chunk index XOR-swizzled by (r ^ r>>4) & 7 so that the
//            row-wise reads of phase 2 and the column-wise reads of phase 3
//            are both free of bank conflicts;
//   phase 2  two threads per (row, group): max |w*s| (NaN-propagating) ->
//            q_scale, written to `scales`, and its correctly rounded
//            reciprocal;
//   phase 3  one thread per (2 columns, 32 rows): the quotient from the
//            correctly rounded reciprocal with one residual correction,
//            whose rounding decision is the IEEE quotient's (quot_rcp1_2,
//            checked against __fdiv_rn around every half-integer), rounding
//            by the 1.5*2^23 addition, nibble placement with one integer
//            multiply-add per code, and one 16-byte store per column (four
//            consecutive output words; four threads write 64 contiguous
//            bytes of a qweight row).  Row blocks whose scales are all fp16
//            normal numbers skip the clamp (|quotient| < 7.5 there).
#include "common.cuh"
#include "internal.h"

namespace awq {
namespace {

constexpr int kPackRows = 128;
constexpr int kPackCols = 128;
constexpr int kPackChunks = kPackCols / 8;     // 16-byte chunks per tile row
constexpr int kPackThreads = 256;
constexpr int kBlocks32 = kPackRows / 32;      // 32-row blocks per tile
constexpr int kClipDen = 20;                   // clip ratio c_i = (20 - i) / 20
constexpr int kClipMaxIndex = 19;

__device__ __forceinline__ int pack_swz(int r) { return (r ^ (r >> 4)) & 7; }

// Per-row arrays are padded by one slot per 32 rows, so the four rows
// 32*cq + i that a warp's lanes read together fall in different banks.
constexpr int kRowStride = kPackRows + kPackRows / 32;
__device__ __forceinline__ int row_slot(int kk, int r) { return kk * kRowStride + r + (r >> 5); }

// nibble position of row offset r8 (0..7) inside its word: order[p] = r8
__device__ __forceinline__ constexpr int nibble_of_row(int r8) {
    return (r8 >> 1) + 4 * (r8 & 1);
}

// NaN-propagating maximum / minimum of three values (a NaN anywhere gives NaN)
__device__ __forceinline__ float max3_nan(float a, float b, float c) {
    float d;
    asm("max.NaN.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}
__device__ __forceinline__ float min3_nan(float a, float b, float c) {
    float d;
    asm("min.NaN.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// |s| of tile column j is kept at j + 4 * (j / 64): the two threads of a
// (row, group) pair in phase 2 read columns 64 apart, which then fall in
// different banks.
__device__ __forceinline__ int sabs_slot(int j) { return j + 4 * (j >> 6); }

// kAsym: codes rint(quotient) + zero of the row, clamped to 0..15; the
// rows' zero points enter through word_init (one per word).
template <int G, bool kFast, bool kAsym>
__device__ __forceinline__ void pack_columns(const uint4* tile, const float2* qr_tile,
                                             const int* bad_tile, const int* zero_tile,
                                             int jp, int cq, int kk, float2 s2,
                                             const uint32_t word_init[4],
                                             uint32_t words[2][4]) {
    const float2 magic2 = make_float2(kRoundMagic, kRoundMagic);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        words[0][q] = word_init[q];
        words[1][q] = word_init[q];
    }
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        const int r = 32 * cq + i;
        const uint32_t v = reinterpret_cast<const uint32_t*>(
            tile + r * kPackChunks + ((jp >> 2) ^ pack_swz(r)))[jp & 3];
        const float2 qr = qr_tile[row_slot(kk, r)];     // (q_scale, 1/q_scale)
        const float qs = qr.x, rq = qr.y;
        const float2 w = __half22float2(*reinterpret_cast<const __half2*>(&v));
        const float2 a = __fmul2_rn(w, s2);
        const float2 nb2 = make_float2(-qs, -qs);
        const float2 y2 = make_float2(rq, rq);
        // a / qs with one residual correction of a * RN(1/qs): its rounding
        // decision is the IEEE quotient's (see quot_rcp1_2)
        const float2 q = quot_rcp1_2(a, nb2, y2);
        float2 t = __fadd2_rn(q, magic2);
        if (kAsym) {
            const float z = (float)zero_tile[row_slot(kk, r)];
            const float lo = kRoundMagic - z, hi = kRoundMagic + 15.f - z;
            t.x = fminf(fmaxf(t.x, lo), hi);
            t.y = fminf(fmaxf(t.y, lo), hi);
            if (bad_tile[row_slot(kk, r)]) t = magic2;   // code = zero point (8)
        } else if (!kFast) {
            t.x = fminf(fmaxf(t.x, kRoundMagic - 7.f), kRoundMagic + 7.f);
            t.y = fminf(fmaxf(t.y, kRoundMagic - 7.f), kRoundMagic + 7.f);
            if (bad_tile[row_slot(kk, r)]) t = magic2;   // code = zero point
        }
        const uint32_t shift = 1u << (4 * nibble_of_row(i & 7));
        words[0][i >> 3] += __float_as_uint(t.x) * shift;
        words[1][i >> 3] += __float_as_uint(t.y) * shift;
    }
}

template <int G, bool kAsym>
__global__ void __launch_bounds__(kPackThreads, 5)
pack_kernel(const uint4* __restrict__ W, int64_t d_out, int64_t d_in,
            const float* __restrict__ s, const uint8_t* __restrict__ clip_idx, int zero_point,
            int32_t* __restrict__ qweight, __half* __restrict__ scales,
            int32_t* __restrict__ qzeros) {
    constexpr int KG = kPackCols / G;               // groups per tile
    extern __shared__ __align__(16) unsigned char smem[];
    uint4* tile = reinterpret_cast<uint4*>(smem);                       // 32 KB
    float* s_tile = reinterpret_cast<float*>(smem + kPackRows * kPackCols * 2);
    float* sabs_tile = s_tile + kPackCols;                               // |s|, padded
    float2* qr_tile = reinterpret_cast<float2*>(sabs_tile + kPackCols + 8);  // [KG][kRowStride]
    int* bad_tile = reinterpret_cast<int*>(qr_tile + KG * kRowStride);  // [KG][kRowStride]
    int* slow_blk = bad_tile + KG * kRowStride;                          // [KG][kBlocks32]
    int* zero_tile = slow_blk + KG * kBlocks32;                          // [KG][kRowStride]
    uint32_t* zw_tile = reinterpret_cast<uint32_t*>(zero_tile + KG * kRowStride);  // [KG][16]
    float* ssgn_tile = reinterpret_cast<float*>(zw_tile + KG * (kPackRows / 8));   // s, padded

    // a programmatic dependent launch: W and s may come from the kernel before
    pdl_wait();
    const int tid = threadIdx.x;
    const int64_t col0 = (int64_t)blockIdx.x * kPackCols;
    const int64_t row0 = (int64_t)blockIdx.y * kPackRows;
    const int64_t ld4 = d_in / 8;

    // ---- phase 1: tile -> shared memory (all eight 16-byte loads in flight)
    {
        const uint4* base = W + row0 * ld4 + col0 / 8;
        const int rows_here = (int)min((int64_t)kPackRows, d_out - row0);
        const int chunks_here = (int)min((int64_t)kPackChunks, (d_in - col0) / 8);
        uint4 v[kPackRows * kPackChunks / kPackThreads];
#pragma unroll
        for (int k = 0; k < kPackRows * kPackChunks / kPackThreads; ++k) {
            const int i = tid + k * kPackThreads;
            const int r = i / kPackChunks, c = i % kPackChunks;
            v[k] = (r < rows_here && c < chunks_here) ? __ldg(base + (int64_t)r * ld4 + c)
                                                       : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int k = 0; k < kPackRows * kPackChunks / kPackThreads; ++k) {
            const int i = tid + k * kPackThreads;
            const int r = i / kPackChunks, c = i % kPackChunks;
            tile[r * kPackChunks + (c ^ pack_swz(r))] = v[k];
        }
    }
    if (tid < kPackCols) {
        const int64_t gc = col0 + tid;
        const float sv = gc < d_in ? (s ? s[gc] : 1.0f) : 1.0f;
        s_tile[tid] = sv;
        sabs_tile[sabs_slot(tid)] = fabsf(sv);
        if (kAsym) ssgn_tile[sabs_slot(tid)] = sv;
    }
    if (tid < KG * kBlocks32) slow_blk[tid] = 0;
    pdl_launch_dependents();   // the tile is read; the next kernel may start launching
    __syncthreads();

    // ---- phase 2: group scale of every (row, group), two threads each.
    if (kAsym) {
        // asymmetric grid: the signed max and min of w s (NaN-propagating)
        for (int task = tid; task < 2 * KG * kPackRows; task += kPackThreads) {
            const int half = task & 1;
            const int r = (task >> 1) % kPackRows, kk = (task >> 1) / kPackRows;
            float mx = __int_as_float(0xff800000), mn = __int_as_float(0x7f800000);
#pragma unroll
            for (int cc = 0; cc < G / 16; ++cc) {
                const int c = kk * (G / 8) + half * (G / 16) + cc;
                const uint4 v = tile[r * kPackChunks + (c ^ pack_swz(r))];
                const uint32_t hw[4] = {v.x, v.y, v.z, v.w};
                const float4 sa = *reinterpret_cast<const float4*>(&ssgn_tile[sabs_slot(8 * c)]);
                const float4 sb =
                    *reinterpret_cast<const float4*>(&ssgn_tile[sabs_slot(8 * c + 4)]);
                const float sv[8] = {sa.x, sa.y, sa.z, sa.w, sb.x, sb.y, sb.z, sb.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float2 w = __half22float2(*reinterpret_cast<const __half2*>(&hw[i]));
                    const float2 a = __fmul2_rn(w, make_float2(sv[2 * i], sv[2 * i + 1]));
                    mx = max3_nan(mx, a.x, a.y);
                    mn = min3_nan(mn, a.x, a.y);
                }
            }
            {
                const float ox = __shfl_xor_sync(0xffffffffu, mx, 1);
                const float on = __shfl_xor_sync(0xffffffffu, mn, 1);
                mx = max3_nan(mx, ox, ox);
                mn = min3_nan(mn, on, on);
            }
            if (half == 0) {
                const bool bad = !(mx <= 3.402823466e38f) || !(mn >= -3.402823466e38f);
                float qs = 1.0f;
                int z = 8;
                if (!bad) {
                    const float range = fmaxf(__fsub_rn(mx, mn), 1e-5f);
                    qs = fminf(__half2float(__float2half_rn(div15_rn(range))), kHalfMax);
                    z = (int)fminf(fmaxf(rintf(div_rn_rcp(-mn, qs, __frcp_rn(qs))), 0.f), 15.f);
                }
                qr_tile[row_slot(kk, r)] = make_float2(qs, __frcp_rn(qs));
                bad_tile[row_slot(kk, r)] = bad;
                zero_tile[row_slot(kk, r)] = z;
                if (bad) raise_device_flag(AWQ_FLAG_NONFINITE_GROUP);
                const int64_t gr = row0 + r, gk = col0 / G + kk;
                if (gr < d_out && gk * G < d_in)
                    scales[gk * d_out + gr] = bad ? __ushort_as_half((unsigned short)0x7E00)
                                                  : __float2half_rn(qs);
            }
        }
        __syncthreads();
        // zero-point words of every 8-row block: nibble p holds row 8c + order[p]
        for (int i = tid; i < KG * (kPackRows / 8); i += kPackThreads) {
            const int kk = i / (kPackRows / 8), c8 = i % (kPackRows / 8);
            uint32_t wv = 0;
#pragma unroll
            for (int i8 = 0; i8 < 8; ++i8)
                wv |= (uint32_t)zero_tile[row_slot(kk, 8 * c8 + i8)] << (4 * nibble_of_row(i8));
            zw_tile[kk * (kPackRows / 8) + c8] = wv;
        }
    } else {
        // max |w s| = max |w| |s|: the sign bits are cleared before the fp16 ->
        // fp32 conversion, so the products are non-negative and a three-input
        // NaN-propagating maximum takes two of them per instruction.
        for (int task = tid; task < 2 * KG * kPackRows; task += kPackThreads) {
            const int half = task & 1;
            const int r = (task >> 1) % kPackRows, kk = (task >> 1) / kPackRows;
            float m = 0.f;
#pragma unroll
            for (int cc = 0; cc < G / 16; ++cc) {
                const int c = kk * (G / 8) + half * (G / 16) + cc;
                const uint4 v = tile[r * kPackChunks + (c ^ pack_swz(r))];
                const uint32_t hw[4] = {v.x & 0x7fff7fffu, v.y & 0x7fff7fffu, v.z & 0x7fff7fffu,
                                        v.w & 0x7fff7fffu};
                const float4 sa = *reinterpret_cast<const float4*>(&sabs_tile[sabs_slot(8 * c)]);
                const float4 sb = *reinterpret_cast<const float4*>(&sabs_tile[sabs_slot(8 * c + 4)]);
                const float sv[8] = {sa.x, sa.y, sa.z, sa.w, sb.x, sb.y, sb.z, sb.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float2 w = __half22float2(*reinterpret_cast<const __half2*>(&hw[i]));
                    const float2 a = __fmul2_rn(w, make_float2(sv[2 * i], sv[2 * i + 1]));
                    m = max3_nan(m, a.x, a.y);
                }
            }
            {
                const float o = __shfl_xor_sync(0xffffffffu, m, 1);
                m = max3_nan(m, o, o);
            }
            if (half == 0) {
                const bool bad = !(m <= 3.402823466e38f);      // a NaN or an infinity
                const int64_t gr = row0 + r, gk = col0 / G + kk;
                // clipping shrinks the range to c * m, c = RN((20 - i) / 20); codes
                // beyond it saturate, so the block takes the clamping path
                bool clipped = false;
                if (clip_idx && gr < d_out && gk * G < d_in) {
                    const int ci = min((int)clip_idx[gr * (d_in / G) + gk], kClipMaxIndex);
                    if (ci > 0) {
                        m = __fmul_rn(m, __fdiv_rn((float)(kClipDen - ci), (float)kClipDen));
                        clipped = true;
                    }
                }
                bool in_range;
                const float qs = bad ? 1.0f : group_scale(m, false, &in_range);
                qr_tile[row_slot(kk, r)] = make_float2(qs, (qs > 0.f) ? __frcp_rn(qs) : 0.f);
                bad_tile[row_slot(kk, r)] = bad;
                if (bad) raise_device_flag(AWQ_FLAG_NONFINITE_GROUP);
                if (bad || clipped || !in_range) slow_blk[kk * kBlocks32 + r / 32] = 1;
                if (gr < d_out && gk * G < d_in)
                    scales[gk * d_out + gr] = bad ? __ushort_as_half((unsigned short)0x7E00)
                                                  : __float2half_rn(qs);
            }
        }
    }
    __syncthreads();

    // ---- phase 3: codes and packed words
    const int64_t C = d_out / 8;
    const int64_t c0 = row0 / 8;
    {
        const int cq = tid & 3;          // 4 output words = 32 rows
        const int jp = tid >> 2;         // 2 input columns
        const int kk = (2 * jp) / G;
        const float2 s2 = make_float2(s_tile[2 * jp], s_tile[2 * jp + 1]);
        // each nibble starts at (zero point - bits of 1.5*2^23); adding the
        // bits of the rounded quotient + 1.5*2^23 leaves the unsigned code
        uint32_t word_init[4];
#pragma unroll
        for (int q = 0; q < 4; ++q)
            word_init[q] = kAsym ? zw_tile[kk * (kPackRows / 8) + 4 * cq + q] -
                                       kRoundMagicBits * 0x11111111u
                                 : 0u - (kRoundMagicBits - (uint32_t)zero_point) * 0x11111111u;
        uint32_t words[2][4];
        if (kAsym)
            pack_columns<G, false, true>(tile, qr_tile, bad_tile, zero_tile, jp, cq, kk, s2,
                                         word_init, words);
        else if (slow_blk[kk * kBlocks32 + cq])
            pack_columns<G, false, false>(tile, qr_tile, bad_tile, zero_tile, jp, cq, kk, s2,
                                          word_init, words);
        else
            pack_columns<G, true, false>(tile, qr_tile, bad_tile, zero_tile, jp, cq, kk, s2,
                                         word_init, words);
        const int64_t cw = c0 + 4 * cq;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int64_t j = col0 + 2 * jp + e;
            if (j >= d_in) continue;
            int32_t* dst = qweight + j * C + cw;
            if ((C & 3) == 0 && cw + 3 < C) {
                *reinterpret_cast<uint4*>(dst) =
                    make_uint4(words[e][0], words[e][1], words[e][2], words[e][3]);
            } else {
                for (int q = 0; q < 4; ++q)
                    if (cw + q < C) dst[q] = (int32_t)words[e][q];
            }
        }
    }

    // ---- qzeros of the tile's groups and words
    uint32_t zword = (uint32_t)zero_point & 0xFu;
    zword *= 0x11111111u;
    for (int i = tid; i < KG * (kPackRows / 8); i += kPackThreads) {
        const int kk = i / (kPackRows / 8), cwl = i % (kPackRows / 8);
        const int64_t gk = col0 / G + kk, cw = c0 + cwl;
        if (gk * G < d_in && cw < C)
            qzeros[gk * C + cw] = (int32_t)(kAsym ? zw_tile[i] : zword);
    }
}

template <int G>
cudaError_t launch_pack_G(const void* W, int64_t d_out, int64_t d_in, const float* s,
                          const uint8_t* clip_idx, int zero_point, int32_t* qweight,
                          void* scales, int32_t* qzeros, cudaStream_t stream) {
    constexpr int KG = kPackCols / G;
    const size_t smem = (size_t)kPackRows * kPackCols * 2 + (2 * kPackCols + 8) * sizeof(float) +
                        (size_t)KG * kRowStride * (sizeof(float2) + sizeof(int)) +
                        (size_t)KG * kBlocks32 * sizeof(int) +
                        (size_t)KG * kRowStride * sizeof(int) +          // zero points
                        (size_t)KG * (kPackRows / 8) * sizeof(uint32_t) +  // zero words
                        (size_t)(kPackCols + 8) * sizeof(float);          // signed s, padded
    const bool asym = zero_point == AWQ_ZERO_POINT_ASYM;
    static int configured[64][2] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64 || !configured[dev][asym]) {
        cudaError_t e = cudaFuncSetAttribute(asym ? pack_kernel<G, true> : pack_kernel<G, false>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) configured[dev][asym] = 1;
    }
    dim3 grid((unsigned)((d_in + kPackCols - 1) / kPackCols),
              (unsigned)((d_out + kPackRows - 1) / kPackRows));
    return launch_pdl(asym ? pack_kernel<G, true> : pack_kernel<G, false>, grid,
                      dim3(kPackThreads), smem, stream,
                      static_cast<const uint4*>(W), d_out, d_in, s, clip_idx, zero_point,
                      qweight, static_cast<__half*>(scales), qzeros);
}

}  // namespace

cudaError_t pack_unit_flags(unsigned int* bits, bool clear) {
    return unit_device_flags(bits, clear);
}

cudaError_t launch_quantize_pack(const void* W, int64_t d_out, int64_t d_in, const float* s,
                                 const uint8_t* clip_idx, int group_size, int zero_point,
                                 int32_t* qweight, void* scales, int32_t* qzeros,
                                 cudaStream_t stream) {
    switch (group_size) {
        case 32:
            return launch_pack_G<32>(W, d_out, d_in, s, clip_idx, zero_point, qweight, scales,
                                     qzeros, stream);
        case 64:
            return launch_pack_G<64>(W, d_out, d_in, s, clip_idx, zero_point, qweight, scales,
                                     qzeros, stream);
        case 128:
            return launch_pack_G<128>(W, d_out, d_in, s, clip_idx, zero_point, qweight, scales,
                                      qzeros, stream);
        default:
            return cudaErrorInvalidValue;
    }
}

}  // namespace awq
