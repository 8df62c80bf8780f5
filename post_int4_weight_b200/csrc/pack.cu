// pack.cu -- group-wise symmetric INT4 quantisation of W*s and packing into
// the AutoAWQ GEMM layout ("From-Scratch AWQ INT4 Quantization on Qwen3-8B",
// sections "Group-wise symmetric INT4", "AutoAWQ / HF-AWQ GEMM on-disk
// format" and exporter step 4; "AWQ architecture, in depth", section
// "Quantization, storage and packing").
//
//   u[r, j]       = clamp(rint(fl32(w*s) / q_scale), -7, 7) + zero_point
//   qweight[j, c] = nibble p holds u[8c + order[p], j], order {0,2,4,6,1,3,5,7}
//   scales[k, r]  = fp16 q_scale;   qzeros[k, c] = zero_point in every nibble
//
// HBM-bound: each weight is read once (2 B) and 0.5 B of codes plus the group
// scale is written.  One CTA handles a 256-row x 128-column tile (one or more
// whole groups):
//   phase 1  coalesced 16-byte loads of the tile into shared memory, with the
//            16-byte chunk index XOR-swizzled by (r ^ r>>5) & 7 so that both
//            later access patterns are free of bank conflicts;
//   phase 2  one thread per (row, group): max |w*s| -> q_scale (fp32 quotient
//            by 7, fp16 round-to-nearest-even), written to `scales`;
//   phase 3  one thread per (4 columns, 32 rows): codes with the exact IEEE
//            quotient, nibbles placed in AutoAWQ order, four consecutive
//            output words per column written with one 16-byte store (eight
//            threads cover 128 contiguous bytes of a qweight row).
#include "common.cuh"
#include "internal.h"

namespace awq {
namespace {

constexpr int kPackRows = 256;
constexpr int kPackCols = 128;
constexpr int kPackChunks = kPackCols / 8;     // 16-byte chunks per tile row
constexpr int kPackThreads = 256;

__device__ __forceinline__ int pack_swz(int r) { return (r ^ (r >> 5)) & 7; }

// nibble position of row offset r8 (0..7) inside its word: order[p] = r8
__device__ __forceinline__ constexpr int nibble_of_row(int r8) {
    return (r8 >> 1) + 4 * (r8 & 1);
}

template <int G>
__global__ void __launch_bounds__(kPackThreads)
pack_kernel(const uint4* __restrict__ W, int64_t d_out, int64_t d_in,
            const float* __restrict__ s, int zero_point, int32_t* __restrict__ qweight,
            __half* __restrict__ scales, int32_t* __restrict__ qzeros) {
    constexpr int KG = kPackCols / G;               // groups per tile
    extern __shared__ __align__(16) unsigned char smem[];
    uint4* tile = reinterpret_cast<uint4*>(smem);                       // 64 KB
    float* s_tile = reinterpret_cast<float*>(smem + kPackRows * kPackCols * 2);
    float* qs_tile = s_tile + kPackCols;                                 // [KG][rows]
    int* bad_tile = reinterpret_cast<int*>(qs_tile + KG * kPackRows);   // [KG][rows]

    const int tid = threadIdx.x;
    const int64_t col0 = (int64_t)blockIdx.x * kPackCols;
    const int64_t row0 = (int64_t)blockIdx.y * kPackRows;
    const int64_t ld4 = d_in / 8;

    // ---- phase 1: tile -> shared memory
    for (int i = tid; i < kPackRows * kPackChunks; i += kPackThreads) {
        const int r = i / kPackChunks, c = i % kPackChunks;
        const int64_t gr = row0 + r, gc = col0 + 8 * c;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (gr < d_out && gc < d_in) v = __ldg(W + gr * ld4 + gc / 8);
        tile[r * kPackChunks + (c ^ pack_swz(r))] = v;
    }
    if (tid < kPackCols) {
        const int64_t gc = col0 + tid;
        s_tile[tid] = gc < d_in ? (s ? s[gc] : 1.0f) : 1.0f;
    }
    __syncthreads();

    // ---- phase 2: group scale of every (row, group)
    for (int task = tid; task < KG * kPackRows; task += kPackThreads) {
        const int r = task % kPackRows, kk = task / kPackRows;
        float m = 0.f;
        bool bad = false;
#pragma unroll
        for (int cc = 0; cc < G / 8; ++cc) {
            const int c = kk * (G / 8) + cc;
            const uint4 v = tile[r * kPackChunks + (c ^ pack_swz(r))];
            const uint32_t hw[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float2 w = __half22float2(*reinterpret_cast<const __half2*>(&hw[i]));
                const float a = __fmul_rn(w.x, s_tile[8 * c + 2 * i]);
                const float b = __fmul_rn(w.y, s_tile[8 * c + 2 * i + 1]);
                bad |= !(fabsf(a) <= 3.402823466e38f) || !(fabsf(b) <= 3.402823466e38f);
                m = fmaxf(m, fmaxf(fabsf(a), fabsf(b)));
            }
        }
        bool in_range;
        float qs = group_scale(m, false, &in_range);
        if (bad) qs = __int_as_float(0x7fc00000);
        qs_tile[kk * kPackRows + r] = qs;
        bad_tile[kk * kPackRows + r] = bad;
        const int64_t gr = row0 + r, gk = col0 / G + kk;
        if (gr < d_out && gk * G < d_in)
            scales[gk * d_out + gr] = bad ? __ushort_as_half((unsigned short)0x7E00)
                                          : __float2half_rn(qs);
    }
    __syncthreads();

    // ---- phase 3: codes and packed words
    const int64_t C = d_out / 8;
    const int64_t c0 = row0 / 8;
    const uint32_t bias = kRoundMagicBits - (uint32_t)zero_point;
    for (int task = tid; task < (kPackCols / 4) * (kPackRows / 32); task += kPackThreads) {
        const int cq = task % (kPackRows / 32);   // 4 output words = 32 rows
        const int jq = task / (kPackRows / 32);   // 4 input columns
        const int kk = (4 * jq) / G;
        float sreg[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) sreg[e] = s_tile[4 * jq + e];
        uint32_t words[4][4] = {};
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const int r = 32 * cq + i;
            const uint2 v = reinterpret_cast<const uint2*>(
                tile + r * kPackChunks + ((jq >> 1) ^ pack_swz(r)))[jq & 1];
            const float qs = qs_tile[kk * kPackRows + r];
            const bool bad = bad_tile[kk * kPackRows + r] != 0;
            const float2 w01 = __half22float2(*reinterpret_cast<const __half2*>(&v.x));
            const float2 w23 = __half22float2(*reinterpret_cast<const __half2*>(&v.y));
            const float wv[4] = {w01.x, w01.y, w23.x, w23.y};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float ws = __fmul_rn(wv[e], sreg[e]);
                const float y = (qs > 0.f) ? __fdiv_rn(ws, qs) : 0.f;
                float t = __fadd_rn(y, kRoundMagic);
                t = fminf(fmaxf(t, kRoundMagic - 7.f), kRoundMagic + 7.f);
                uint32_t u = __float_as_uint(t) - bias;
                if (bad) u = (uint32_t)zero_point;
                words[e][i >> 3] |= (u & 0xFu) << (4 * nibble_of_row(i & 7));
            }
        }
        const int64_t cw = c0 + 4 * cq;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int64_t j = col0 + 4 * jq + e;
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
    zword |= zword << 4;
    zword |= zword << 8;
    zword |= zword << 16;
    for (int i = tid; i < KG * (kPackRows / 8); i += kPackThreads) {
        const int kk = i / (kPackRows / 8), cwl = i % (kPackRows / 8);
        const int64_t gk = col0 / G + kk, cw = c0 + cwl;
        if (gk * G < d_in && cw < C) qzeros[gk * C + cw] = (int32_t)zword;
    }
}

template <int G>
cudaError_t launch_pack_G(const void* W, int64_t d_out, int64_t d_in, const float* s,
                          int zero_point, int32_t* qweight, void* scales, int32_t* qzeros,
                          cudaStream_t stream) {
    constexpr int KG = kPackCols / G;
    const size_t smem = (size_t)kPackRows * kPackCols * 2 + kPackCols * sizeof(float) +
                        (size_t)KG * kPackRows * (sizeof(float) + sizeof(int));
    cudaError_t e = cudaFuncSetAttribute(pack_kernel<G>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)((d_in + kPackCols - 1) / kPackCols),
              (unsigned)((d_out + kPackRows - 1) / kPackRows));
    pack_kernel<G><<<grid, kPackThreads, smem, stream>>>(
        static_cast<const uint4*>(W), d_out, d_in, s, zero_point, qweight,
        static_cast<__half*>(scales), qzeros);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_quantize_pack(const void* W, int64_t d_out, int64_t d_in, const float* s,
                                 int group_size, int zero_point, int32_t* qweight,
                                 void* scales, int32_t* qzeros, cudaStream_t stream) {
    switch (group_size) {
        case 32:
            return launch_pack_G<32>(W, d_out, d_in, s, zero_point, qweight, scales, qzeros,
                                     stream);
        case 64:
            return launch_pack_G<64>(W, d_out, d_in, s, zero_point, qweight, scales, qzeros,
                                     stream);
        case 128:
            return launch_pack_G<128>(W, d_out, d_in, s, zero_point, qweight, scales, qzeros,
                                      stream);
        default:
            return cudaErrorInvalidValue;
    }
}

}  // namespace awq
