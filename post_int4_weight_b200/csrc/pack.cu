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
// scale (2/g B) and zero word (0.5/g B) are written.  One CTA of 4 warps
// handles a 64-row x 128-column tile (one to four whole groups), 11 CTAs
// per SM so that one CTA's tile streams in while others compute (the
// 64-row tile halves the last wave's work against a 128-row one):
//   load     one thread issues two TMA copies (cp.async.bulk.tensor, 64
//            columns x 64 rows each, 128-byte swizzle: 16-byte chunk c of
//            row r sits at chunk c ^ (r & 7)); no thread spends an
//            instruction on loading;
//   scale    two threads per row (one per 64-column half) take max |w*s|
//            (NaN-propagating) of their half from 16-byte shared-memory reads
//            (conflict-free under the swizzle) -> q_scale, its correctly
//            rounded reciprocal, the stored fp16 scale;
//   codes    warp w packs rows 32(w/2)..32(w/2)+31 of the 64-column half
//            w % 2; lane l takes 2 consecutive columns of it (4-byte reads:
//            the warp reads one whole 128-byte row, conflict-free, and the
//            swizzle term r & 7 = i & 7 is a constant of the unrolled row
//            loop).  The quotient comes from the correctly rounded
//            reciprocal with one residual correction, whose rounding
//            decision is the IEEE quotient's (quot_rcp1_2, checked against
//            __fdiv_rn around every half-integer); the 1.5*2^23 addition
//            rounds it; one integer multiply-add per code places its
//            nibble; the four words of a column (32 rows) leave in one
//            16-byte store.  Row blocks whose scales are all fp16 normal
//            numbers skip the clamp (|quotient| < 7.5 there).
#include <cstring>

#include "common.cuh"
#include "internal.h"

namespace awq {
namespace {

constexpr int kPackRows = 64;                   // two threads per row
constexpr int kPackCols = 128;
constexpr int kBoxCols = 64;                    // 128 bytes: one swizzle row
constexpr int kBoxBytes = kPackRows * kBoxCols * 2;   // 8 KB per box
constexpr int kTileBytes = 2 * kBoxBytes;
constexpr int kPackThreads = 2 * kPackRows;
constexpr int kPackWarps = kPackThreads / 32;
constexpr int kRowsPerWarp = 32;                // rows of one warp's codes (one half of the tile)
constexpr int kPackCtasPerSm = 11;              // the shared-memory limit
constexpr int kClipDen = 20;                    // clip ratio c_i = (20 - i) / 20
constexpr int kClipMaxIndex = 19;
// per-(group, row) arrays: rows padded so the groups of one warp's lanes
// (g = 32: four groups) fall in different banks
constexpr int kRowStride = kPackRows + 4;

struct PackParams {
    CUtensorMap tmap;          // W fp16 [d_out, d_in], box {64, 64}, 128-byte swizzle
    int64_t d_out, d_in;
    const float* s;            // [d_in] or NULL (s = 1)
    const uint8_t* clip_idx;   // [d_out, d_in / G] or NULL
    int zero_point;            // 7, 8 or AWQ_ZERO_POINT_ASYM
    int32_t* qweight;          // [d_in, d_out / 8]
    __half* scales;            // [d_in / G, d_out]
    int32_t* qzeros;           // [d_in / G, d_out / 8]
};

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

// |s| and s of tile column j are kept at j + 4 * (j / 64): the two halves'
// threads of a warp read columns 64 apart, which then fall in different banks.
__device__ __forceinline__ int s_slot(int j) { return j + 4 * (j >> 6); }

// Byte offset of 16-byte chunk c (0..7) of row r in a 128-byte-swizzled box.
__device__ __forceinline__ int swz(int r, int c) { return r * 128 + ((c ^ (r & 7)) << 4); }

// Codes of one lane's 2 columns over the warp's 32 rows, packed into four
// words per column (one 16-byte store).  kSlow: clamp the codes (and store
// the zero point for a non-finite group); taken per lane outside the row
// loop, so the loop itself has no branch.
template <bool kSlow, bool kAsym>
__device__ __forceinline__ void pack_rows(const unsigned char* box, int chunk, float2 s01,
                                          const float2* qr_row, const int* bad_row,
                                          const int* zero_row, uint32_t words[2][4]) {
    const float2 magic2 = make_float2(kRoundMagic, kRoundMagic);
#pragma unroll
    for (int i = 0; i < kRowsPerWarp; ++i) {
        // row rb + i: (rb + i) & 7 == i & 7, so the swizzle is a constant
        const uint32_t v = *reinterpret_cast<const uint32_t*>(box + i * 128 +
                                                              ((chunk ^ (i & 7)) << 4));
        const float2 qr = qr_row[i];           // (q_scale, 1 / q_scale)
        const float2 nb2 = make_float2(-qr.x, -qr.x), y2 = make_float2(qr.y, qr.y);
        const float2 w01 = __half22float2(*reinterpret_cast<const __half2*>(&v));
        // w s / q_scale with one residual correction of w s * RN(1 / q_scale):
        // its rounding decision is the IEEE quotient's (see quot_rcp1_2)
        float2 t01 = __fadd2_rn(quot_rcp1_2(__fmul2_rn(w01, s01), nb2, y2), magic2);
        if (kSlow) {
            float lo = kRoundMagic - 7.f, hi = kRoundMagic + 7.f;
            if (kAsym) {
                const float z = (float)zero_row[i];
                lo = kRoundMagic - z;
                hi = kRoundMagic + 15.f - z;
            }
            t01 = make_float2(fminf(fmaxf(t01.x, lo), hi), fminf(fmaxf(t01.y, lo), hi));
            if (bad_row[i]) t01 = magic2;   // code = zero point
        }
        const uint32_t shift = 1u << (4 * nibble_of_row(i & 7));
        const int hw = i >> 3;
        words[0][hw] += __float_as_uint(t01.x) * shift;
        words[1][hw] += __float_as_uint(t01.y) * shift;
    }
}

template <int G, bool kAsym>
__global__ void __launch_bounds__(kPackThreads, kPackCtasPerSm)
pack_kernel(const __grid_constant__ PackParams p) {
    constexpr int KG = kPackCols / G;                 // groups per tile
    constexpr int kBlocks = kPackRows / kRowsPerWarp;  // 32-row blocks per tile
    static_assert(kPackWarps == 2 * kBlocks, "one warp per (32-row block, 64-column half)");
    extern __shared__ unsigned char smem_raw[];
    // the 128-byte swizzle wants 1024-byte aligned boxes
    const uint32_t raw = smem_addr(smem_raw);
    unsigned char* tile = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
    float* s_tile = reinterpret_cast<float*>(tile + kTileBytes);          // [136] signed s
    float* sabs_tile = s_tile + kPackCols + 8;                            // [136] |s|
    float2* qr_tile = reinterpret_cast<float2*>(sabs_tile + kPackCols + 8);  // [KG][kRowStride]
    int* zero_tile = reinterpret_cast<int*>(qr_tile + KG * kRowStride);     // [KG][kRowStride]
    int* bad_tile = zero_tile + KG * kRowStride;                            // [KG][kRowStride]
    int* slow_blk = bad_tile + KG * kRowStride;                             // [KG][kBlocks]
    uint32_t* zw_tile = reinterpret_cast<uint32_t*>(slow_blk + KG * kBlocks);  // [KG][16]
    uint64_t* bar = reinterpret_cast<uint64_t*>(zw_tile + KG * (kPackRows / 8) + 2);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t col0 = (int64_t)blockIdx.x * kPackCols;
    const int64_t row0 = (int64_t)blockIdx.y * kPackRows;

    if (tid == 0) {
        mbar_init(bar, 1);
        mbar_fence_init();
    }
    if (tid < KG * kBlocks) slow_blk[tid] = 0;
    // a programmatic dependent launch: W and s may come from the kernel before
    pdl_wait();
    __syncthreads();   // the barrier's initialisation is visible to every thread
    if (tid == 0) {
        // the second box only when it starts inside the rows (d_in % 64 may
        // leave a tile half empty); a box's rows or columns beyond W read
        // zeros.  Tile columns at or beyond d_in are never stored or flagged.
        const bool box1 = col0 + kBoxCols < p.d_in;
        tma_prefetch_desc(&p.tmap);
        mbar_arrive_expect_tx(bar, box1 ? kTileBytes : kBoxBytes);
        tma_load_2d(tile, &p.tmap, (int32_t)col0, (int32_t)row0, bar);
        if (box1)
            tma_load_2d(tile + kBoxBytes, &p.tmap, (int32_t)(col0 + kBoxCols), (int32_t)row0,
                        bar);
    }
    for (int j = tid; j < kPackCols; j += kPackThreads) {
        const int64_t gc = col0 + j;
        const float sv = gc < p.d_in ? (p.s ? p.s[gc] : 1.0f) : 1.0f;
        s_tile[s_slot(j)] = sv;
        sabs_tile[s_slot(j)] = fabsf(sv);
    }
    // the only wait of the kernel; a copy that has not landed after the
    // drain limit leaves the tile's outputs unwritten and the timeout bit set
    const bool ok = __syncthreads_and(mbar_wait_drain(bar, 0));
    pdl_launch_dependents();   // the tile is read; the next kernel may start launching
    if (!ok) {
        if (tid == 0) raise_device_flag(AWQ_FLAG_WAIT_TIMEOUT);
        return;
    }

    // ---- group scale of every (row, group) it covers: two threads per row
    {
        const int r = tid >> 1, h = tid & 1;
        const unsigned char* box = tile + h * kBoxBytes;
        // G = 128: one group split over the pair; G = 64: the half is the
        // group; G = 32: chunks 0-3 and 4-7 are two groups
        constexpr int kOwn = (G == 32) ? 2 : 1;
        float mx[kOwn], mn[kOwn];
#pragma unroll
        for (int o = 0; o < kOwn; ++o) {
            mx[o] = kAsym ? __int_as_float(0xff800000) : 0.f;
            mn[o] = __int_as_float(0x7f800000);
        }
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const int o = (G == 32) ? (c >> 2) : 0;
            uint4 v = *reinterpret_cast<const uint4*>(box + swz(r, c));
            const float* sp = kAsym ? s_tile : sabs_tile;
            const float4 sa = *reinterpret_cast<const float4*>(&sp[s_slot(64 * h + 8 * c)]);
            const float4 sb = *reinterpret_cast<const float4*>(&sp[s_slot(64 * h + 8 * c + 4)]);
            const float sv[8] = {sa.x, sa.y, sa.z, sa.w, sb.x, sb.y, sb.z, sb.w};
            if (!kAsym) {   // max |w s| = max |w| |s|: products of non-negative values
                v.x &= 0x7fff7fffu;
                v.y &= 0x7fff7fffu;
                v.z &= 0x7fff7fffu;
                v.w &= 0x7fff7fffu;
            }
            const uint32_t hw[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float2 w = __half22float2(*reinterpret_cast<const __half2*>(&hw[i]));
                const float2 a = __fmul2_rn(w, make_float2(sv[2 * i], sv[2 * i + 1]));
                mx[o] = max3_nan(mx[o], a.x, a.y);
                if (kAsym) mn[o] = min3_nan(mn[o], a.x, a.y);
            }
        }
        if (G == 128) {
            const float ox = __shfl_xor_sync(0xffffffffu, mx[0], 1);
            mx[0] = max3_nan(mx[0], ox, ox);
            if (kAsym) {
                const float on = __shfl_xor_sync(0xffffffffu, mn[0], 1);
                mn[0] = min3_nan(mn[0], on, on);
            }
        }
        const int64_t gr = row0 + r;
        if (G != 128 || h == 0) {
#pragma unroll
            for (int o = 0; o < kOwn; ++o) {
                const int kk = (G == 128) ? 0 : (G == 64 ? h : 2 * h + o);
                const int64_t gk = col0 / G + kk;
                const bool live = gr < p.d_out && gk * G < p.d_in;   // a stored group
                float qs;
                bool bad;
                if (kAsym) {
                    bad = !(mx[o] <= 3.402823466e38f) || !(mn[o] >= -3.402823466e38f);
                    qs = 1.0f;
                    int z = 8;
                    if (!bad) {
                        const float range = fmaxf(__fsub_rn(mx[o], mn[o]), 1e-5f);
                        qs = fminf(__half2float(__float2half_rn(div15_rn(range))), kHalfMax);
                        z = (int)fminf(fmaxf(rintf(div_rn_rcp(-mn[o], qs, __frcp_rn(qs))), 0.f),
                                       15.f);
                    }
                    qr_tile[kk * kRowStride + r] = make_float2(qs, __frcp_rn(qs));
                    zero_tile[kk * kRowStride + r] = z;
                } else {
                    float m = mx[o];
                    bad = !(m <= 3.402823466e38f);      // a NaN or an infinity
                    // clipping shrinks the range to c * m, c = RN((20 - i) / 20);
                    // codes beyond it saturate, so the block takes the clamping path
                    bool clipped = false;
                    if (p.clip_idx && live) {
                        const int ci =
                            min((int)p.clip_idx[gr * (p.d_in / G) + gk], kClipMaxIndex);
                        if (ci > 0) {
                            m = __fmul_rn(m, __fdiv_rn((float)(kClipDen - ci), (float)kClipDen));
                            clipped = true;
                        }
                    }
                    bool in_range;
                    qs = bad ? 1.0f : group_scale(m, false, &in_range);
                    qr_tile[kk * kRowStride + r] =
                        make_float2(qs, (qs > 0.f) ? __frcp_rn(qs) : 0.f);
                    if (bad || clipped || !in_range) slow_blk[kk * kBlocks + r / kRowsPerWarp] = 1;
                }
                bad_tile[kk * kRowStride + r] = bad;
                if (live) {
                    p.scales[gk * p.d_out + gr] = bad ? __ushort_as_half((unsigned short)0x7E00)
                                                      : __float2half_rn(qs);
                    if (bad) raise_device_flag(AWQ_FLAG_NONFINITE_GROUP);
                }
            }
        }
    }
    __syncthreads();
    if (kAsym) {
        // zero-point words of every 8-row block: nibble p holds row 8c + order[p]
        for (int i = tid; i < KG * (kPackRows / 8); i += kPackThreads) {
            const int kk = i / (kPackRows / 8), c8 = i % (kPackRows / 8);
            uint32_t wv = 0;
#pragma unroll
            for (int i8 = 0; i8 < 8; ++i8)
                wv |= (uint32_t)zero_tile[kk * kRowStride + 8 * c8 + i8] << (4 * nibble_of_row(i8));
            zw_tile[kk * (kPackRows / 8) + c8] = wv;
        }
        __syncthreads();
    }

    // ---- codes and packed words: warp = 32 rows of one 64-column half,
    // lane = 2 columns of it
    const int64_t C = p.d_out / 8;
    {
        const int b = warp & 1;                   // which 64-column half (box)
        const int blk = warp >> 1;                // which 32-row block
        const int jt = 64 * b + 2 * lane;         // first tile column of the lane
        const int kk = jt / G;
        const int rb = blk * kRowsPerWarp;        // first row of the warp
        const unsigned char* box = tile + b * kBoxBytes + rb * 128 + (lane & 3) * 4;
        const int chunk = lane >> 2;              // 16-byte chunk (8 columns) of the row
        const float2 s01 = *reinterpret_cast<const float2*>(&s_tile[s_slot(jt)]);
        const float2* qr_row = qr_tile + kk * kRowStride + rb;
        const int* bad_row = bad_tile + kk * kRowStride + rb;
        const int* zero_row = zero_tile + kk * kRowStride + rb;
        // each nibble starts at (zero point - bits of 1.5*2^23); adding the
        // bits of the rounded quotient + 1.5*2^23 leaves the unsigned code
        uint32_t words[2][4];
#pragma unroll
        for (int hw = 0; hw < 4; ++hw) {
            const uint32_t init =
                kAsym ? zw_tile[kk * (kPackRows / 8) + rb / 8 + hw] - kRoundMagicBits * 0x11111111u
                      : 0u - (kRoundMagicBits - (uint32_t)p.zero_point) * 0x11111111u;
#pragma unroll
            for (int e = 0; e < 2; ++e) words[e][hw] = init;
        }
        if (kAsym || slow_blk[kk * kBlocks + blk] != 0)
            pack_rows<true, kAsym>(box, chunk, s01, qr_row, bad_row, zero_row, words);
        else
            pack_rows<false, kAsym>(box, chunk, s01, qr_row, bad_row, zero_row, words);
        const int64_t cw = row0 / 8 + rb / 8;      // first output word of the warp
        if (cw < C) {   // d_out % 8 == 0: each word is wholly inside or outside
            const bool four = cw + 3 < C;
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int64_t j = col0 + jt + e;
                if (j >= p.d_in) continue;
                int32_t* dst = p.qweight + j * C + cw;
                if (four && (((uintptr_t)dst & 15u) == 0)) {
                    *reinterpret_cast<uint4*>(dst) =
                        make_uint4(words[e][0], words[e][1], words[e][2], words[e][3]);
                } else {
#pragma unroll
                    for (int hw = 0; hw < 4; ++hw)
                        if (cw + hw < C) dst[hw] = (int32_t)words[e][hw];
                }
            }
        }
    }

    // ---- qzeros of the tile's groups and words
    uint32_t zword = (uint32_t)p.zero_point & 0xFu;
    zword *= 0x11111111u;
    for (int i = tid; i < KG * (kPackRows / 8); i += kPackThreads) {
        const int kk = i / (kPackRows / 8), cwl = i % (kPackRows / 8);
        const int64_t gk = col0 / G + kk, cw = row0 / 8 + cwl;
        if (gk * G < p.d_in && cw < C)
            p.qzeros[gk * C + cw] = (int32_t)(kAsym ? zw_tile[i] : zword);
    }
}

template <int G>
size_t pack_smem_bytes() {
    constexpr int KG = kPackCols / G;
    return 1024 /* alignment */ + kTileBytes + 2 * (kPackCols + 8) * sizeof(float) +
           (size_t)KG * kRowStride * (sizeof(float2) + 2 * sizeof(int)) +
           (size_t)KG * (kPackRows / kRowsPerWarp) * sizeof(int) +
           (size_t)KG * (kPackRows / 8) * sizeof(uint32_t) + 2 * sizeof(uint32_t) +
           sizeof(uint64_t);
}

template <int G>
cudaError_t launch_pack_G(const PackParams& p, cudaStream_t stream) {
    const size_t smem = pack_smem_bytes<G>();
    const bool asym = p.zero_point == AWQ_ZERO_POINT_ASYM;
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
    dim3 grid((unsigned)((p.d_in + kPackCols - 1) / kPackCols),
              (unsigned)((p.d_out + kPackRows - 1) / kPackRows));
    return launch_pdl(asym ? pack_kernel<G, true> : pack_kernel<G, false>, grid,
                      dim3(kPackThreads), smem, stream, p);
}

}  // namespace

cudaError_t pack_unit_flags(unsigned int* bits, bool clear) {
    return unit_device_flags(bits, clear);
}

cudaError_t launch_quantize_pack(const void* W, int64_t d_out, int64_t d_in, const float* s,
                                 const uint8_t* clip_idx, int group_size, int zero_point,
                                 int32_t* qweight, void* scales, int32_t* qzeros,
                                 cudaStream_t stream) {
    EncodeTiledFn encode = encode_tiled_fn();
    if (!encode) return cudaErrorNotSupported;
    PackParams p;
    std::memset(&p, 0, sizeof(p));
    const cuuint64_t gdim[2] = {(cuuint64_t)d_in, (cuuint64_t)d_out};
    const cuuint64_t gstride[1] = {(cuuint64_t)d_in * 2};
    const cuuint32_t box[2] = {(cuuint32_t)kBoxCols, (cuuint32_t)kPackRows};
    const cuuint32_t estride[2] = {1, 1};
    if (encode(&p.tmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(W), gdim, gstride,
               box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    p.d_out = d_out;
    p.d_in = d_in;
    p.s = s;
    p.clip_idx = clip_idx;
    p.zero_point = zero_point;
    p.qweight = qweight;
    p.scales = static_cast<__half*>(scales);
    p.qzeros = qzeros;
    switch (group_size) {
        case 32: return launch_pack_G<32>(p, stream);
        case 64: return launch_pack_G<64>(p, stream);
        case 128: return launch_pack_G<128>(p, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace awq
