// output_error.cu -- optional output-space scoring of every grid point
//   err[i] = || X (W - W_hat_i)^T ||_F^2,   W_hat_i = Q(W * s_i) / s_i
// ("AWQ architecture, in depth", section "The scale search as code": the
// group's output after fake quantisation against the full-precision output;
// "Weight-Only Quantization: GPTQ and AWQ", section 2: the output error is
// X (W - W_hat)).
//
// The only dense contraction of the path, on the 5th-generation tensor
// cores.  Per grid point i (launched one after the other on the stream):
//   dw_builder_kernel  one warp per row of W: the same group fake
//                      quantisation as the search (exact fp16 q_scale, exact
//                      IEEE quotient by the corrected reciprocal), then
//                      dW = (w s - q q_scale) / s scaled by a per-row power
//                      of two c_r (no entry of a row falls into the fp16
//                      subnormal range; a bound on the row's largest |dW|
//                      maps it below 2^13) and written as an fp16 pair
//                      hi = fp16(dW c_r), lo = fp16(dW c_r - hi): the K axis
//                      of the product is [dW_hi | dW_lo] against [X | X], so
//                      the tensor cores see dW to ~22 bits, not 11;
//   oe_gemm_kernel     persistent, one CTA per SM, 18 warps: warp 0 issues
//                      TMA loads into a 5-stage mbarrier ring; a stage holds
//                      one 128x32 tile of X and the matching 256x32 tiles of
//                      dW hi and dW lo (64-byte swizzle), so every X tile
//                      feeds both halves and X crosses DRAM once per tile;
//                      one thread of warp 1 issues tcgen05.mma (kind::f16,
//                      M=128, N=256, K=16, fp32 accumulation in TMEM), four
//                      per stage (two K slices x hi, lo), and commits each
//                      stage back to the producer.  Output tiles go in
//                      groups of 8 row blocks of dW: all token blocks sweep
//                      one group before the next starts, the group's dW
//                      tiles (100 MB at 4096 x 12288) are read with an L2
//                      evict-last policy and X with evict-first, so dW
//                      crosses DRAM once per grid point and X once per group.  TMEM holds the MMA accumulator
//                      (columns 0-255) and a running sum (256-511).  Every 32
//                      K-blocks (2048 of K) warps 2-17 (four per TMEM lane
//                      quadrant, 64 columns each) drain the accumulator into
//                      the running sum with round-to-nearest fp32 additions
//                      (tcgen05.ld / st), so no accumulation chain inside the
//                      tensor core is longer than 128 MMAs (its accumulation
//                      does not round to nearest, and long chains drift
//                      towards zero).  The epilogue releases the accumulator
//                      as soon as it has read it, so the next segment's MMAs
//                      run while the running sum is updated.  At the end of a tile each column is
//                      multiplied by 1/c_r (exact) and the squares summed.
//                      X dW^T is never written out.
// A final kernel sums the per-CTA partials of every grid point in a fixed
// order (fp64) and picks the first minimum.
#include <cstring>

#include "common.cuh"
#include "internal.h"

namespace awq {
namespace {

// ----------------------------------------------------------- tile shape
constexpr int kBM = 128;                    // tokens per tile (TMEM lanes)
constexpr int kBN = 256;                    // output rows per tile (TMEM columns)
constexpr int kBK = 32;                     // 32 fp16 = 64 bytes: one swizzle row
constexpr int kUmmaK = 16;                  // K of one kind::f16 MMA
constexpr int kStages = 5;
constexpr int kABytes = kBM * kBK * 2;      // 8 KB of X
constexpr int kBBytes = kBN * kBK * 2;      // 16 KB of dW hi (and as much of dW lo)
constexpr int kStageBytes = kABytes + 2 * kBBytes;   // 40 KB
constexpr int kGroupN = 8;                  // dW row blocks per raster group
constexpr int kTmemCols = 2 * kBN;          // accumulator + running sum
constexpr int kEpiWarps = 16;               // four per TMEM lane quadrant
constexpr int kEpiCols = kBN / (kEpiWarps / 4);   // accumulator columns per epilogue warp
constexpr int kGemmThreads = 32 * (2 + kEpiWarps);   // producer, MMA, epilogue
constexpr int kSegBlocks = 32;              // K-blocks (x 4 MMAs) accumulated per drain
constexpr int kMaxOeCtas = 1024;
constexpr int kMaxGridOe = 32;

// UMMA instruction descriptor for kind::f16: fp32 accumulator (bits 4-5 = 1),
// A and B fp16 (format 0), both K-major, N >> 3 at bit 17, M >> 4 at bit 24.
constexpr uint32_t kIdesc = (1u << 4) | ((uint32_t)(kBN >> 3) << 17) |
                            ((uint32_t)(kBM >> 4) << 24);

// Shared-memory matrix descriptor of a K-major tile written by TMA with the
// 64-byte swizzle (rows of 64 bytes, 16-byte chunks XOR-permuted within each
// 4-chunk row by the row's bits): start address >> 4 (bits 0-13), leading
// byte offset (unused for this layout; 1), stride byte offset = 512 bytes
// between 8-row groups (bits 32-45), descriptor version 1 (bits 46-47),
// layout 64B-swizzle = 4 (bits 61-63).  The second K=16 slice of a row
// starts 32 bytes further (the swizzle is applied to the final address).
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr) {
    uint64_t d = (uint64_t)((addr >> 4) & 0x3FFFu);
    d |= (uint64_t)1u << 16;
    d |= (uint64_t)(512u >> 4) << 32;
    d |= (uint64_t)1u << 46;
    d |= (uint64_t)4u << 61;
    return d;
}

// Output tile t of the raster: groups of kGroupN dW row blocks; within a
// group the token block advances slowest, so the CTAs working at one time
// share the group's dW tiles and each X tile.
__device__ __forceinline__ void tile_mn(int t, int m_blocks, int n_blocks, int* m, int* n) {
    const int per_group = kGroupN * m_blocks;
    const int g = t / per_group;
    const int local = t - g * per_group;
    const int ng = min(kGroupN, n_blocks - g * kGroupN);
    *m = local / ng;
    *n = g * kGroupN + local % ng;
}

__device__ __forceinline__ void umma_f16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                         uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        :: "r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(kIdesc), "r"(accumulate) : "memory");
}

__device__ __forceinline__ void umma_commit(uint64_t* bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
        :: "r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// 16 consecutive fp32 columns of this warp's 32 TMEM lanes.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float* v) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
          "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]),
          "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// Store 16 fp32 columns into this warp's 32 TMEM lanes (then wait for it).
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float* v) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
        :: "r"(taddr), "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])),
           "r"(__float_as_uint(v[2])), "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])),
           "r"(__float_as_uint(v[5])), "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])),
           "r"(__float_as_uint(v[8])), "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])),
           "r"(__float_as_uint(v[11])), "r"(__float_as_uint(v[12])),
           "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
           "r"(__float_as_uint(v[15]))
        : "memory");
}

__device__ __forceinline__ void tmem_wait_st() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

struct GemmParams {
    CUtensorMap tmA;        // X  fp16 [T, d_in], box {32, 128}, 64B swizzle
    CUtensorMap tmB;        // dW fp16 [d_out, 2 d_in] (hi | lo), box {32, 256}, 64B swizzle
    int32_t m_blocks, n_blocks, k_blocks;   // k_blocks of X (and of each dW half)
    int32_t d_in;
    int32_t alpha, n_grid;
    int64_t d_out;
    const float* inv_c;     // [d_out] 1 / c_r of this grid point
    double* partial;        // [gridDim.x][n_grid]
    int* dev_err;
};

// Bounded wait that also gives up at once when another role of the CTA has
// already given up (so a broken pipeline ends in one timeout, not one per
// tile).
__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity,
                                              volatile int* abort_flag, int* dev_err) {
    if (*abort_flag) return false;
    if (mbar_wait_bounded(bar, parity)) return true;
    *abort_flag = 1;
    atomicOr(dev_err, kDevErrWaitTimeout);
    return false;
}

__global__ void __maxnreg__(96)
oe_gemm_kernel(const __grid_constant__ GemmParams p) {
    extern __shared__ unsigned char smem_raw[];
    // the 128-byte swizzle atoms want 1024-byte aligned stages
    const uint32_t raw = smem_addr(smem_raw);
    unsigned char* smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
    unsigned char* stages = smem;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
    uint64_t* empty = full + kStages;
    uint64_t* tfull = empty + kStages;       // accumulator ready (MMA -> epilogue)
    uint64_t* tempty = tfull + 2;            // accumulator drained (epilogue -> MMA)
    uint64_t* drain = tempty + 2;            // all issued MMAs done (abort path)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    double* red = reinterpret_cast<double*>(tmem_slot + 4);   // [kEpiWarps]

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n_tiles = p.m_blocks * p.n_blocks;

    if (tid == 0) {
        *abort_flag = 0;
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {   // [0]: segment in TMEM / segment drained
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], kEpiWarps);
        }
        mbar_init(drain, 1);
        mbar_fence_init();
        tma_prefetch_desc(&p.tmA);
        tma_prefetch_desc(&p.tmB);
    }
    if (warp == 1) {   // the whole warp allocates the accumulators
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     :: "r"(smem_addr(tmem_slot)), "r"(kTmemCols) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        // ---------------------------------------------------- TMA producer
        if (lane == 0) {
            const uint64_t pol_x = l2_policy_evict_first(), pol_dw = l2_policy_evict_last();
            uint32_t it = 0;
            uint32_t issued[kStages] = {};
            for (int t = blockIdx.x; t < n_tiles && !*abort_flag; t += gridDim.x) {
                int m_blk, n_blk;
                tile_mn(t, p.m_blocks, p.n_blocks, &m_blk, &n_blk);
                for (int kb = 0; kb < p.k_blocks; ++kb, ++it) {
                    const int s = it % kStages;
                    const uint32_t use = it / kStages;
                    if (use > 0 && !wait_or_abort(&empty[s], (use - 1) & 1u, abort_flag, p.dev_err))
                        break;
                    unsigned char* a = stages + s * kStageBytes;
                    mbar_arrive_expect_tx(&full[s], kStageBytes);
                    tma_load_2d_hint(a, &p.tmA, kb * kBK, m_blk * kBM, &full[s], pol_x);
                    tma_load_2d_hint(a + kABytes, &p.tmB, kb * kBK, n_blk * kBN, &full[s], pol_dw);
                    tma_load_2d_hint(a + kABytes + kBBytes, &p.tmB, p.d_in + kb * kBK, n_blk * kBN,
                                     &full[s], pol_dw);
                    ++issued[s];
                }
            }
            if (*abort_flag) {   // leave no TMA copy writing this CTA's shared memory
                for (int s = 0; s < kStages; ++s)
                    if (issued[s] > 0 && !mbar_wait_drain(&full[s], (issued[s] - 1) & 1u))
                        atomicOr(p.dev_err, kDevErrWaitTimeout);
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------- MMA issuer
        if (lane == 0) {
            uint32_t it = 0, seg = 0;
            const int kb_total = p.k_blocks;
            for (int t = blockIdx.x; t < n_tiles && !*abort_flag; t += gridDim.x) {
                bool ok = true;
                for (int kb0 = 0; kb0 < kb_total && ok; kb0 += kSegBlocks, ++seg) {
                    // the epilogue has drained the previous segment
                    if (seg > 0 &&
                        !wait_or_abort(&tempty[0], (seg - 1) & 1u, abort_flag, p.dev_err)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const int kb1 = min(kb_total, kb0 + kSegBlocks);
                    for (int kb = kb0; kb < kb1; ++kb, ++it) {
                        const int s = it % kStages;
                        if (!wait_or_abort(&full[s], (it / kStages) & 1u, abort_flag,
                                           p.dev_err)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t a = smem_addr(stages + s * kStageBytes);
                        const uint32_t bh = a + kABytes, bl = bh + kBBytes;
#pragma unroll
                        for (int k = 0; k < kBK / kUmmaK; ++k) {
                            // X times dW hi, then the same X times dW lo
                            umma_f16(tmem_base, smem_desc(a + k * kUmmaK * 2),
                                     smem_desc(bh + k * kUmmaK * 2),
                                     (kb > kb0 || k > 0) ? 1u : 0u);
                            umma_f16(tmem_base, smem_desc(a + k * kUmmaK * 2),
                                     smem_desc(bl + k * kUmmaK * 2), 1u);
                        }
                        umma_commit(&empty[s]);   // stage free once these MMAs are done
                    }
                    if (ok) umma_commit(&tfull[0]);   // this K segment is in TMEM
                }
                if (!ok) break;
            }
            if (*abort_flag) {   // no MMA may still write TMEM when it is freed
                umma_commit(drain);
                if (!mbar_wait_drain(drain, 0)) atomicOr(p.dev_err, kDevErrWaitTimeout);
            }
        }
    } else {
        // ---------------------------------------------------- epilogue
        const int q = warp & 3;                 // TMEM lane quadrant of this warp
        const int h = (warp - 2) / 4;           // which kEpiCols-wide slice of the columns
        const int kb_total = p.k_blocks;
        const int segs = (kb_total + kSegBlocks - 1) / kSegBlocks;
        const uint32_t lane_base = (uint32_t)(q * 32) << 16;
        const uint32_t acc_addr = tmem_base + lane_base + (uint32_t)(h * kEpiCols);
        const uint32_t run_addr = acc_addr + (uint32_t)kBN;
        double acc = 0.0;
        uint32_t seg = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
            for (int sg = 0; sg < segs; ++sg, ++seg) {
                ok = __all_sync(0xffffffffu,
                                wait_or_abort(&tfull[0], seg & 1u, abort_flag, p.dev_err));
                if (!ok) break;
                tc_fence_after();
                // read the whole accumulator slice, then let the MMAs refill it
                float a[kEpiCols];
#pragma unroll
                for (int c0 = 0; c0 < kEpiCols; c0 += 16) tmem_ld16(acc_addr + (uint32_t)c0, a + c0);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&tempty[0]);
                // the running sum (columns the MMAs do not write) meanwhile
#pragma unroll
                for (int c0 = 0; c0 < kEpiCols; c0 += 16) {
                    float v[16];
                    if (sg > 0) {
                        tmem_ld16(run_addr + (uint32_t)c0, v);
#pragma unroll
                        for (int i = 0; i < 16; ++i) v[i] = __fadd_rn(a[c0 + i], v[i]);
                    } else {
#pragma unroll
                        for (int i = 0; i < 16; ++i) v[i] = a[c0 + i];
                    }
                    tmem_st16(run_addr + (uint32_t)c0, v);
                }
                tmem_wait_st();
            }
            if (!ok) break;
            // the running sum holds this tile's slice of X dW^T
            int m_blk, n_blk;
            tile_mn(t, p.m_blocks, p.n_blocks, &m_blk, &n_blk);
            const int64_t n0 = (int64_t)n_blk * kBN + h * kEpiCols;
            float s0 = 0.f, s1 = 0.f;
#pragma unroll 1
            for (int c0 = 0; c0 < kEpiCols; c0 += 16) {
                float v[16];
                tmem_ld16(run_addr + (uint32_t)c0, v);
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int64_t n = n0 + c0 + i;
                    const float y = v[i] * (n < p.d_out ? __ldg(p.inv_c + n) : 0.f);
                    if (i & 1) s1 = fmaf(y, y, s1); else s0 = fmaf(y, y, s0);
                }
            }
            acc += (double)(s0 + s1);
        }
        // fixed-order reduction: lanes, then the epilogue warps
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (lane == 0) red[warp - 2] = acc;
    }
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
        double v = 0.0;
        for (int i = 0; i < kEpiWarps; ++i) v += red[i];
        p.partial[(int64_t)blockIdx.x * p.n_grid + p.alpha] = v;
    }
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;"
                     :: "r"(tmem_base), "r"(kTmemCols) : "memory");
    }
}

// ------------------------------------------------------------ dW builder
// One warp per row of W; lane l takes 16-byte chunks l, l + 32, ... of the
// row, so a group of g channels is g/8 consecutive lanes.
template <int G>
__device__ __forceinline__ float seg_max(float v) {
#pragma unroll
    for (int o = 1; o < G / 8; o <<= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
template <int G>
__device__ __forceinline__ float seg_min(float v) {
#pragma unroll
    for (int o = 1; o < G / 8; o <<= 1) v = fminf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// kAsym: the asymmetric grid (AWQ_ASYMMETRIC), as the search and the pack
// take it: range = max(max ws - min ws, 1e-5), q_scale = fp16(range / 15),
// zero = clamp(rint(-min ws / q_scale), 0, 15), q = clamp(rint(ws / q_scale)
// + zero, 0, 15) with exact quotients, and W - W_hat = (ws - (q - zero)
// q_scale) / s.  |ws - (q - zero) q_scale| <= 3 max |ws| as in the symmetric
// grid, so the row bound of pass 1 holds for both.
template <int G, bool kAsym>
__global__ void __launch_bounds__(256)
dw_builder_kernel(const uint4* __restrict__ W, int64_t d_out, int64_t d_in,
                  const float* __restrict__ S, const float* __restrict__ inv_s,
                  int fp32_scale, __half* __restrict__ dW, float* __restrict__ inv_c) {
    pdl_wait();
    const int lane = threadIdx.x & 31;
    const int64_t r = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (r >= d_out) return;
    const int64_t chunks = d_in / 8;
    const uint4* wrow = W + r * chunks;
    const float4* S4 = reinterpret_cast<const float4*>(S);
    const float4* I4 = reinterpret_cast<const float4*>(inv_s);

    // pass 1: a bound on max |dW| of the row: per group 3 max|ws| max(1/s).
    // Every lane runs the same trips (the shuffles need the whole warp); a
    // group's g/8 chunks are consecutive lanes, all active or all inactive.
    float bound = 0.f;
    for (int64_t base = 0; base < chunks; base += 32) {
        const int64_t c = base + lane;
        const bool act = c < chunks;
        const uint4 v = act ? __ldg(wrow + c) : make_uint4(0, 0, 0, 0);
        const float4 z4 = make_float4(0.f, 0.f, 0.f, 0.f);
        const float4 sa = act ? __ldg(S4 + 2 * c) : z4, sb = act ? __ldg(S4 + 2 * c + 1) : z4;
        const float4 ia = act ? __ldg(I4 + 2 * c) : z4, ib = act ? __ldg(I4 + 2 * c + 1) : z4;        const uint32_t hw[4] = {v.x, v.y, v.z, v.w};
        const float sv[8] = {sa.x, sa.y, sa.z, sa.w, sb.x, sb.y, sb.z, sb.w};
        float m = 0.f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 w = __half22float2(*reinterpret_cast<const __half2*>(&hw[i]));
            m = fmaxf(m, fmaxf(fabsf(w.x * sv[2 * i]), fabsf(w.y * sv[2 * i + 1])));
        }
        float is = fmaxf(fmaxf(fmaxf(ia.x, ia.y), fmaxf(ia.z, ia.w)),
                         fmaxf(fmaxf(ib.x, ib.y), fmaxf(ib.z, ib.w)));
        m = seg_max<G>(m);
        is = seg_max<G>(is);
        bound = fmaxf(bound, 3.0f * m * is);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) bound = fmaxf(bound, __shfl_xor_sync(0xffffffffu, bound, o));
    // c_r = 2^(12 - E) with bound < 2^(E + 1): the row's |dW| c_r stays below 2^13
    int e = 0;
    if (bound > 0.f && bound <= 3.402823466e38f) e = ((__float_as_int(bound) >> 23) & 0xff) - 127;
    e = max(-100, min(100, e));
    const float c = __int_as_float((127 + 12 - e) << 23);
    if (lane == 0) inv_c[r] = __int_as_float((127 - 12 + e) << 23);

    // pass 2: the fake quantisation and the scaled fp16 pair (hi, lo) of dW
    uint4* drow_hi = reinterpret_cast<uint4*>(dW + r * 2 * d_in);
    uint4* drow_lo = reinterpret_cast<uint4*>(dW + r * 2 * d_in + d_in);
    for (int64_t base = 0; base < chunks; base += 32) {
        const int64_t ch = base + lane;
        const bool act = ch < chunks;
        const float4 z4 = make_float4(0.f, 0.f, 0.f, 0.f);
        const uint4 v = act ? __ldg(wrow + ch) : make_uint4(0, 0, 0, 0);
        const float4 sa = act ? __ldg(S4 + 2 * ch) : z4, sb = act ? __ldg(S4 + 2 * ch + 1) : z4;
        const float4 ia = act ? __ldg(I4 + 2 * ch) : z4, ib = act ? __ldg(I4 + 2 * ch + 1) : z4;        const uint32_t hw[4] = {v.x, v.y, v.z, v.w};
        const float sv[8] = {sa.x, sa.y, sa.z, sa.w, sb.x, sb.y, sb.z, sb.w};
        const float iv[8] = {ia.x, ia.y, ia.z, ia.w, ib.x, ib.y, ib.z, ib.w};
        float ws[8];
        float m = 0.f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 w = __half22float2(*reinterpret_cast<const __half2*>(&hw[i]));
            ws[2 * i] = __fmul_rn(w.x, sv[2 * i]);
            ws[2 * i + 1] = __fmul_rn(w.y, sv[2 * i + 1]);
            m = fmaxf(m, fmaxf(fabsf(ws[2 * i]), fabsf(ws[2 * i + 1])));
        }
        float qs, rq, zf = 0.f;
        if (kAsym) {
            float mx = ws[0], mn = ws[0];
#pragma unroll
            for (int i = 1; i < 8; ++i) {
                mx = fmaxf(mx, ws[i]);
                mn = fminf(mn, ws[i]);
            }
            mx = seg_max<G>(mx);
            mn = seg_min<G>(mn);
            const float range = fmaxf(__fsub_rn(mx, mn), 1e-5f);
            qs = div15_rn(range);
            if (!fp32_scale) qs = fminf(__half2float(__float2half_rn(qs)), kHalfMax);
            rq = __frcp_rn(qs);
            zf = fminf(fmaxf(rintf(div_rn_rcp(-mn, qs, rq)), 0.f), 15.f);
            // a NaN or infinite ws makes its own d, and so the error, non-finite
        } else {
            m = seg_max<G>(m);
            bool in_range;
            qs = group_scale(m, fp32_scale != 0, &in_range);
            rq = (qs > 0.f) ? __frcp_rn(qs) : 0.f;
        }
        uint32_t out[4], out_lo[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float d2[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const float a = ws[2 * i + h];
                float q;
                if (kAsym) {
                    float t = __fadd_rn(__fadd_rn(div_rn_rcp(a, qs, rq), kRoundMagic), zf);
                    t = fminf(fmaxf(t, kRoundMagic), kRoundMagic + 15.f);
                    q = __fsub_rn(__fadd_rn(t, -kRoundMagic), zf);   // level q - zero
                } else {
                    const float y = (qs > 0.f) ? div_rn_rcp(a, qs, rq) : 0.f;
                    float t = __fadd_rn(y, kRoundMagic);
                    t = fminf(fmaxf(t, kRoundMagic - 7.f), kRoundMagic + 7.f);
                    q = __fadd_rn(t, -kRoundMagic);
                }
                const float d = __fmaf_rn(-q, qs, a);          // (w - w_hat) * s
                d2[h] = __fmul_rn(__fmul_rn(d, iv[2 * i + h]), c);
            }
            const __half2 hv = __floats2half2_rn(d2[0], d2[1]);
            const float2 hf = __half22float2(hv);
            const __half2 lv = __floats2half2_rn(__fsub_rn(d2[0], hf.x), __fsub_rn(d2[1], hf.y));
            out[i] = *reinterpret_cast<const uint32_t*>(&hv);
            out_lo[i] = *reinterpret_cast<const uint32_t*>(&lv);
        }
        if (act) {
            drow_hi[ch] = make_uint4(out[0], out[1], out[2], out[3]);
            drow_lo[ch] = make_uint4(out_lo[0], out_lo[1], out_lo[2], out_lo[3]);
        }
    }
}

struct OeWs {
    float* S;
    float* inv_s;
    double* partial;
    int* dev_words;
    __half* dW;
    float* inv_c;
};

size_t dw_bytes(int64_t d_out, int64_t d_in) {
    return align_up((size_t)d_out * (size_t)d_in * 2 * 2, kWsAlign);   // hi and lo
}

OeWs carve_oe_ws(void* ws, int64_t d_out, int64_t d_in, int n_grid) {
    char* p = static_cast<char*>(ws);
    OeWs w;
    const size_t tab = align_up((size_t)n_grid * (size_t)d_in * sizeof(float), kWsAlign);
    w.S = reinterpret_cast<float*>(p);
    w.inv_s = reinterpret_cast<float*>(p + tab);
    p += 2 * tab;
    w.partial = reinterpret_cast<double*>(p);
    p += align_up((size_t)kMaxOeCtas * kMaxGridOe * sizeof(double), kWsAlign);
    w.dev_words = reinterpret_cast<int*>(p);
    p += kWsAlign;
    w.inv_c = reinterpret_cast<float*>(p);
    p += align_up((size_t)d_out * sizeof(float), kWsAlign);
    w.dW = reinterpret_cast<__half*>(p);
    return w;
}

template <int G>
cudaError_t launch_builder(const void* W, int64_t d_out, int64_t d_in, const float* S,
                           const float* inv_s, int flags, __half* dW, float* inv_c,
                           cudaStream_t st) {
    const dim3 grid((unsigned)((d_out + 7) / 8));
    return launch_pdl((flags & AWQ_ASYMMETRIC) ? dw_builder_kernel<G, true>
                                               : dw_builder_kernel<G, false>,
                      grid, dim3(256), 0, st,
                      static_cast<const uint4*>(W), d_out, d_in, S, inv_s,
                      (int)((flags & AWQ_SCALE_FP32) != 0), dW, inv_c);
}

}  // namespace

size_t output_error_workspace(int64_t T, int64_t d_out, int64_t d_in, int group_size,
                              int n_grid) {
    (void)T;
    (void)group_size;
    const size_t tab = align_up((size_t)n_grid * (size_t)d_in * sizeof(float), kWsAlign);
    return 2 * tab + align_up((size_t)kMaxOeCtas * kMaxGridOe * sizeof(double), kWsAlign) +
           kWsAlign + align_up((size_t)d_out * sizeof(float), kWsAlign) + dw_bytes(d_out, d_in);
}

awq_status launch_output_error(const void* X, int64_t T, const void* W, int64_t d_out,
                               int64_t d_in, const float* x_mean, int group_size, int n_grid,
                               int flags, double* err, int32_t* best_idx, float* s_best,
                               void* ws, cudaStream_t stream) {
    DeviceInfo dev;
    if (query_device(&dev) != cudaSuccess) return AWQ_ERR_CUDA;
    EncodeTiledFn encode = encode_tiled_fn();
    if (!encode) return AWQ_ERR_CUDA;
    OeWs w = carve_oe_ws(ws, d_out, d_in, n_grid);

    GemmParams p;
    std::memset(&p, 0, sizeof(p));
    {
        const cuuint64_t gdim[2] = {(cuuint64_t)d_in, (cuuint64_t)T};
        const cuuint64_t gstride[1] = {(cuuint64_t)d_in * 2};
        const cuuint32_t box[2] = {(cuuint32_t)kBK, (cuuint32_t)kBM};
        const cuuint32_t es[2] = {1, 1};
        if (encode(&p.tmA, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(X), gdim,
                   gstride, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return AWQ_ERR_CUDA;
    }
    {
        const cuuint64_t gdim[2] = {(cuuint64_t)(2 * d_in), (cuuint64_t)d_out};
        const cuuint64_t gstride[1] = {(cuuint64_t)d_in * 2 * 2};
        const cuuint32_t box[2] = {(cuuint32_t)kBK, (cuuint32_t)kBN};
        const cuuint32_t es[2] = {1, 1};
        if (encode(&p.tmB, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, w.dW, gdim, gstride, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return AWQ_ERR_CUDA;
    }
    p.m_blocks = (int32_t)((T + kBM - 1) / kBM);
    p.n_blocks = (int32_t)((d_out + kBN - 1) / kBN);
    p.k_blocks = (int32_t)(d_in / kBK);
    p.d_in = (int32_t)d_in;
    p.n_grid = n_grid;
    p.d_out = d_out;
    p.inv_c = w.inv_c;
    p.partial = w.partial;
    p.dev_err = w.dev_words;
    const int64_t tiles = (int64_t)p.m_blocks * p.n_blocks;
    int grid = (int)std::min<int64_t>(tiles, std::min<int64_t>(dev.num_sms, kMaxOeCtas));

    const size_t smem = (size_t)kStages * kStageBytes + 1024 /*alignment*/ + 512;
    static int configured[64] = {};
    if (dev.device >= 0 && dev.device < 64 && !configured[dev.device]) {
        if (note_cuda(cudaFuncSetAttribute(oe_gemm_kernel,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem),
                      "oe_gemm smem attribute") != cudaSuccess)
            return AWQ_ERR_CUDA;
        configured[dev.device] = 1;
    }

    if (note_cuda(launch_scale_table(x_mean, d_in, n_grid, w.S, w.inv_s, w.dev_words,
                                     dev.num_sms, stream, kTableInverse),
                  "scale table launch") != cudaSuccess)
        return AWQ_ERR_CUDA;
    for (int a = 0; a < n_grid; ++a) {
        cudaError_t e;
        const float* Sa = w.S + (int64_t)a * d_in;
        const float* Ia = w.inv_s + (int64_t)a * d_in;
        switch (group_size) {
            case 32: e = launch_builder<32>(W, d_out, d_in, Sa, Ia, flags, w.dW, w.inv_c, stream); break;
            case 64: e = launch_builder<64>(W, d_out, d_in, Sa, Ia, flags, w.dW, w.inv_c, stream); break;
            case 128: e = launch_builder<128>(W, d_out, d_in, Sa, Ia, flags, w.dW, w.inv_c, stream); break;
            default: return AWQ_ERR_UNSUPPORTED;
        }
        if (note_cuda(e, "dw_builder launch") != cudaSuccess) return AWQ_ERR_CUDA;
        p.alpha = a;
        oe_gemm_kernel<<<grid, kGemmThreads, smem, stream>>>(p);
        if (note_cuda(cudaGetLastError(), "oe_gemm launch") != cudaSuccess) return AWQ_ERR_CUDA;
    }
    if (note_cuda(launch_finalize(w.partial, grid, n_grid, w.S, d_in, w.dev_words, err,
                                  best_idx, s_best, stream),
                  "finalize launch") != cudaSuccess)
        return AWQ_ERR_CUDA;
    return AWQ_OK;
}

}  // namespace awq
