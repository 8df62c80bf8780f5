// common.cuh -- device helpers shared by the sm_100a kernels of libawq_b200.
//
// Nothing here is shared with the CPU oracle; the two are written apart.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace awq {

// 1.5 * 2^23: adding it to |y| < 2^22 rounds y to an integer (ties to even)
// in the last place, because the sum's unit in the last place is 1.
constexpr float kRoundMagic = 12582912.0f;
constexpr uint32_t kRoundMagicBits = 0x4B400000u;
constexpr float kHalfMax = 65504.0f;             // largest finite fp16
constexpr float kHalfMinNormal = 6.103515625e-05f;  // 2^-14
constexpr float kFloatMinNormal = 1.17549435e-38f;  // 2^-126

// Host-visible error bits written into a workspace word by the kernels.
constexpr int kDevErrWaitTimeout = 1;

// Bound on any spin-wait of a pipeline: 2 seconds of %globaltimer.
constexpr uint64_t kWaitLimitNs = 2000000000ull;
// Bound on a drain wait: after a pipeline wait gave up, a CTA still waits for
// its own copies (or MMAs) in flight before it exits, so that none of them
// writes shared memory or TMEM that the CTA no longer owns.  Ten times the
// pipeline's limit: a copy that has not landed by then means the memory
// system is not making progress at all; the CTA then leaves with the timeout
// bit set, and its outputs are reported invalid.
constexpr uint64_t kDrainLimitNs = 20000000000ull;

// ------------------------------------------------------ sticky device flags
// Condition bits (AWQ_FLAG_* of awq.h) that kernels raise when they meet
// non-finite data or give up a bounded wait.  Each .cu file is its own device
// module (the library is built without relocatable device code), so each
// gets its own copy of this word; awq_last_device_flags() reads and clears
// every module's copy through the host accessor each file defines with
// unit_device_flags().  A raise is one atomic OR, taken only on those rare
// paths.
static __device__ unsigned int g_unit_flags;

__device__ __forceinline__ void raise_device_flag(unsigned int bits) {
    atomicOr(&g_unit_flags, bits);
}

// Host side: ORs this module's word into *bits and, if `clear`, zeroes it.
// Synchronous (cudaMemcpyFromSymbol / ToSymbol); the caller has synchronised
// the device first.
static inline cudaError_t unit_device_flags(unsigned int* bits, bool clear) {
    unsigned int v = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&v, g_unit_flags, sizeof v);
    if (e != cudaSuccess) return e;
    *bits |= v;
    if (clear && v) {
        const unsigned int zero = 0;
        e = cudaMemcpyToSymbol(g_unit_flags, &zero, sizeof zero);
    }
    return e;
}

__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ---------------------------------------------------------------- mbarrier

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;"
                 :: "r"(smem_addr(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_fence_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("{\n\t.reg .b64 st;\n\t"
                 "mbarrier.arrive.shared::cta.b64 st, [%0];\n\t}"
                 :: "r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("{\n\t.reg .b64 st;\n\t"
                 "mbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}"
                 :: "r"(smem_addr(bar)), "r"(bytes) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok) : "r"(smem_addr(bar)), "r"(parity) : "memory");
    return ok != 0;
}

// Wait for the phase with the given parity to complete; gives up after
// kWaitLimitNs and returns false (the caller reports the error and unwinds).
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (global_ns() - t0 > kWaitLimitNs) return false;
    }
    return true;
}

// A drain wait: the same, with the longer kDrainLimitNs.
__device__ __forceinline__ bool mbar_wait_drain(uint64_t* bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (global_ns() - t0 > kDrainLimitNs) return false;
    }
    return true;
}

// ------------------------------------------------- dependent launches
// Programmatic dependent launch: a kernel launched with the programmatic
// stream-serialisation attribute may start while its predecessor drains; it
// must call pdl_wait() before touching anything the predecessor writes (or
// anything it writes that the predecessor may still read).
__device__ __forceinline__ void pdl_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Approximate reciprocal (MUFU, <= 1 ulp); used only where an ulp cannot
// change a result beyond the documented tolerance.
__device__ __forceinline__ float rcp_approx(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// ---------------------------------------------------------------- TMA

// 2-D tiled bulk tensor load global -> shared, completion counted on `bar`.
// x is the innermost (contiguous) coordinate in elements.
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map,
                                            int32_t x, int32_t y, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];"
        :: "r"(smem_addr(dst)), "l"(reinterpret_cast<uint64_t>(map)),
           "r"(x), "r"(y), "r"(smem_addr(bar))
        : "memory");
}

// The same with an L2 cache policy (from make_l2_policy) attached to the reads.
__device__ __forceinline__ void tma_load_2d_hint(void* dst, const CUtensorMap* map, int32_t x,
                                                 int32_t y, uint64_t* bar, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        ".L2::cache_hint [%0], [%1, {%2, %3}], [%4], %5;"
        :: "r"(smem_addr(dst)), "l"(reinterpret_cast<uint64_t>(map)),
           "r"(x), "r"(y), "r"(smem_addr(bar)), "l"(policy)
        : "memory");
}

// L2 cache policies for tma_load_2d_hint: data read once (evict first) and
// data that later reads of the same kernel should still find (evict last).
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ uint64_t l2_policy_evict_last() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];"
                 :: "l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ---------------------------------------------------------------- numerics

// Round-to-nearest-even fp32 quotient m / 7 for finite m >= 0, from the
// rounded reciprocal c = RN(1/7) and one residual correction (the residual
// m - 7 q0 is exact in an FMA).  Equal to the IEEE quotient for every
// non-negative finite fp32 m: a GPU test compares all 2^31 of them with
// __fdiv_rn.  Values below 2^-100 take the IEEE division (their residual
// could be subnormal).
__device__ __forceinline__ float div7_rn(float m) {
    if (m < 0x1p-100f) return __fdiv_rn(m, 7.0f);
    const float c = 0.142857149f;            // RN(1/7) = 0x3E124925
    const float q0 = __fmul_rn(m, c);
    const float r = __fmaf_rn(-q0, 7.0f, m);
    return __fmaf_rn(r, c, q0);
}

// div7_rn without the guard for tiny m: equal to it for m >= 2^-100, and for
// smaller m a value below 2^-25, which rounds to the same fp16 value (zero).
// Used where only the fp16 rounding of the quotient matters; an infinite m
// gives NaN.
// The quotient a / b from y = RN(1 / b) with one residual correction, for
// the rounding decision rint(a / b) only: it can differ from the IEEE
// quotient by an ulp, which changes rint's result only within an ulp of a
// half-integer; there it agrees with rint(__fdiv_rn(a, b)) for every fp16
// divisor b and every a within 8 ulps of each half-integer multiple of b in
// [-16 b, 16 b] (checked on the GPU).  Two-wide: the same operations as
// __fmul2_rn / __ffma2_rn component by component.
__device__ __forceinline__ float2 quot_rcp1_2(float2 a, float2 nb, float2 y) {
    float2 q = __fmul2_rn(a, y);
    const float2 r = __ffma2_rn(q, nb, a);
    return __ffma2_rn(r, y, q);
}

// RN(m / 15) for finite m >= 0 (the asymmetric grid's scale): two residual
// corrections of m * RN(1/15); tiny m, where a residual could underflow,
// takes the IEEE division.  Checked against __fdiv_rn for every
// non-negative finite fp32 value.
__device__ __forceinline__ float div15_rn(float m) {
    if (m < 0x1p-100f) return __fdiv_rn(m, 15.0f);
    const float c = 0.0666666701f;           // RN(1/15) = 0x3D888889
    float q = __fmul_rn(m, c);
    float r = __fmaf_rn(-q, 15.0f, m);
    q = __fmaf_rn(r, c, q);
    r = __fmaf_rn(-q, 15.0f, m);
    return __fmaf_rn(r, c, q);
}
__device__ __forceinline__ float div7_rn_for_fp16(float m) {
    const float c = 0.142857149f;            // RN(1/7)
    const float q0 = __fmul_rn(m, c);
    const float r = __fmaf_rn(-q0, 7.0f, m);
    return __fmaf_rn(r, c, q0);
}

// Round-to-nearest-even fp32 quotient a / b from y = RN(1/b), for b an fp16
// value (positive, normal or subnormal) and |a / b| < 2^24: two residual
// corrections (P. Markstein, "Computation of elementary functions on the
// IBM RISC System/6000 processor", IBM J. Res. Dev. 34(1), 1990).  The
// first makes the quotient faithful, the second rounds it correctly.
// Checked against __fdiv_rn by a GPU test over every fp16 b.
__device__ __forceinline__ float div_rn_rcp(float a, float b, float y) {
    float q = __fmul_rn(a, y);
    float r = __fmaf_rn(-q, b, a);
    q = __fmaf_rn(r, y, q);
    r = __fmaf_rn(-q, b, a);
    return __fmaf_rn(r, y, q);
}

// RN(a / b) in fp64 from y = RN(1 / b): the product a*y is within about one
// ulp of the quotient and the residual a - q*b is exact in an FMA, so one
// correction q + r*y gives the correctly rounded quotient (Markstein's
// construction).  Used for |w| / max|w| of fp16 values, where it is exact
// for every pair of non-negative finite fp16 values with b > 0 (checked
// against __ddiv_rn for all of them, also in the scaled form below).
__device__ __forceinline__ double ddiv_rn_rcp(double a, double b, double y) {
    const double q = __dmul_rn(a, y);
    const double r = __fma_rn(-q, b, a);
    return __fma_rn(r, y, q);
}

// A non-negative finite fp32 value as an fp64 scaled by 2^-896: the fp32
// bits shifted right by 3 put its exponent field in the low bits of the fp64
// exponent field, so the result is exactly v * 2^(127 - 1023) (a normal
// fp64 for every nonzero fp32 value, and 0 for 0).  For quotients of fp16
// values both operands take the same scale: the scaled reciprocal of a
// divisor in [2^-24, 65504] stays normal and the residual of ddiv_rn_rcp
// stays exact, so the scaled quotient is the same number.
__device__ __forceinline__ double f32_scaled_f64(float v) {
    return __hiloint2double((int)(__float_as_uint(v) >> 3), 0);
}

// Group scale from the group's largest |w * s| (round-to-nearest-even
// throughout): fp32 quotient by 7, then fp16 unless fp32 scales are asked
// for.  An fp16 overflow is held at 65504; a non-finite maximum gives NaN.
// *exact_range is set when every |ws| / scale is known to be below 7.5, so
// that the code needs no clamp.
__device__ __forceinline__ float group_scale(float m, bool fp32_scale, bool* exact_range) {
    const float qsf = div7_rn(m);
    float qs;
    bool in_range;
    if (fp32_scale) {
        qs = qsf;
        in_range = qs >= kFloatMinNormal;
    } else {
        qs = __half2float(__float2half_rn(qsf));
        in_range = (qs >= kHalfMinNormal) && (qs <= kHalfMax);
        if (qs > kHalfMax) qs = kHalfMax;
    }
    if (!(m <= 3.402823466e38f)) qs = __int_as_float(0x7fc00000);
    *exact_range = in_range;
    return qs;
}

}  // namespace awq
