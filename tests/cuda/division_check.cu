// Test-only kernels: compare the library's division helpers (common.cuh)
// with the IEEE round-to-nearest division __fdiv_rn.  Built by
// tests/test_gpu_division.py into a scratch shared library.
#include "common.cuh"

// every non-negative finite fp32 bit pattern in [lo, hi)
__global__ void check_div7(uint32_t lo, uint32_t hi, unsigned long long* bad,
                           uint32_t* first_bad) {
    for (uint64_t i = lo + blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; i < hi;
         i += (uint64_t)gridDim.x * blockDim.x) {
        const float m = __uint_as_float((uint32_t)i);
        const float a = awq::div7_rn(m);
        const float b = __fdiv_rn(m, 7.0f);
        if (__float_as_uint(a) != __float_as_uint(b)) {
            atomicAdd(bad, 1ull);
            atomicMin(first_bad, (uint32_t)i);
        }
    }
}

// every non-negative finite fp32 bit pattern in [lo, hi): m / 15
__global__ void check_div15(uint32_t lo, uint32_t hi, unsigned long long* bad,
                            uint32_t* first_bad) {
    for (uint64_t i = lo + blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; i < hi;
         i += (uint64_t)gridDim.x * blockDim.x) {
        const float m = __uint_as_float((uint32_t)i);
        const float a = awq::div15_rn(m);
        const float b = __fdiv_rn(m, 15.0f);
        if (__float_as_uint(a) != __float_as_uint(b)) {
            atomicAdd(bad, 1ull);
            atomicMin(first_bad, (uint32_t)i);
        }
    }
}

// for every positive finite fp16 divisor b (blockIdx.x selects it), numerators
// a near every half-integer multiple of b in [-16b, 16b] (+-8 ulps) and a
// stride of other values
__global__ void check_div_rcp(unsigned long long* bad, uint32_t* first_bad_b) {
    const uint32_t hb = blockIdx.x + 1;           // 0x0001 .. 0x7bff
    const float b = __half2float(__ushort_as_half((unsigned short)hb));
    const float y = __frcp_rn(b);
    for (int t = threadIdx.x; t < 32 * 17 * 2 + 4096; t += blockDim.x) {
        float a;
        if (t < 32 * 17 * 2) {
            const int k = t / 34, d = (t % 34) / 2, sgn = t & 1;
            const float base = __fmul_rn((float)(k - 16) + 0.5f, b);
            a = __uint_as_float(__float_as_uint(base) + (uint32_t)(d - 8));
            if (sgn) a = -a;
        } else {
            const int u = t - 32 * 17 * 2;
            a = __fmul_rn(b, ((float)u - 2048.0f) * (15.5f / 2048.0f) + 1e-3f * (float)(u & 7));
        }
        if (!(fabsf(a) <= 3.0e38f)) continue;
        const float q = awq::div_rn_rcp(a, b, y);
        const float r = __fdiv_rn(a, b);
        if (__float_as_uint(q) != __float_as_uint(r)) {
            atomicAdd(bad, 1ull);
            atomicMin(first_bad_b, hb);
        }
    }
}

// every pair (a, b) of non-negative finite fp16 values with b > 0 (blockIdx.x
// selects b): ddiv_rn_rcp against the IEEE fp64 quotient __ddiv_rn, both on
// the plain fp64 values and in the form the weight-mean kernel uses (both
// operands scaled by 2^-896 through f32_scaled_f64, the reciprocal of the
// scaled divisor)
__global__ void check_ddiv_rcp(unsigned long long* bad, uint32_t* first_bad_b) {
    const uint32_t hb = blockIdx.x + 1;           // 0x0001 .. 0x7bff
    const float bf = __half2float(__ushort_as_half((unsigned short)hb));
    const double b = (double)bf;
    const double y = __drcp_rn(b);
    const double bs = awq::f32_scaled_f64(bf);
    const double ys = __drcp_rn(bs);
    for (uint32_t ha = threadIdx.x; ha <= 0x7bffu; ha += blockDim.x) {
        const float af = __half2float(__ushort_as_half((unsigned short)ha));
        const double r = __ddiv_rn((double)af, b);
        const double q = awq::ddiv_rn_rcp((double)af, b, y);
        const double qs = awq::ddiv_rn_rcp(awq::f32_scaled_f64(af), bs, ys);
        if (__double_as_longlong(q) != __double_as_longlong(r) ||
            __double_as_longlong(qs) != __double_as_longlong(r)) {
            atomicAdd(bad, 1ull);
            atomicMin(first_bad_b, hb);
        }
    }
}

// for every positive finite fp16 divisor b, numerators around every
// half-integer multiple of b in [-16b, 16b] (+-8 ulps): the rounding decision
// of the one-correction quotient (pack's codes) against rint(__fdiv_rn)
__global__ void check_code_rcp1(unsigned long long* bad, uint32_t* first_bad_b) {
    const uint32_t hb = blockIdx.x + 1;           // 0x0001 .. 0x7bff
    const float b = __half2float(__ushort_as_half((unsigned short)hb));
    const float y = __frcp_rn(b);
    for (int t = threadIdx.x; t < 32 * 17 * 2; t += blockDim.x) {
        const int k = t / 34, d = (t % 34) / 2, sgn = t & 1;
        const float base = __fmul_rn((float)(k - 16) + 0.5f, b);
        float a = __uint_as_float(__float_as_uint(base) + (uint32_t)(d - 8));
        if (sgn) a = -a;
        if (!(fabsf(a) <= 3.0e38f)) continue;
        const float2 q = awq::quot_rcp1_2(make_float2(a, a), make_float2(-b, -b),
                                          make_float2(y, y));
        if (__float_as_uint(rintf(q.x)) != __float_as_uint(rintf(__fdiv_rn(a, b)))) {
            atomicAdd(bad, 1ull);
            atomicMin(first_bad_b, hb);
        }
    }
}

extern "C" int run_checks(unsigned long long* out) {
    // out[0]: div7 mismatches, out[1]: first bad bits, out[2]: div_rcp
    // mismatches, out[3]: first bad fp16 divisor, out[4]: ddiv_rcp
    // mismatches, out[5]: its first bad fp16 divisor, out[6]: div15
    // mismatches, out[7]: first bad bits, out[8]: one-correction code
    // decision mismatches, out[9]: its first bad fp16 divisor
    unsigned long long* d_bad;
    uint32_t* d_first;
    if (cudaMalloc(&d_bad, 5 * sizeof(unsigned long long)) != cudaSuccess) return 1;
    if (cudaMalloc(&d_first, 5 * sizeof(uint32_t)) != cudaSuccess) return 1;
    cudaMemset(d_bad, 0, 5 * sizeof(unsigned long long));
    cudaMemset(d_first, 0xff, 5 * sizeof(uint32_t));
    check_div7<<<4096, 256>>>(0u, 0x7f800000u, d_bad, d_first);
    check_div_rcp<<<0x7bff, 256>>>(d_bad + 1, d_first + 1);
    check_ddiv_rcp<<<0x7bff, 256>>>(d_bad + 2, d_first + 2);
    check_div15<<<4096, 256>>>(0u, 0x7f800000u, d_bad + 3, d_first + 3);
    check_code_rcp1<<<0x7bff, 256>>>(d_bad + 4, d_first + 4);
    if (cudaDeviceSynchronize() != cudaSuccess) return 2;
    unsigned long long h_bad[5];
    uint32_t h_first[5];
    cudaMemcpy(h_bad, d_bad, sizeof h_bad, cudaMemcpyDeviceToHost);
    cudaMemcpy(h_first, d_first, sizeof h_first, cudaMemcpyDeviceToHost);
    out[0] = h_bad[0];
    out[1] = h_first[0];
    out[2] = h_bad[1];
    out[3] = h_first[1];
    out[4] = h_bad[2];
    out[5] = h_first[2];
    out[6] = h_bad[3];
    out[7] = h_first[3];
    out[8] = h_bad[4];
    out[9] = h_first[4];
    cudaFree(d_bad);
    cudaFree(d_first);
    return 0;
}
