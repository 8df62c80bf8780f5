/*
 * awq.h -- C ABI of the B200 (sm_100a) AWQ INT4 weight-quantisation library
 * (libawq_b200.so).
 *
 * The method (activation-aware weight quantisation, AWQ) as the pages define
 * it:
 *   "From-Scratch AWQ INT4 Quantization on Qwen3-8B" -- sections
 *       "AWQ scaling", "Group-wise symmetric INT4",
 *       "AutoAWQ / HF-AWQ GEMM on-disk format" (and the exporter's step 4);
 *   "AWQ architecture, in depth: the calibration pipeline, scale search,
 *       packed format and serving kernels" -- sections "The scale search as
 *       code" and "Quantization, storage and packing";
 *   "Weight-Only Quantization: GPTQ and AWQ" -- section 5 (AWQ) and
 *       sections 6-9 (the packed format).
 *
 * Conventions shared by every entry point:
 *   - Every tensor argument is a DEVICE pointer owned by the caller; the
 *     library never allocates, frees or retains memory.  Scratch memory comes
 *     from the caller's workspace (size from awq_workspace_size); its
 *     contents need not be initialised and are clobbered.
 *   - Matrices are row-major and dense: W is fp16 [d_out, d_in] (row stride
 *     d_in), X is fp16 [T, ld] with the first d_in columns used.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Every
 *     call only enqueues kernels on it and returns; nothing synchronises.
 *     Outputs are valid once the stream has reached that point.
 *   - Arguments are validated on the host before anything is enqueued; on a
 *     validation error nothing is enqueued and the outputs are untouched.
 *     A launch failure returns AWQ_ERR_CUDA.  The library never aborts.
 *   - A device pointer must be 16-byte aligned (AWQ_ERR_ALIGNMENT otherwise).
 *   - Errors found on the device (non-finite inputs, a bounded wait that
 *     gave up) are reported twice: in the outputs, as each entry point
 *     states, and as sticky condition bits of the device (AWQ_FLAG_*), which
 *     awq_last_device_flags() returns and clears.
 *   - Results are deterministic: the same inputs give the same bits.
 *   - The calls may run concurrently on different streams provided their
 *     workspaces do not overlap.
 */
#ifndef AWQ_B200_AWQ_H
#define AWQ_B200_AWQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum awq_status {
    AWQ_OK = 0,
    AWQ_ERR_INVALID_ARG = 1,   /* a size, count or pointer is out of range   */
    AWQ_ERR_UNSUPPORTED = 2,   /* valid but not implemented (e.g. group size) */
    AWQ_ERR_ALIGNMENT = 3,     /* a pointer or leading dimension misaligned   */
    AWQ_ERR_WORKSPACE = 4,     /* workspace NULL or smaller than required      */
    AWQ_ERR_CUDA = 5,          /* a CUDA runtime call or launch failed         */
    AWQ_ERR_NONFINITE = 6,     /* non-finite data met on the device (flags)    */
    AWQ_ERR_DEVICE_TIMEOUT = 7 /* a bounded device-side wait gave up (flags)   */
} awq_status;

/* Flags of awq_scale_search / awq_output_error / awq_clip_search. */
#define AWQ_SCALE_FP16 0  /* group scale rounded to fp16 (the stored format) */
#define AWQ_SCALE_FP32 1  /* group scale kept in fp32 (the worked example)  */
/* awq_scale_search only: duo scaling candidates ("AWQ architecture ...",
 * section "The scale search as code"): s_i = max(x^r / (w_mean^(1-r) +
 * 1e-4), 1e-4), normalised as usual, with w_mean[j] the mean over every row
 * of the segments of |W[r, j]| / max_k |W[r, k]| (fp64); needs
 * d_in <= 16384 and the AWQ_OP_SCALE_SEARCH_DUO workspace. */
#define AWQ_DUO_SCALING 2
/* awq_scale_search only: the asymmetric INT4 grid ("AWQ architecture ...",
 * section "Quantization, storage and packing": a 16-bit scale and a 4-bit
 * zero point per group and output channel).  Per group, with ws = w * s:
 * range = max(max ws - min ws, 1e-5), q_scale = fp16(range / 15),
 * zero = clamp(rint(-min ws / q_scale), 0, 15),
 * q = clamp(rint(ws / q_scale) + zero, 0, 15), w_hat = (q - zero) q_scale / s.
 * Pack the result with awq_quantize_pack(zero_point = AWQ_ZERO_POINT_ASYM). */
#define AWQ_ASYMMETRIC 4
/* zero_point argument of awq_quantize_pack selecting the asymmetric grid */
#define AWQ_ZERO_POINT_ASYM (-1)
/* awq_scale_search only, a TEST HOOK for the failure path of the bounded
 * device waits: CTA 0's first weight load is armed for 16 bytes more than
 * the copy carries, so that load's completion is a phase nothing finishes
 * (the copy itself lands).  The CTA's waits give up after their 2 s limit
 * and its drain after 20 s; the call then reports best_idx = -2 (err and
 * s_best invalid) and raises AWQ_FLAG_WAIT_TIMEOUT, no copy is left in
 * flight, and later calls run normally.  Never set outside such a test. */
#define AWQ_TEST_STALL_WAIT 0x40000000

/* Operation ids of awq_workspace_size. */
#define AWQ_OP_ACT_STATS    0
#define AWQ_OP_SCALE_SEARCH 1
#define AWQ_OP_OUTPUT_ERROR 2
#define AWQ_OP_CLIP_SEARCH  3
#define AWQ_OP_SCALE_SEARCH_DUO 4   /* awq_scale_search with AWQ_DUO_SCALING */
#define AWQ_OP_CLIP_SEARCH_OUTPUT 5 /* awq_clip_search_output */

/* Clip ratios: index i stands for c_i = (AWQ_CLIP_DEN - i) / AWQ_CLIP_DEN
 * rounded to fp32; 0 is no clipping, at most AWQ_CLIP_MAX ratios. */
#define AWQ_CLIP_DEN 20
#define AWQ_CLIP_MAX 20

/* Condition bits raised on the device (awq_last_device_flags). */
#define AWQ_FLAG_NONFINITE_X     0x1u  /* awq_act_stats: a column of X held a NaN or
                                          an infinity (its x_mean is NaN or inf)  */
#define AWQ_FLAG_NONFINITE_SCORE 0x2u  /* awq_scale_search / awq_output_error /
                                          awq_clip_search: an error sum was not
                                          finite (NaN or inf in W, x_mean or s);
                                          best_idx is -1, err NaN or inf          */
#define AWQ_FLAG_NONFINITE_GROUP 0x4u  /* awq_quantize_pack: a group held a NaN or
                                          an infinity (it stored scale NaN)      */
#define AWQ_FLAG_NONFINITE_SCALE 0x8u  /* awq_norm_group_scale: a member scale or
                                          the shared scale was not finite        */
#define AWQ_FLAG_WAIT_TIMEOUT    0x10u /* a bounded wait inside a kernel gave up
                                          (best_idx -2; outputs invalid)         */

/*
 * Sticky device-side condition bits of the CURRENT device.  The kernels of
 * every entry point raise AWQ_FLAG_* bits there (in addition to what their
 * outputs show) when they meet non-finite data or give up a bounded wait;
 * the bits accumulate over calls, streams and host threads until read with
 * clear != 0.
 *
 *   flags   HOST output: the bits raised since the last clearing read
 *   clear   nonzero: zero the bits after reading them
 *
 * Synchronises the current device first (cudaDeviceSynchronize), so every
 * call enqueued before it is reflected.  Returns AWQ_ERR_DEVICE_TIMEOUT if
 * AWQ_FLAG_WAIT_TIMEOUT is set, else AWQ_ERR_NONFINITE if any other bit is
 * set, else AWQ_OK; AWQ_ERR_CUDA if the synchronisation or the read failed
 * (e.g. an earlier kernel faulted), with awq_last_error() holding the text.
 * Clearing while other host threads enqueue work on the device may drop bits
 * raised by that work.
 */
awq_status awq_last_device_flags(uint32_t *flags, int clear);

/* Human-readable name of a status code (static storage; never NULL). */
const char *awq_status_string(int status);

/* Version of this ABI (major * 100 + minor). */
int awq_abi_version(void);

/* Text of the last failed CUDA runtime call seen by the library on the
 * calling host thread (which call, the error name and its description), for
 * an AWQ_ERR_CUDA.  Static thread-local storage; never NULL. */
const char *awq_last_error(void);

/*
 * Bytes of workspace that `op` needs for the given sizes.  For
 * AWQ_OP_ACT_STATS only d_in matters; for AWQ_OP_SCALE_SEARCH d_in, the
 * group size and n_grid; for AWQ_OP_OUTPUT_ERROR all of them (T is the token
 * count, d_out_total the rows of W); for AWQ_OP_CLIP_SEARCH the group size
 * and d_in (16.6 KB plus 4 bytes per input channel).  Writes *bytes; returns
 * AWQ_ERR_INVALID_ARG for an unknown op or out-of-range size.
 */
awq_status awq_workspace_size(int op, int64_t T, int64_t d_out_total,
                              int64_t d_in, int group_size, int n_grid,
                              size_t *bytes);

/*
 * Per-input-channel activation magnitude, the AWQ salience statistic
 * ("From-Scratch AWQ ...", section "AWQ scaling": x = |X|.mean(0);
 * "AWQ architecture ...", section "The scale search as code").
 *
 *   x_mean[j] = (1/T) * sum_{t<T} |X[t, j]|,   j < d_in
 *
 * The sum is exact (every |fp16| is an integer multiple of 2^-24), then
 * divided by T in fp64 and rounded to fp32.  A column holding a NaN gives
 * NaN, one holding an infinity (and no NaN) gives +inf; either raises
 * AWQ_FLAG_NONFINITE_X.
 *
 *   X        fp16 [T, ld] device, 16-byte aligned; ld % 8 == 0, ld >= d_in
 *   T        tokens, 1 <= T <= 2^23
 *   d_in     channels, 1 <= d_in <= 2^24, d_in % 8 == 0
 *   x_mean   fp32 [d_in] device output
 *   ws       workspace of awq_workspace_size(AWQ_OP_ACT_STATS, ...) bytes;
 *            that size is currently 0, and ws may then be NULL
 */
awq_status awq_act_stats(const void *X, int64_t T, int64_t d_in, int64_t ld,
                         float *x_mean, void *ws, size_t ws_bytes,
                         void *stream);

/*
 * AWQ per-channel scale search over an alpha grid, fused over all grid
 * points ("From-Scratch AWQ ...", sections "AWQ scaling" and "Group-wise
 * symmetric INT4"; "AWQ architecture ...", section "The scale search as
 * code").  For i < n_grid, alpha_i = i / n_grid:
 *
 *   s_i[j]   = max(x_mean[j], 1e-4)^alpha_i, then divided by
 *              sqrt(max_j s_i[j] * min_j s_i[j])     (fp64, rounded to fp32)
 *   per row r and group k of group_size channels, in fp32:
 *     ws       = W[r, j] * s_i[j]
 *     q_scale  = fp16_rne(max |ws| / 7)  (AWQ_SCALE_FP16; 0 for an all-zero
 *                group; held at 65504 if it overflows fp16)
 *     q        = clamp(rint(ws / q_scale), -7, 7)
 *   err[i]   = sum over every segment, row and channel of
 *              ((W[r, j] - q * q_scale / s_i[j]) * x_mean[j])^2
 *   best_idx = first i with the smallest err[i];  s_best = s_{best_idx}.
 *
 * The n_seg weight segments share the input (e.g. q/k/v, or gate/up): one
 * scale vector is searched for all of them and their errors are summed.
 *
 *   n_seg       1..AWQ_MAX_SEGMENTS
 *   W           HOST array of n_seg DEVICE pointers, fp16 [d_out[k], d_in]
 *   d_out       HOST array of n_seg row counts, each >= 1
 *   d_in        channels, multiple of group_size
 *   x_mean      fp32 [d_in] device (from awq_act_stats)
 *   group_size  32, 64 or 128
 *   n_grid      1..32 grid points (20 in the method)
 *   flags       AWQ_SCALE_FP16 or AWQ_SCALE_FP32, optionally with
 *               AWQ_DUO_SCALING, AWQ_ASYMMETRIC, AWQ_TEST_STALL_WAIT
 *   err         fp64 [n_grid] device output
 *   best_idx    int32 [1] device output; -1 if any err is not finite (NaN or
 *               infinite input; raises AWQ_FLAG_NONFINITE_SCORE), -2 if a
 *               device-side wait gave up (raises AWQ_FLAG_WAIT_TIMEOUT)
 *   s_best      fp32 [d_in] device output (NaN when best_idx < 0)
 *   ws          workspace of awq_workspace_size(AWQ_OP_SCALE_SEARCH, ...)
 * Each term is evaluated in fp32 as (ws - q * q_scale)^2 * (x_mean/s_i)^2,
 * summed in fp32 over a thread's share of 8 units and in fp64 in a fixed
 * order after that, so results are deterministic; against the exact score
 * of the same decisions the relative difference is about 3e-8 on a
 * 4096 x 4096 layer (the tested bar is 1e-5).
 */
#define AWQ_MAX_SEGMENTS 8
awq_status awq_scale_search(int n_seg, const void *const *W,
                            const int64_t *d_out, int64_t d_in,
                            const float *x_mean, int group_size, int n_grid,
                            int flags, double *err, int32_t *best_idx,
                            float *s_best, void *ws, size_t ws_bytes,
                            void *stream);

/*
 * awq_scale_search without a workspace, for callers that cannot allocate
 * device memory (a plug-in whose host framework owns all device memory and
 * offers it no allocator, a section where a cudaMalloc's possible device
 * synchronisation is not acceptable, a C caller holding only its own input
 * and output buffers).  The pages have no counterpart: this is a deployment
 * convenience, not part of the method.
 *
 * Same arguments, results and errors as awq_scale_search, minus ws/ws_bytes.
 * The scratch is one static device array of AWQ_NOALLOC_SCRATCH_BYTES inside
 * the library; every GPU that uses the library keeps it until the process
 * exits.  Calls whose workspace need (awq_workspace_size with
 * AWQ_OP_SCALE_SEARCH, or AWQ_OP_SCALE_SEARCH_DUO when flags hold
 * AWQ_DUO_SCALING) exceeds it return AWQ_ERR_WORKSPACE with nothing
 * enqueued -- e.g. d_in = 16384 fits with n_grid <= 29, d_in = 12288 with
 * n_grid <= 32; duo scaling needs d_in * 8 bytes per weight-mean CTA on top
 * and so fits only small d_in (d_in <= 2048 at 20 grid points).  The first call on a device looks the array's address up
 * (cudaGetSymbolAddress, that device current) and caches it for the life of
 * the process: make it before any stream capture on that device, and do not
 * use this entry point on a device after a cudaDeviceReset of it (the cached
 * address belonged to the destroyed context).  All calls on a device share the array;
 * each call rewrites every scratch byte it reads, but calls that overlap on
 * the GPU (unordered streams) race on it.  Allocates nothing.
 */
#define AWQ_NOALLOC_SCRATCH_BYTES (4u << 20)
awq_status awq_scale_search_noalloc(int n_seg, const void *const *W,
                                    const int64_t *d_out, int64_t d_in,
                                    const float *x_mean, int group_size,
                                    int n_grid, int flags, double *err,
                                    int32_t *best_idx, float *s_best,
                                    void *stream);

/*
 * Group-wise symmetric INT4 quantisation of W * s and packing into the
 * AutoAWQ GEMM layout ("From-Scratch AWQ ...", sections "Group-wise
 * symmetric INT4", "AutoAWQ / HF-AWQ GEMM on-disk format" and exporter
 * step 4; "AWQ architecture ...", section "Quantization, storage and
 * packing").  Codes are decided exactly as in awq_scale_search (fp16 group
 * scale) with the IEEE fp32 quotient ws / q_scale:
 *
 *   u[r, j]        = q[r, j] + zero_point                (0..15)
 *   qweight[j, c]  = nibble p (bits 4p..4p+3) holds u[8c + order[p], j],
 *                    order = {0, 2, 4, 6, 1, 3, 5, 7}
 *   scales[k, r]   = fp16 q_scale of row r, group k
 *   qzeros[k, c]   = zero_point in all eight nibbles
 *
 *   W           fp16 [d_out, d_in] device
 *   d_out       multiple of 8;  d_in multiple of group_size
 *   s           fp32 [d_in] device scale (s_best), or NULL for s = 1 (RTN)
 *   clip_idx    uint8 [d_out, d_in / group_size] device clip ratio indices
 *               from awq_clip_search, or NULL for none: group (r, k) uses the
 *               range c * max|ws| with c = (20 - i) / 20 (indices above 19
 *               count as 19), q_scale = fp16(fl32(fl32(c m) / 7)), and codes
 *               beyond the range saturate at +-7
 *   group_size  32, 64 or 128
 *   zero_point  7 or 8 (8: codes 1..15; 7: codes 0..14), or
 *               AWQ_ZERO_POINT_ASYM for the asymmetric grid of
 *               AWQ_ASYMMETRIC: codes 0..15 and qzeros holding each (group,
 *               row)'s zero point in the same nibble order as qweight
 *               (clip_idx must then be NULL); a non-finite group stores
 *               scale NaN, zero point 8 and codes 8
 *   qweight     int32 [d_in, d_out / 8] device output
 *   scales      fp16 [d_in / group_size, d_out] device output
 *   qzeros      int32 [d_in / group_size, d_out / 8] device output
 * A group holding a non-finite value stores scale NaN (0x7E00) and code
 * zero_point for all its weights, and raises AWQ_FLAG_NONFINITE_GROUP.
 */
awq_status awq_quantize_pack(const void *W, int64_t d_out, int64_t d_in,
                             const float *s, const uint8_t *clip_idx,
                             int group_size, int zero_point, int32_t *qweight,
                             void *scales, int32_t *qzeros, void *stream);

/*
 * One shared scale for the linears that follow one norm ("From-Scratch AWQ
 * ...", section "AutoAWQ / HF-AWQ GEMM on-disk format", exporter steps 1-2:
 * the per-linear scales of q/k/v, or of gate/up, are aggregated into one
 * scale per norm group by their geometric mean, folded into the norm, and
 * the members are re-quantised with it by awq_quantize_pack):
 *
 *   s_shared[j] = (s_0[j] * ... * s_{n-1}[j])^(1/n)
 *
 * evaluated as the fp64 product in member order, then sqrt for n = 2 and
 * pow(., 1/n) otherwise, rounded once to fp32; n = 1 copies s_0.
 *
 *   n          1..AWQ_MAX_SEGMENTS member scales
 *   s          HOST array of n DEVICE pointers, fp32 [d_in] each (each
 *              normally the s_best of a one-segment awq_scale_search)
 *   d_in       1..2^24 channels
 *   s_shared   fp32 [d_in] device output (a channel whose member scales
 *              hold a NaN, an infinity, or whose product leaves the fp64
 *              range gets that non-finite value and raises
 *              AWQ_FLAG_NONFINITE_SCALE)
 */
awq_status awq_norm_group_scale(int n, const float *const *s, int64_t d_in,
                                float *s_shared, void *stream);

/*
 * Per (row, group) clip search at a fixed scale ("AWQ architecture ...",
 * section "The pipeline end to end", step 5: an optional search of a
 * clipping range per output channel that shrinks the quantisation range to
 * cut rounding error on outliers; the pages give no formula, the reading
 * is this one).  For every row r, group k and i < n_clip, with
 * c_i = (20 - i) / 20 rounded to fp32:
 *
 *   q_scale_i = fp16_rne(fl32(fl32(c_i * max_j |w_j s_j|) / 7))
 *   q_j       = clamp(rint(w_j s_j / q_scale_i), -7, 7)
 *   e_i       = sum_j ((w_j - q_j q_scale_i / s_j) * x_mean_j)^2
 *
 * and clip_idx[r, k] = the first i with the smallest e_i.  err[0] is the
 * total error without clipping (i = 0 everywhere), err[1] the total with
 * the chosen ratios; both are reduced in a fixed order (deterministic).
 * Each e_i is summed in fp32 (so two ratios within ~1e-6 of each other may
 * be ordered differently from an exact evaluation); codes use an
 * approximate reciprocal of q_scale (the stored codes come from
 * awq_quantize_pack's exact quotient).
 *
 *   W           fp16 [d_out, d_in] device;  d_out >= 1
 *   d_in        multiple of group_size
 *   x_mean      fp32 [d_in] device
 *   s           fp32 [d_in] device (normally s_best), or NULL for s = 1
 *   group_size  32, 64 or 128
 *   n_clip      1..AWQ_CLIP_MAX ratios (10: down to 0.55)
 *   flags       AWQ_SCALE_FP16 or AWQ_SCALE_FP32
 *   clip_idx    uint8 [d_out, d_in / group_size] device output
 *   err         fp64 [2] device output (NaN if W holds a non-finite value;
 *               such a group keeps index 0; a non-finite total raises
 *               AWQ_FLAG_NONFINITE_SCORE)
 *   ws          workspace of awq_workspace_size(AWQ_OP_CLIP_SEARCH, ...),
 *               256-byte aligned
 */
awq_status awq_clip_search(const void *W, int64_t d_out, int64_t d_in,
                           const float *x_mean, const float *s, int group_size,
                           int n_clip, int flags, uint8_t *clip_idx,
                           double *err, void *ws, size_t ws_bytes,
                           void *stream);

/*
 * The clip search scored in output space ("AWQ architecture ...", section
 * "The pipeline end to end", step 5: the clipping range; section "The scale
 * search as code": candidates scored on the output).  The pages give no
 * formula; the reading: ratios and clipped fake quantisation exactly as in
 * awq_clip_search (codes decided by the IEEE quotient), and each row r,
 * group k and ratio i scored by the group's share of the output error
 *
 *   e[r,k,i] = sum_t ( sum_{j in group k} X[t,j] (W[r,j] - W_hat_i[r,j]) )^2
 *
 * (evaluated as v^T H_k v with H_k = X_k^T X_k: the Gram matrix in fp64,
 * rounded to fp32, the forms in fp32 with fp64 sums across the warp, so e
 * is within about 1e-6 relative of the fp64 definition and two ratios
 * closer than that may be ordered differently).  clip_idx[r,k] = the first
 * i with the smallest e; err[0] = sum of e[.,.,0] (no clipping), err[1] =
 * sum of the chosen e, fixed-order sums (deterministic).
 *
 *   X           fp16 [T, ld] device (the linear's input); 1 <= T <= 2^24,
 *               ld % 8 == 0, ld >= d_in
 *   W           fp16 [d_out, d_in] device;  1 <= d_out <= 2^22
 *   s           fp32 [d_in] device scale (normally s_best), or NULL for 1
 *   group_size  32, 64 or 128;  d_in a multiple of it, <= 2^20
 *   n_clip      1..AWQ_CLIP_MAX;  flags AWQ_SCALE_FP16 or AWQ_SCALE_FP32
 *   clip_idx    uint8 [d_out, d_in / group_size] device output (feeds
 *               awq_quantize_pack's clip_idx)
 *   err         fp64 [2] device output (NaN if W holds a non-finite value,
 *               raising AWQ_FLAG_NONFINITE_SCORE; such a group keeps index 0)
 *   ws          workspace of awq_workspace_size(AWQ_OP_CLIP_SEARCH_OUTPUT,
 *               T, d_out, d_in, group_size, 1, ...): the Gram matrices
 *               (d_in * group_size fp32) and per-CTA partials; 256-byte aligned
 */
awq_status awq_clip_search_output(const void *X, int64_t T, int64_t ld, const void *W,
                                  int64_t d_out, int64_t d_in, const float *s,
                                  int group_size, int n_clip, int flags,
                                  uint8_t *clip_idx, double *err, void *ws,
                                  size_t ws_bytes, void *stream);

/*
 * Optional output-space scoring of every grid point ("AWQ architecture
 * ...", section "The scale search as code": the group's output after
 * fake quantisation compared with the full-precision output; "Weight-Only
 * Quantization: GPTQ and AWQ", section 2: the output error is X (W - W_hat)):
 *
 *   err[i] = || X (W - W_hat_i)^T ||_F^2,   W_hat_i = Q(W * s_i) / s_i
 *
 * with s_i and Q exactly as in awq_scale_search (symmetric, or the
 * asymmetric grid with AWQ_ASYMMETRIC).  The contraction runs on
 * the tensor cores with fp16 operands and fp32 accumulation.  W - W_hat_i
 * is formed exactly in fp32, scaled per row by a power of two, and split
 * into two fp16 parts hi + lo (lo = the rounding error of hi), so that the
 * product sees the difference to about 22 bits; X is fp16 already, so
 * X (hi + lo)^T accumulates both parts into one fp32 accumulator.  The
 * running accumulator is folded into a second fp32 sum every 2048 terms of
 * the (hi, lo)-doubled reduction, the squares are summed in fp32 per 128 x 256 output tile and
 * in fp64 across tiles.  The result is tested against the fp64
 * definition at 1e-5 relative.
 *
 *   X           fp16 [T, d_in] device;  1 <= T <= 2^24
 *   W           fp16 [d_out, d_in] device; d_out % 8 == 0
 *   x_mean      fp32 [d_in] device (defines s_i)
 *   group_size  32, 64 or 128;  d_in multiple of group_size and of 64
 *   n_grid      1..32
 *   flags       AWQ_SCALE_FP16 or AWQ_SCALE_FP32, optionally | AWQ_ASYMMETRIC
 *               (W_hat from the asymmetric grid of awq_scale_search; pack the
 *               chosen scale with AWQ_ZERO_POINT_ASYM)
 *   err         fp64 [n_grid] device output (NaN for every i if W holds a
 *               non-finite value)
 *   best_idx    int32 [1] device output (first minimum; -1 if non-finite,
 *               raising AWQ_FLAG_NONFINITE_SCORE; -2 if a bounded wait
 *               inside a kernel gave up, raising AWQ_FLAG_WAIT_TIMEOUT)
 *   s_best      fp32 [d_in] device output s_{best_idx} (NaN if best_idx < 0),
 *               or NULL when the caller does not want it
 *   ws          workspace of awq_workspace_size(AWQ_OP_OUTPUT_ERROR, ...),
 *               256-byte aligned
 * Errors: AWQ_ERR_INVALID_ARG / AWQ_ERR_UNSUPPORTED / AWQ_ERR_ALIGNMENT /
 * AWQ_ERR_WORKSPACE before any launch, AWQ_ERR_CUDA when a launch fails
 * (awq_last_error() then holds the CUDA error text).
 */
awq_status awq_output_error(const void *X, int64_t T, const void *W,
                            int64_t d_out, int64_t d_in, const float *x_mean,
                            int group_size, int n_grid, int flags,
                            double *err, int32_t *best_idx, float *s_best,
                            void *ws, size_t ws_bytes, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* AWQ_B200_AWQ_H */
