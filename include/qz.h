/*
 * qz.h -- C ABI of the B200 (sm_100a) weight-only quantization library libqz.so.
 *
 * The library quantizes bf16 weight matrices with group-wise affine
 * quantization, packs the codes, and runs the matmuls that consume the packed
 * weights directly (dequantizing on the fly).  Every compute step runs in the
 * library's own CUDA kernels.
 *
 * Definitions (HF Transformers "Quantization concepts" guide, section
 * "Mapping values to fewer bits", and taqaniya.com "What is quantization",
 * IBM absmax example):
 *   S = (val_max - val_min) / (q_max - q_min)      scale (fp32, IEEE)
 *   Z = q_min - round(val_min / S)                  zero-point
 *   q = clamp(round(x / S + Z), q_min, q_max)       code (round half to even)
 *   x_hat = S * (q - Z)                             dequantized weight
 * with these fixed readings: the range [val_min, val_max] is widened to
 * contain 0.0; S == 0 becomes 1.0; S is stored as bf16 rounded toward +inf and
 * the stored value is the one quantization divides by; x_hat is the exact
 * fp32 product rounded to nearest-even bf16.
 *
 * Formats (argument triple bits / symmetric / group_size):
 *   bits 4, symmetric 0   codes 0..15 (unsigned nibble), zero 0..15 (uint8)
 *   bits 4, symmetric 1   codes -7..7 (two's-complement nibble), no zeros
 *   bits 8, symmetric 0   codes -128..127, zero -128..127 (int8 in a byte)
 *   bits 8, symmetric 1   codes -127..127 (absmax, range [-a, a]), no zeros
 * Granularity (section "Choose granularity"): group_size g > 0 with K % g == 0
 * quantizes runs of g consecutive values along each row, one scale (and zero)
 * per run, stored at [n * (K / g) + k / g]; g == K is per-channel (one per
 * output row); g == 0 is per-tensor (a single scale/zero).
 *
 * Layouts (all row-major, all device memory):
 *   w        N x K bf16 (N = output features, K = input features)
 *   codes    bits 4: N x K/2 bytes, value k in the low nibble of byte k/2 when
 *            k is even and in the high nibble when k is odd (section "int8
 *            and int4", packing figure); bits 8: N x K bytes
 *   scales   bf16, N x K/g (g > 0) or 1 (g == 0)
 *   zeros    uint8/int8 bytes, same shape as scales (asymmetric only)
 *   a        M x K bf16 activations; y = a * w_hat^T, M x N bf16
 *
 * Conventions for every entry point:
 *   - Pointers are DEVICE pointers and must be 16-byte aligned (scales and
 *     zeros: 2- and 1-byte aligned).  The caller owns and allocates every
 *     buffer, including workspaces; the library never allocates, frees or
 *     synchronizes.  `stream` is a cudaStream_t (NULL = legacy default stream)
 *     and all work is asynchronous on it.
 *   - Argument errors are returned synchronously before any launch and leave
 *     every buffer untouched.  QZ_ERR_CUDA reports a failed launch.
 *   - Inputs must be finite; NaN/Inf inputs (or a weight range whose width
 *     overflows fp32) give unspecified codes.
 *   - Calls are thread-safe.  Two calls that run concurrently need distinct
 *     workspaces.
 */
#ifndef QZ_H_
#define QZ_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define QZ_API __attribute__((visibility("default")))
#else
#define QZ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    QZ_OK = 0,
    QZ_ERR_INVALID_ARG = 1,     /* null pointer, bad size or shape */
    QZ_ERR_ALIGNMENT = 2,       /* a pointer is not aligned as required */
    QZ_ERR_UNSUPPORTED = 3,     /* a format or shape the kernels do not cover */
    QZ_ERR_WORKSPACE = 4,       /* workspace pointer missing or too small */
    QZ_ERR_CUDA = 5,            /* a CUDA call or launch failed */
    QZ_ERR_DEVICE_TIMEOUT = 6   /* a bounded device-side wait ran out */
} qz_status;

/* Operation ids for qz_workspace_bytes. */
enum {
    QZ_OP_QUANTIZE_PACK = 0,
    QZ_OP_DEQUANTIZE = 1,
    QZ_OP_W4A16_GEMV = 2,
    QZ_OP_W4A16_GEMM = 3,
    QZ_OP_W8A16_GEMV = 4,
    QZ_OP_W8A16_GEMM = 5,
    QZ_OP_GPTQ = 6,
    QZ_OP_FP4A16_GEMV = 7,
    QZ_OP_FP4A4_GEMM = 8
};

/* FP4 formats (kind argument of the qz_fp4_* entry points). */
enum {
    QZ_FP4_MX = 0,   /* MXFP4: blocks of 32, E8M0 (power-of-two) block scales */
    QZ_FP4_NV = 1    /* NVFP4: blocks of 16, E4M3 block scales, one fp32 tensor scale */
};

/* Static description of a status code (never NULL). */
QZ_API const char *qz_status_string(int status);

/* Library ABI version (major * 100 + minor). */
QZ_API int qz_version(void);

/*
 * Sizes in bytes of the three output buffers of qz_quantize_pack for an
 * N x K matrix in the given format (section "Choose granularity": one scale,
 * plus one zero when asymmetric, per group).  zeros_bytes is 0 when symmetric.
 * Host-only; never touches the GPU.
 */
QZ_API qz_status qz_packed_bytes(int64_t N, int64_t K, int32_t bits, int32_t symmetric,
                          int64_t group_size, size_t *codes_bytes,
                          size_t *scales_bytes, size_t *zeros_bytes);

/*
 * Device workspace needed by `op` for the given sizes (0 when none).  The
 * workspace of QZ_OP_QUANTIZE_PACK (per-tensor only) and of the GEMV/GEMM
 * paths that share tiles between CTAs must be zero-filled once before its
 * first use; every call that completes leaves its counters (and the
 * per-tensor word) at zero again, and the rest is scratch.  Host-only.  The kernels
 * size their grids for the device's SM count (a B200 has 148; a device with
 * more is treated as 148); the size returned here serves every SM count up
 * to 148, so it does not depend on the device.
 */
QZ_API qz_status qz_workspace_bytes(int32_t op, int64_t M, int64_t N, int64_t K,
                             int64_t group_size, size_t *bytes);

/*
 * The workspace a call uses when its grid is sized for `sms` SMs
 * (1 <= sms <= 148; a device's own count, capped at 148, is what the
 * kernels use).  qz_workspace_bytes returns the largest of these over every
 * `sms`, so a buffer of that size serves any device.  Host-only; a planning
 * query, not part of the method.
 */
QZ_API qz_status qz_workspace_bytes_for_sms(int32_t op, int64_t M, int64_t N, int64_t K,
                                            int64_t group_size, int32_t sms, size_t *bytes);

/*
 * quantize_pack: w (N x K bf16) -> codes, scales (bf16), zeros.
 * Quantization concepts guide, "Mapping values to fewer bits" (S, Z, q) and
 * "int8 and int4" (packing).  Requirements: N >= 1; K >= 1, K % 8 == 0;
 * group_size 0, or a divisor of K that is a multiple of 8 (the fast
 * warp-per-group kernel covers 32, 64, 128 and 256; other sizes, including
 * per-channel group_size == K, run one thread block per group).  `zeros`
 * must be NULL when symmetric and non-NULL otherwise.  Per-tensor
 * (group_size 0) needs a zero-filled workspace of qz_workspace_bytes bytes;
 * other formats accept workspace NULL.
 */
QZ_API qz_status qz_quantize_pack(const void *w, int64_t N, int64_t K, int32_t bits,
                           int32_t symmetric, int64_t group_size, void *codes,
                           void *scales, void *zeros, void *workspace,
                           size_t workspace_bytes, void *stream);

/*
 * dequantize: codes/scales/zeros -> w_hat (N x K bf16),
 * w_hat = bf16_rne(S * (q - Z)) (guide: "Dequantization reverses the
 * mapping"; the bf16 rounding is this library's fixed reading).  Same format
 * requirements as qz_quantize_pack; no workspace.
 */
QZ_API qz_status qz_dequantize(const void *codes, const void *scales, const void *zeros,
                        int64_t N, int64_t K, int32_t bits, int32_t symmetric,
                        int64_t group_size, void *w_hat, void *stream);

/*
 * W4A16 decode GEMV: y (M x N bf16) = a (M x K bf16) * w_hat^T where w_hat is
 * the int4 asymmetric group-wise weight (bits 4, symmetric 0) given by codes,
 * scales, zeros.  Quantization concepts guide, "Quantize weights or
 * activations" (weight-only: weights are dequantized to the compute dtype
 * before each matmul; decoding one token at a time is bound by reading the
 * weights) and the GPTQ explainer's fused dequantize-in-matmul kernels.
 * Each w_hat is formed exactly as qz_dequantize forms it, products are
 * accumulated in fp32, y is rounded to bf16.  Requirements: 1 <= M <= 64
 * (batched decode; 17..64 tokens take a variant that keeps the activations
 * in shared memory); N >= 1; K % 128 == 0; group_size a multiple of 32
 * dividing K.  Workspace:
 * qz_workspace_bytes(QZ_OP_W4A16_GEMV, M, N, K, group_size) bytes,
 * zero-filled before first use (0 bytes means workspace may be NULL).
 */
QZ_API qz_status qz_w4a16_gemv(const void *a, const void *codes, const void *scales,
                        const void *zeros, int64_t M, int64_t N, int64_t K,
                        int64_t group_size, void *y, void *workspace,
                        size_t workspace_bytes, void *stream);

/*
 * W4A16 prefill GEMM: the same product as qz_w4a16_gemv for any M >= 1,
 * dequantizing weight tiles into tensor memory for the tcgen05 tensor cores
 * (guide, "Quantize weights or activations": prefill and large batches are
 * compute-bound).  M <= 32 runs the decode kernel of qz_w4a16_gemv (faster there).  Each
 * output tile is 128 weight rows x up to 256 tokens, and the MMAs cover only
 * the tile's tokens (rounded up to 16).  Persistent CTAs take whole tiles
 * round robin; when the last, partial wave (or all tiles, when they are fewer
 * than the CTAs) would leave CTAs idle long enough, its tiles' K steps are
 * shared evenly by the CTAs instead (stream-K), whose fp32 partials meet in
 * the workspace and are added in K order (results do not depend on timing;
 * they depend on the device's SM count through the schedule).
 * Requirements: M >= 1; N >= 1; K % 128 == 0;
 * group_size a multiple of 64 dividing K (32 suffices for M <= 32).
 * Workspace: qz_workspace_bytes(QZ_OP_W4A16_GEMM, M, N, K, group_size)
 * bytes (0 when no tile is shared), zero-filled before first use; each call
 * that completes leaves its arrival counters at zero again (the partials
 * are scratch), so the buffer serves the next call unchanged.  A device-side wait that runs out (see qz_set_device_wait_limit)
 * makes the kernel return early and the next qz_device_status call reports
 * QZ_ERR_DEVICE_TIMEOUT; the workspace of that call must then be zero-filled
 * again before reuse.
 */
QZ_API qz_status qz_w4a16_gemm(const void *a, const void *codes, const void *scales,
                        const void *zeros, int64_t M, int64_t N, int64_t K,
                        int64_t group_size, void *y, void *workspace,
                        size_t workspace_bytes, void *stream);

/*
 * W8A16 decode GEMV: y = a * w_hat^T for the int8 symmetric per-channel
 * weight (bits 8, symmetric 1, group_size K; codes N x K int8, scales N bf16;
 * taqaniya.com IBM absmax example).  w_hat = bf16_rne(S * q), fp32
 * accumulation, bf16 y.  Requirements: 1 <= M <= 64; N >= 1; K % 128 == 0.
 * Workspace as for qz_w4a16_gemv with QZ_OP_W8A16_GEMV.
 */
QZ_API qz_status qz_w8a16_gemv(const void *a, const void *codes, const void *scales,
                        int64_t M, int64_t N, int64_t K, void *y, void *workspace,
                        size_t workspace_bytes, void *stream);

/*
 * W8A16 prefill GEMM: the same product as qz_w8a16_gemv for any M >= 1
 * (taqaniya.com "What is quantization", IBM absmax example, for the int8
 * symmetric weight; Quantization concepts guide, "Quantize weights or
 * activations": weight-only methods dequantize to the compute dtype before
 * each matmul, and prefill is compute-bound).  Weight tiles are dequantized (w_hat = bf16_rne(S * q), exactly as
 * qz_dequantize forms it) into tensor memory as the A operand of tcgen05
 * BF16 MMAs with fp32 accumulation; y is rounded to bf16.  M <= 32 runs the
 * decode kernel of qz_w8a16_gemv.  Tiles and their schedule as for
 * qz_w4a16_gemm.
 * Arguments: a (M x K bf16, row-major), codes (N x K int8, row-major),
 * scales (N bf16), y (M x N bf16, row-major), all device pointers owned by
 * the caller; a, codes and y 16-byte aligned, scales 2-byte aligned.
 * Requirements: M >= 1; N >= 1; K % 128 == 0.  Workspace:
 * qz_workspace_bytes(QZ_OP_W8A16_GEMM, M, N, K, K) bytes, zero-filled before
 * first use; each call that completes leaves its counters at zero again.  Errors: argument
 * errors return before any launch; QZ_ERR_CUDA if the launch fails; a
 * device-side wait that runs out makes the kernel return early, the next
 * qz_device_status call reports QZ_ERR_DEVICE_TIMEOUT, and the workspace of
 * that call must be zero-filled again before reuse.
 */
QZ_API qz_status qz_w8a16_gemm(const void *a, const void *codes, const void *scales,
                        int64_t M, int64_t N, int64_t K, void *y, void *workspace,
                        size_t workspace_bytes, void *stream);

/*
 * GPTQ layer-wise quantization (GPTQ explainer, azimuth.plus/paper/gptq:
 * sections on OBQ's error-compensating updates, the fixed column order, the
 * lazy batched updates and the Cholesky decomposition of the inverse
 * Hessian, and the algorithm paragraph with H = 2 X X^T).
 *   w        N x K bf16 weights (row-major; rows are outputs);
 *   x        n_samples x K bf16 calibration samples (one per row), so the
 *            page's X (one sample per column) is x^T and H = 2 x^T x;
 *   damp     the damping term is lambda = damp * mean(diag H) (1 if that
 *            mean is 0); 0.01 is the customary value (the page gives none);
 *   codes, scales, zeros: the packed format of qz_quantize_pack for the
 *            same bits / symmetric / group_size, consumed unchanged by the
 *            decode GEMVs and the prefill GEMMs.
 * The columns are quantized in their natural order, in lazy blocks of 128.
 * Each group's scale and zero come from the group's weights as they stand
 * (already compensated) when its first column is reached; every code is the
 * round-to-nearest code of that column's compensated weight, computed in
 * fp32 exactly as qz_quantize_pack computes codes.  The Hessian, its factor
 * and the compensation run in fp64.  Requirements: N >= 1; n_samples >= 1;
 * K % 8 == 0; group_size a multiple of 32 dividing K with group_size % 128
 * == 0 or 128 % group_size == 0 (so groups and blocks nest); damp >= 0.
 * Workspace: qz_workspace_bytes(QZ_OP_GPTQ, 1, N, K, group_size) bytes
 * (fp64: two K x K matrices, the N x K working weights and N x 128 errors),
 * any contents.  Inputs must be finite.
 */
QZ_API qz_status qz_gptq_quantize(const void *w, const void *x, int64_t N, int64_t K,
                                  int64_t n_samples, int32_t bits, int32_t symmetric,
                                  int64_t group_size, double damp, void *codes, void *scales,
                                  void *zeros, void *workspace, size_t workspace_bytes,
                                  void *stream);

/*
 * FP4 with block scales (Quantization concepts guide, section "FP4 with
 * block scales"; section "FP8" for E4M3).  An FP4 (E2M1) code has 1 sign,
 * 2 exponent and 1 mantissa bit and stands for 0, 0.5, 1, 1.5, 2, 3, 4 or 6
 * (or its negative): code = sign << 3 | index of the magnitude in that list.
 * Layouts: codes N x K/2 bytes, packed as the int4 format (value k in the
 * low nibble of byte k/2 when k is even); block scales N x K/B bytes, one per
 * B consecutive values of a row (MXFP4: B = 32, the E8M0 byte e + 127 of the
 * scale 2^e; NVFP4: B = 16, an E4M3 byte); NVFP4 also has one fp32 tensor
 * scale.  Readings of this library (the page fixes neither the block sizes
 * nor how scales are chosen): MXFP4 e is the smallest integer with
 * max|x| <= 6 * 2^e; NVFP4 s_t = amax / 2688 (6 x 448) in fp32 and the block
 * scale is the smallest E4M3 value >= fp32(amax_b / fp32(6 s_t)); each code
 * is the nearest E2M1 value to x / scale (fp32; NVFP4 scale fp32(s_b * s_t)),
 * ties to the even mantissa bit.  Dequantized bf16: MXFP4 e2m1 * 2^e (exact),
 * NVFP4 bf16_rne(fp32(fp32(e2m1 * s_b) * s_t)).
 */
QZ_API qz_status qz_fp4_packed_bytes(int64_t N, int64_t K, int32_t kind, size_t *codes_bytes,
                                     size_t *scales_bytes);

/*
 * FP4 quantize: w (N x K bf16, 16-byte aligned) -> codes (16-byte aligned),
 * block scales and, for NVFP4, *tensor_scale (one fp32 in device memory,
 * 4-byte aligned; it also holds the tensor's amax while the call runs; must
 * be NULL for MXFP4).  Requirements: K a multiple of the block size.
 */
QZ_API qz_status qz_fp4_quantize(const void *w, int64_t N, int64_t K, int32_t kind, void *codes,
                                 void *block_scales, void *tensor_scale, void *stream);

/* FP4 dequantize to N x K bf16 (w_hat 16-byte aligned, codes 4-byte aligned). */
QZ_API qz_status qz_fp4_dequantize(const void *codes, const void *block_scales,
                                   const void *tensor_scale, int64_t N, int64_t K, int32_t kind,
                                   void *w_hat, void *stream);

/*
 * FP4A16 decode GEMV: y (M x N bf16) = a (M x K bf16) * w_hat^T for FP4
 * weights with block scales ("Quantize weights or activations": NVFP4 runs a
 * matmul with 4-bit weights and 16-bit activations for decoding).  Each
 * weight enters the fp32-accumulated product as e2m1 * s_b exactly (bf16
 * holds it without rounding) and NVFP4's tensor scale multiplies the sums
 * before y is rounded to bf16.  Requirements: 1 <= M <= 16; N >= 1;
 * K % 128 == 0.  Workspace: qz_workspace_bytes(QZ_OP_FP4A16_GEMV, M, N, K,
 * 0) bytes, zero-filled before first use (0 bytes means NULL is allowed).
 */
QZ_API qz_status qz_fp4a16_gemv(const void *a, const void *codes, const void *block_scales,
                                const void *tensor_scale, int64_t M, int64_t N, int64_t K,
                                int32_t kind, void *y, void *workspace, size_t workspace_bytes,
                                void *stream);

/*
 * W4A4 prefill GEMM with FP4 weights and activations ("Quantize weights or
 * activations": for compute-bound prefill, quantizing the activations too lets
 * the matmul itself run on 4-bit tensor cores, NVFP4 W4A4; section "FP4 with
 * block scales" for the format).  The tensor cores apply the block scales
 * inside the MMA, so they need the scales of every 128 rows in the "MMA scale
 * layout": atoms of 128 rows x 4 consecutive scales of a row (512 bytes),
 * scale j of row r at byte (r % 32) * 16 + ((r % 128) / 32) * 4 + j % 4 of
 * atom (r / 128, j / 4), which starts at ((r / 128) * (K / B / 4) + j / 4) *
 * 512; rows are padded with zero scales to a multiple of 128.
 *
 * qz_fp4_mma_scale_bytes: bytes of that layout for `rows` rows.
 * qz_fp4_scales_to_mma: block scales as written by qz_fp4_quantize (rows x
 *   K/B bytes, 4-byte aligned) -> the MMA scale layout (16-byte aligned); a
 *   one-time conversion for weights.
 * qz_fp4a4_gemm: y (M x N bf16) = a_hat (M x K) * w_hat^T, where a_hat is a
 *   (M x K bf16, 16-byte aligned) quantized inside the call to the same FP4
 *   kind exactly as qz_fp4_quantize would (NVFP4 with its own tensor scale
 *   from max |a|), w_hat the FP4 weights: codes (N x K/2, 16-byte aligned),
 *   scales_mma (from qz_fp4_scales_to_mma) and, for NVFP4, tensor_scale (one
 *   fp32 in device memory; NULL for MXFP4).  The sums are fp32; NVFP4 scales
 *   them by fp32(s_t(a) * s_t(w)) before rounding to bf16.  After the call
 *   the workspace holds the quantized activations: codes (M x K/2 bytes) at
 *   offset 0, their scales in the MMA scale layout at offset
 *   round_up(M * K / 2, 256), and (NVFP4) max |a| as fp32 after those,
 *   at the next multiple of 256.
 * Requirements: M, N >= 1; K % 256 == 0.  Workspace: qz_workspace_bytes(
 * QZ_OP_FP4A4_GEMM, M, N, K, 0) bytes, 256-byte aligned; it need not be
 * zero-filled and is not left zero-filled, so it must not be a buffer that
 * the split-K calls above count on.
 */
QZ_API qz_status qz_fp4_mma_scale_bytes(int64_t rows, int64_t K, int32_t kind, size_t *bytes);
QZ_API qz_status qz_fp4_scales_to_mma(const void *block_scales, int64_t rows, int64_t K,
                                      int32_t kind, void *scales_mma, void *stream);
QZ_API qz_status qz_fp4a4_gemm(const void *a, const void *codes, const void *scales_mma,
                               const void *tensor_scale, int64_t M, int64_t N, int64_t K,
                               int32_t kind, void *y, void *workspace, size_t workspace_bytes,
                               void *stream);

/*
 * Size of the scratch array built into the library for
 * qz_w4a16_gemv_noalloc (8 MiB, held on every GPU that loads the library).
 */
#define QZ_GEMV_NOALLOC_SCRATCH_BYTES (8u << 20)

/*
 * W4A16 decode GEMV that allocates nothing and takes no workspace.  The
 * quantization pages have no counterpart to this entry point: it exists for
 * callers that cannot allocate device memory -- for example a plugin inside a
 * host application that owns all device memory and offers no allocator, or
 * latency-critical code that cannot afford cudaMalloc (which may synchronize
 * the device).  Arguments, requirements and results are those of
 * qz_w4a16_gemv for 1 <= M <= 16; the split-K scratch lives in a fixed array of
 * QZ_GEMV_NOALLOC_SCRATCH_BYTES inside the library.
 *   - Sizes whose scratch need (qz_workspace_bytes(QZ_OP_W4A16_GEMV, ...))
 *     exceeds that maximum are rejected with QZ_ERR_WORKSPACE before any
 *     launch.
 *   - The first call on a device looks up the array's device address on that
 *     device (with it current); make that first call before any stream
 *     capture.  A look-up that fails returns QZ_ERR_CUDA and is not
 *     remembered: the next call on that device tries again.
 *   - Each call clears the part of the array that must start at zero (with
 *     cudaMemsetAsync on `stream`) and never calls cudaMalloc, cudaFree or
 *     any allocating routine.
 *   - All calls share the one array, which keeps the last call's contents:
 *     calls that overlap on the GPU (different streams, or different host
 *     threads on one device) race on it and give undefined results.
 */
QZ_API qz_status qz_w4a16_gemv_noalloc(const void *a, const void *codes, const void *scales,
                                       const void *zeros, int64_t M, int64_t N, int64_t K,
                                       int64_t group_size, void *y, void *stream);

/*
 * Device-side wait bound used by kernels that wait on mbarriers (the GEMM),
 * in nanoseconds of wall time per wait; 0 restores the default (2 s).
 * Not part of the method: a safety bound so that a broken pipeline returns an
 * error instead of hanging the GPU.  Host-only setter, applies to later calls.
 */
QZ_API void qz_set_device_wait_limit(uint64_t limit);

/*
 * How a decode GEMV launch (qz_w4a16_gemv, qz_w8a16_gemv, qz_w4a16_gemm with
 * M <= 32) may overlap the kernel launched before it on the same stream.
 * Not part of the method: a launch-latency optimisation for decode loops.
 *   0  (default) plain stream order.
 *   1  programmatic dependent launch: the GEMV may start while the previous
 *      kernel finishes and fetches its first K blocks of packed codes, scales
 *      and zeros at once; it reads activations and writes y and the
 *      workspace only after that kernel has completed.  Only for callers
 *      whose weights are not written by the kernel launched just before the
 *      GEMV on the stream (weights quantized once and kept, as in a decode
 *      loop); otherwise the GEMV may read stale weights.
 * Host-only, process-wide, applies to later calls.  Returns
 * QZ_ERR_INVALID_ARG for other values.  qz_w4a16_gemv_noalloc always uses 0.
 */
QZ_API qz_status qz_set_launch_overlap(int32_t mode);

/*
 * Reads and clears the device error word of the current device (written by a
 * kernel whose bounded wait ran out).  Synchronizes the current device.
 * Returns QZ_OK or QZ_ERR_DEVICE_TIMEOUT (or QZ_ERR_CUDA).
 */
QZ_API qz_status qz_device_status(void);

#ifdef __cplusplus
}
#endif

#endif /* QZ_H_ */
