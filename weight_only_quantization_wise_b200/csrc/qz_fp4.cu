// qz_fp4.cu -- FP4 (E2M1) weights with block scales: quantize and dequantize.
//
// Quantization concepts guide, section "FP4 with block scales": an FP4 value
// has 1 sign, 2 exponent and 1 mantissa bit and represents only 0, 0.5, 1,
// 1.5, 2, 3, 4 and 6 (and their negatives), so every small block of values
// carries its own scale, stored in the format.  MXFP4 (micro-scaling) uses a
// power-of-two scale, which only shifts exponents; NVFP4 uses smaller blocks
// with an FP8 (E4M3, section "FP8") scale that can fall between powers of two,
// plus one scale for the tensor that keeps the FP8 block scales in range.
//
// Layouts (this library's readings: the page fixes neither block sizes nor
// how a scale is chosen):
//   codes         N x K/2 bytes, value k in the low nibble of byte k/2 when k
//                 is even (the packing of the int4 format); a code is
//                 sign << 3 | magnitude index (0, 0.5, 1, 1.5, 2, 3, 4, 6);
//   block scales  N x K/B bytes: MXFP4 B = 32, the E8M0 byte e + 127 of the
//                 scale 2^e; NVFP4 B = 16, an E4M3 byte;
//   tensor scale  NVFP4 only: one fp32.
// Scales: MXFP4 e is the smallest integer with max|x| <= 6 * 2^e (clamped to
// [-127, 127]); NVFP4 s_t = fp32(amax / 2688) (6 x 448: the largest E2M1
// and E4M3 values), s_b = the smallest E4M3 value >= fp32(amax_b /
// fp32(6 s_t)), at most 448, 0 for an all-zero block.  Codes: x divided by
// the block's scale (2^e, or fp32(s_b * s_t)) in fp32, rounded to the
// nearest E2M1 magnitude, ties to the even mantissa bit, saturating at 6.
// Dequantized bf16: MXFP4 e2m1 * 2^e (exact); NVFP4
// bf16_rne(fp32(fp32(e2m1 * s_b) * s_t)) (the inner product is exact).
#include <cuda_runtime.h>

#include "qz_internal.cuh"

namespace qz {
namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t h) { return __uint_as_float(h << 16); }

// E4M3 byte (sign ignored) -> value.
__device__ __forceinline__ float e4m3_value(uint32_t b) {
    const uint32_t e = (b >> 3) & 15u, m = b & 7u;
    if (e == 0) return (float)m * 0.001953125f;                  // m * 2^-9 (exact)
    return __uint_as_float(((e + 120u) << 23) | (m << 20));
}

// The smallest E4M3 value >= t (t >= 0), at most 448 (byte 0x7E); 0 for t = 0.
// Bytes 1..0x7E are increasing in value without gaps between the subnormal
// and normal ranges (m * 2^-9, then (8 + m) * 2^(e - 10)).
__device__ __forceinline__ uint32_t e4m3_round_up(float t) {
    if (!(t > 0.0f)) return 0u;
    if (t < 0.015625f) {                                         // below 2^-6: subnormal step 2^-9
        const float m = ceilf(t * 512.0f);                       // exact scaling
        return (uint32_t)m;                                      // 8 -> 0x08 = 2^-6
    }
    // Normal range: adding 2^20 - 1 to the fp32 bits and dropping the low 20
    // bits keeps three mantissa bits rounded up (a carry moves into the
    // exponent), which leaves the biased exponent and mantissa of the E4M3
    // value shifted by (127 - 7) << 3; anything above 448 (0x7E) is clamped.
    const uint32_t r = (__float_as_uint(t) + 0x000FFFFFu) >> 20;
    const uint32_t b = r - 960u;
    return b > 0x7Eu ? 0x7Eu : b;
}

__device__ __forceinline__ float e2m1_value(uint32_t c) {
    const uint32_t i = c & 7u;
    const float mag = i < 4 ? 0.5f * (float)i : (i == 4 ? 2.0f : i == 5 ? 3.0f : i == 6 ? 4.0f : 6.0f);
    return (c & 8u) ? -mag : mag;
}

__device__ __forceinline__ int64_t grid_stride() { return (int64_t)gridDim.x * blockDim.x; }
__device__ __forceinline__ int64_t thread_index() {
    return (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
}

__device__ __forceinline__ uint32_t bf16x2_absmax(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("max.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a & 0x7FFF7FFFu), "r"(b & 0x7FFF7FFFu));
    return d;
}

__device__ __forceinline__ uint32_t chunk_absmax(uint32_t m2, const uint4 &v) {
    return bf16x2_absmax(m2, bf16x2_absmax(bf16x2_absmax(v.x, v.y), bf16x2_absmax(v.z, v.w)));
}

// max |w| over the tensor into *amax (fp32 bits, non-negative: ordered as
// unsigned integers).  Four 16-byte loads in flight per thread.
__global__ void __launch_bounds__(kThreads) fp4_amax_kernel(const uint4 *__restrict__ w,
                                                           int64_t chunks, unsigned *amax) {
    uint32_t m2 = 0u;
    const int64_t stride = grid_stride();
    int64_t c = thread_index();
    for (; c + 3 * stride < chunks; c += 4 * stride) {
        uint4 v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) v[u] = __ldg(w + c + u * stride);
#pragma unroll
        for (int u = 0; u < 4; ++u) m2 = chunk_absmax(m2, v[u]);
    }
    for (; c < chunks; c += stride) m2 = chunk_absmax(m2, __ldg(w + c));
    float m = fmaxf(bf16_bits_to_f32(m2 & 0xFFFFu), bf16_bits_to_f32(m2 >> 16));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    __shared__ float part[kThreads / 32];
    if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int i = 1; i < kThreads / 32; ++i) m = fmaxf(m, part[i]);
        atomicMax(amax, __float_as_uint(m));
    }
}

__device__ __forceinline__ float nv_tensor_scale(float amax) {
    return amax > 0.0f ? __fdiv_rn(amax, 2688.0f) : 1.0f;
}

// Byte offset of scale j of row r in the MMA scale layout: atoms of 128
// rows x 4 scales (512 bytes), row r at (r % 32) * 16 + ((r % 128) / 32) * 4
// + j % 4 inside its atom, atoms ordered (r / 128, j / 4) with `atoms_k`
// atoms per 128-row block.
__device__ __forceinline__ int64_t mma_scale_offset(int64_t r, int64_t j, int64_t atoms_k) {
    return (((r >> 7) * atoms_k + (j >> 2)) << 9) + ((r & 31) << 4) + (((r >> 5) & 3) << 2) + (j & 3);
}

// Eight values (v[i] -> nibble i) as E2M1 codes: the hardware conversion
// rounds to the nearest E2M1 value, ties to the even mantissa bit (0.25 -> 0,
// 0.75 -> 1, 1.25 -> 1, 1.75 -> 2, 2.5 -> 2, 3.5 -> 4, 5 -> 4), and saturates
// at 6 -- the rounding stated above -- but keeps the sign of a negative value
// that rounds to zero; such a nibble (8) becomes 0 here, as the oracle writes
// it.
__device__ __forceinline__ uint32_t e2m1_pack8(const float (&v)[8]) {
    uint32_t w;
    asm("{\n\t.reg .b8 c0, c1, c2, c3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 c0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 c1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 c2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 c3, %8, %7;\n\t"
        "mov.b32 %0, {c0, c1, c2, c3};\n\t}"
        : "=r"(w)
        : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]),
          "f"(v[7]));
    const uint32_t mag = w & 0x77777777u;
    const uint32_t nonzero = (mag + 0x77777777u) & 0x88888888u;   // bit 3 set where mag != 0
    return mag | (w & nonzero);
}

// Markstein's corrected quotients of two values at once with the packed
// fp32x2 operations (each lane rounds exactly as the scalar fma and mul do):
// q0 = RN(x r), e = fma(q0, -s, x) = x - q0 s (exact), u = RN(q0 + e r).
// xlo, xhi: the two values' fp32 bits; r = RN(1 / s).
__device__ __forceinline__ void quotient2(uint32_t xlo, uint32_t xhi, float r, float s,
                                          float &ulo, float &uhi) {
    uint32_t lo, hi;
    asm("{\n\t.reg .b64 x, rr, ns, q, e, u;\n\t"
        "mov.b64 x, {%2, %3};\n\t"
        "mov.b64 rr, {%4, %4};\n\t"
        "mov.b64 ns, {%5, %5};\n\t"
        "mul.rn.f32x2 q, x, rr;\n\t"
        "fma.rn.f32x2 e, q, ns, x;\n\t"
        "fma.rn.f32x2 u, e, rr, q;\n\t"
        "mov.b64 {%0, %1}, u;\n\t}"
        : "=r"(lo), "=r"(hi)
        : "r"(xlo), "r"(xhi), "r"(__float_as_uint(r)), "r"(__float_as_uint(-s)));
    ulo = __uint_as_float(lo);
    uhi = __uint_as_float(hi);
}

// One thread per block of BS values (BS / 8 chunks of 16 bytes).  MMA:
// scales in the MMA scale layout (blocks_per_row scales per row) instead of
// row-major.
//
// x / scale without a division: MXFP4 multiplies by 2^-e (exact).  NVFP4 uses
// Markstein's correction (Markstein 1990, the theorem on correctly rounded
// quotients from a correctly rounded reciprocal): with r = RN(1/s) and
// q0 = RN(x r), the residual x - q0 s is exact under fma and
// RN(q0 + (x - q0 s) r) = RN(x / s), barring underflow or overflow.  Blocks
// whose scale is subnormal (or whose reciprocal would overflow) take the IEEE
// division instead; a quotient that underflows is below 0.25 and codes to 0
// either way.
template <int KIND, bool MMA = false>
__global__ void __launch_bounds__(kThreads)
fp4_quantize_kernel(const uint4 *__restrict__ w, int64_t blocks, uint8_t *__restrict__ codes,
                    uint8_t *__restrict__ scales, const unsigned *__restrict__ amax_bits,
                    int64_t blocks_per_row = 0) {
    constexpr int BS = KIND == 0 ? 32 : 16;
    float s_t = 1.0f;
    if (KIND == 1) s_t = nv_tensor_scale(__uint_as_float(*amax_bits));
    // NVFP4: amax_b / fp32(6 s_t) by Markstein's correction from one
    // reciprocal per thread (as for the codes below), where every operand
    // stays normal; otherwise the IEEE division
    const float d6 = __fmul_rn(6.0f, s_t);
    const float r6 = __frcp_rn(d6);
    const bool d6_normal = d6 >= 0x1p-96f && d6 <= 0x1p96f;
    // The next block's loads are issued before this block is converted, so
    // each thread keeps a load in flight while it computes.
    const int64_t stride = grid_stride();
    int64_t b = thread_index();
    uint4 nxt[BS / 8];
    if (b < blocks) {
#pragma unroll
        for (int c = 0; c < BS / 8; ++c) nxt[c] = __ldg(w + b * (BS / 8) + c);
    }
    for (; b < blocks; b += stride) {
        uint32_t x[BS / 2];
#pragma unroll
        for (int c = 0; c < BS / 8; ++c) {
            x[4 * c + 0] = nxt[c].x; x[4 * c + 1] = nxt[c].y;
            x[4 * c + 2] = nxt[c].z; x[4 * c + 3] = nxt[c].w;
        }
        if (b + stride < blocks) {
#pragma unroll
            for (int c = 0; c < BS / 8; ++c) nxt[c] = __ldg(w + (b + stride) * (BS / 8) + c);
        }
        uint32_t m2 = bf16x2_absmax(x[0], x[1]);
#pragma unroll
        for (int i = 2; i < BS / 2; i += 2) m2 = bf16x2_absmax(m2, bf16x2_absmax(x[i], x[i + 1]));
        const float amax = fmaxf(bf16_bits_to_f32(m2 & 0xFFFFu), bf16_bits_to_f32(m2 >> 16));
        float scale, r;
        bool exact_div = false;
        uint32_t sb;
        if (KIND == 0) {
            int e = -127;
            if (amax > 0.0f) {
                e = ilogbf(amax) - 3;
                while (amax > ldexpf(6.0f, e)) ++e;              // the smallest such e
                if (e < -127) e = -127;
                if (e > 127) e = 127;
            }
            sb = (uint32_t)(e + 127);
            scale = ldexpf(1.0f, e);
            r = ldexpf(1.0f, -e);                                // exact: x * r = x / 2^e
        } else {
            const float q0 = __fmul_rn(amax, r6);
            const float t = d6_normal && amax >= 0x1p-100f && q0 >= 0x1p-100f
                                ? __fmaf_rn(__fmaf_rn(-q0, d6, amax), r6, q0)
                                : __fdiv_rn(amax, d6);
            sb = e4m3_round_up(t);
            scale = __fmul_rn(e4m3_value(sb), s_t);
            r = __frcp_rn(scale);
            // 2^-96 <= scale <= 2^96 keeps x, r, q0 s and the residual normal
            // for every quotient of 0.25 or more (smaller ones code to 0)
            exact_div = !(scale >= 0x1p-96f && scale <= 0x1p96f);
        }
        if (MMA) {
            const int64_t row = b <= 0xFFFFFFFFll && blocks_per_row <= 0xFFFFFFFFll
                                    ? (int64_t)((uint32_t)b / (uint32_t)blocks_per_row)
                                    : b / blocks_per_row;
            scales[mma_scale_offset(row, b - row * blocks_per_row, blocks_per_row >> 2)] =
                (uint8_t)sb;
        } else {
            scales[b] = (uint8_t)sb;
        }
        uint32_t packed[BS / 8];
#pragma unroll
        for (int g = 0; g < BS / 8; ++g) {
            float u[8];
            if (KIND == 1 && !exact_div) {
#pragma unroll
                for (int i = 0; i < 8; i += 2) {      // values i, i + 1: one bf16 pair
                    const uint32_t wv = x[(8 * g + i) / 2];
                    quotient2(wv << 16, wv & 0xFFFF0000u, r, scale, u[i], u[i + 1]);
                }
            } else {
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const uint32_t h =
                        (i & 1) ? (x[(8 * g + i) / 2] >> 16) : (x[(8 * g + i) / 2] & 0xFFFFu);
                    const float xv = bf16_bits_to_f32(h);
                    if (KIND == 0)
                        u[i] = xv * r;
                    else
                        u[i] = scale > 0.0f ? __fdiv_rn(xv, scale) : 0.0f;
                }
            }
            packed[g] = e2m1_pack8(u);
        }
        uint32_t *dst = reinterpret_cast<uint32_t *>(codes + b * (BS / 2));
#pragma unroll
        for (int i = 0; i < BS / 8; ++i) dst[i] = packed[i];
    }
}

// Row-major block scales (rows x words_per_row 32-bit words of 4 scales) into
// the MMA scale layout; rows up to the next multiple of 128 get zero scales.
__global__ void __launch_bounds__(kThreads)
fp4_scales_to_mma_kernel(const uint32_t *__restrict__ src, int64_t rows, int64_t words_per_row,
                         int64_t total, uint32_t *__restrict__ dst) {
    for (int64_t i = thread_index(); i < total; i += grid_stride()) {
        const int64_t r = i / words_per_row, jw = i - r * words_per_row;
        const uint32_t v = r < rows ? __ldg(src + i) : 0u;
        dst[mma_scale_offset(r, 4 * jw, words_per_row) >> 2] = v;
    }
}

__global__ void fp4_finish_kernel(float *tensor_scale) {
    *tensor_scale = nv_tensor_scale(*tensor_scale);
}

// One thread per 8 values (4 code bytes -> 16 bytes of bf16).
template <int KIND>
__global__ void __launch_bounds__(kThreads)
fp4_dequantize_kernel(const uint32_t *__restrict__ codes, const uint8_t *__restrict__ scales,
                      const float *__restrict__ tensor_scale, int64_t words,
                      uint4 *__restrict__ out) {
    constexpr int BS = KIND == 0 ? 32 : 16;
    const float s_t = KIND == 1 ? *tensor_scale : 1.0f;
    for (int64_t i = thread_index(); i < words; i += grid_stride()) {
        const uint32_t cw = __ldg(codes + i);
        const uint32_t sb = __ldg(scales + (i * 8) / BS);
        uint32_t o[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            float v[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const float q = e2m1_value((cw >> (4 * (2 * j + h))) & 0xFu);
                if (KIND == 0) {
                    v[h] = q * ldexpf(1.0f, (int)sb - 127);               // exact
                } else {
                    v[h] = __fmul_rn(__fmul_rn(q, e4m3_value(sb)), s_t);  // inner product exact
                }
            }
            o[j] = dev::pack_bf16x2(v[0], v[1]);
        }
        out[i] = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

unsigned grid_for(int64_t items, int per_sm = 16) {
    const int64_t cap = (int64_t)device_sm_count() * per_sm;
    const int64_t b = (items + kThreads - 1) / kThreads;
    return (unsigned)(b < 1 ? 1 : (b < cap ? b : cap));
}

// The amax pass ends with one atomicMax per CTA on a single word, which the
// L2 serialises: four CTAs per SM keep four 16-byte loads per thread in
// flight with a quarter of the atomics of the quantize grid.
unsigned amax_grid(int64_t chunks) { return grid_for(chunks, 4); }

}  // namespace

int fp4_block_size(int kind) { return kind == 0 ? 32 : 16; }

qz_status launch_fp4_quantize(const void *w, int64_t N, int64_t K, int kind, void *codes,
                              void *scales, void *tensor_scale, cudaStream_t st) {
    const int64_t blocks = N * K / fp4_block_size(kind);
    const uint4 *w4 = static_cast<const uint4 *>(w);
    if (kind == 0) {
        fp4_quantize_kernel<0><<<grid_for(blocks), kThreads, 0, st>>>(
            w4, blocks, static_cast<uint8_t *>(codes), static_cast<uint8_t *>(scales), nullptr);
        return launch_status();
    }
    unsigned *amax = static_cast<unsigned *>(tensor_scale);      // amax first, then s_t
    if (cudaMemsetAsync(amax, 0, sizeof(unsigned), st) != cudaSuccess) return QZ_ERR_CUDA;
    const int64_t chunks = N * K / 8;
    fp4_amax_kernel<<<amax_grid(chunks), kThreads, 0, st>>>(w4, chunks, amax);
    fp4_quantize_kernel<1><<<grid_for(blocks), kThreads, 0, st>>>(
        w4, blocks, static_cast<uint8_t *>(codes), static_cast<uint8_t *>(scales), amax);
    fp4_finish_kernel<<<1, 1, 0, st>>>(static_cast<float *>(tensor_scale));
    return launch_status();
}

// Activations for the W4A4 GEMM: codes row-major, scales in the MMA scale
// layout (rows beyond M zero), and for NVFP4 max |a| in *amax_word (the GEMM
// forms the tensor scale from it as qz_fp4_quantize does).
qz_status launch_fp4_quantize_mma(const void *a, int64_t M, int64_t K, int kind, void *codes,
                                  void *scales_mma, void *amax_word, cudaStream_t st) {
    const int bs = fp4_block_size(kind);
    const int64_t blocks = M * K / bs, per_row = K / bs;
    const uint4 *a4 = static_cast<const uint4 *>(a);
    if (M % 128 != 0) {
        // the last 128-row block holds padding rows: their scales must read 0
        const int64_t atom_row = (per_row / 4) * 512;
        if (cudaMemsetAsync(static_cast<uint8_t *>(scales_mma) + (M / 128) * atom_row, 0,
                            (size_t)atom_row, st) != cudaSuccess)
            return QZ_ERR_CUDA;
    }
    unsigned *amax = static_cast<unsigned *>(amax_word);
    if (kind == 0) {
        fp4_quantize_kernel<0, true><<<grid_for(blocks), kThreads, 0, st>>>(
            a4, blocks, static_cast<uint8_t *>(codes), static_cast<uint8_t *>(scales_mma), nullptr,
            per_row);
        return launch_status();
    }
    if (cudaMemsetAsync(amax, 0, sizeof(unsigned), st) != cudaSuccess) return QZ_ERR_CUDA;
    const int64_t chunks = M * K / 8;
    fp4_amax_kernel<<<amax_grid(chunks), kThreads, 0, st>>>(a4, chunks, amax);
    fp4_quantize_kernel<1, true><<<grid_for(blocks), kThreads, 0, st>>>(
        a4, blocks, static_cast<uint8_t *>(codes), static_cast<uint8_t *>(scales_mma), amax, per_row);
    return launch_status();
}

qz_status launch_fp4_scales_to_mma(const void *scales, int64_t rows, int64_t K, int kind,
                                   void *scales_mma, cudaStream_t st) {
    const int64_t words_per_row = K / fp4_block_size(kind) / 4;
    const int64_t total = ceil_div(rows, 128) * 128 * words_per_row;
    fp4_scales_to_mma_kernel<<<grid_for(total), kThreads, 0, st>>>(
        static_cast<const uint32_t *>(scales), rows, words_per_row, total,
        static_cast<uint32_t *>(scales_mma));
    return launch_status();
}

qz_status launch_fp4_dequantize(const void *codes, const void *scales, const void *tensor_scale,
                                int64_t N, int64_t K, int kind, void *w_hat, cudaStream_t st) {
    const int64_t words = N * K / 8;
    const uint32_t *c = static_cast<const uint32_t *>(codes);
    const uint8_t *s = static_cast<const uint8_t *>(scales);
    uint4 *out = static_cast<uint4 *>(w_hat);
    if (kind == 0)
        fp4_dequantize_kernel<0><<<grid_for(words), kThreads, 0, st>>>(c, s, nullptr, words, out);
    else
        fp4_dequantize_kernel<1><<<grid_for(words), kThreads, 0, st>>>(
            c, s, static_cast<const float *>(tensor_scale), words, out);
    return launch_status();
}

}  // namespace qz
