// qz_quantize.cu -- group-wise affine quantize + pack, and dequantize.
//
// Quantization concepts guide (HF Transformers), section "Mapping values to
// fewer bits": S = (max - min) / (q_max - q_min), Z = q_min - round(min / S),
// q = round(x / S + Z), x ~ S (q - Z); symmetric form: range [-a, a], Z = 0.
// Section "Choose granularity": one scale (and zero) per group of consecutive
// values along a row, per row, or per tensor.  Section "int8 and int4": two
// int4 codes per byte, the first in the low nibble.
//
// Fixed readings (see qz.h): the range contains 0.0; S computed in fp32 and
// stored as bf16 rounded toward +inf; S == 0 -> 1; codes clamped; rounding is
// half-to-even; quantization divides by the stored bf16 scale.
//
// Data layout: the N x K bf16 input is a flat array of N*K/8 16-byte chunks
// (8 values each).  Because K is a multiple of the group size, groups never
// straddle rows, so group j covers chunks [j*g/8, (j+1)*g/8) of the flat
// array and its scale/zero live at index j -- the same index the row-major
// [n][k/g] layout gives.
#include <cuda_runtime.h>

#include <type_traits>

#include "qz_internal.cuh"

namespace qz {
namespace {

template <int BITS, bool SYM>
struct Range {
    static constexpr int qmax = SYM ? ((1 << (BITS - 1)) - 1) : (BITS == 4 ? 15 : 127);
    static constexpr int qmin = SYM ? -qmax : (BITS == 4 ? 0 : -128);
};

// Scale and zero-point of one group from its (0-extended) min/max or absmax.
template <int BITS, bool SYM>
__device__ __forceinline__ void group_params(float vmin, float vmax, float amax,
                                             uint32_t &s_bits, float &s_f, int &z) {
    using R = Range<BITS, SYM>;
    float s;
    if (SYM) s = __fdiv_rn(amax, (float)R::qmax);
    else     s = __fdiv_rn(__fsub_rn(vmax, vmin), (float)(R::qmax - R::qmin));
    if (s == 0.0f) s = 1.0f;
    s_bits = dev::bf16_round_up_bits(s);
    s_f = __uint_as_float(s_bits << 16);
    z = SYM ? 0 : R::qmin - (int)rintf(__fdiv_rn(vmin, s_f));
}

// One code: clamp(round_half_even(x / S + Z)).
template <int BITS, bool SYM>
__device__ __forceinline__ int quantize_one(float x, float s_f, float z_f) {
    using R = Range<BITS, SYM>;
    float u = __fadd_rn(__fdiv_rn(x, s_f), z_f);
    int q = (int)rintf(u);
    return min(max(q, R::qmin), R::qmax);
}

__device__ __forceinline__ void unpack8(const uint4 &v, float (&x)[8]) {
    x[0] = dev::bf16_lo(v.x); x[1] = dev::bf16_hi(v.x);
    x[2] = dev::bf16_lo(v.y); x[3] = dev::bf16_hi(v.y);
    x[4] = dev::bf16_lo(v.z); x[5] = dev::bf16_hi(v.z);
    x[6] = dev::bf16_lo(v.w); x[7] = dev::bf16_hi(v.w);
}

template <bool SYM>
__device__ __forceinline__ void accumulate_stats(const float (&x)[8], float &vmin,
                                                 float &vmax, float &amax) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        if (SYM) amax = fmaxf(amax, fabsf(x[i]));
        else { vmin = fminf(vmin, x[i]); vmax = fmaxf(vmax, x[i]); }
    }
}

// Codes of one 8-value chunk (int4: one 32-bit word, value i in nibble i;
// int8: two words, value i in byte i), computed with the IEEE division as the
// definition states it.
template <int BITS, bool SYM>
__device__ __forceinline__ uint2 chunk_codes_exact(const float (&x)[8], float s_f, int z) {
    const float z_f = (float)z;
    if (BITS == 4) {
        uint32_t word = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i)
            word |= (uint32_t)(quantize_one<BITS, SYM>(x[i], s_f, z_f) & 0xF) << (4 * i);
        return make_uint2(word, 0u);
    }
    uint32_t lo = 0, hi = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        lo |= (uint32_t)(quantize_one<BITS, SYM>(x[i], s_f, z_f) & 0xFF) << (8 * i);
        hi |= (uint32_t)(quantize_one<BITS, SYM>(x[i + 4], s_f, z_f) & 0xFF) << (8 * i);
    }
    return make_uint2(lo, hi);
}

// Store the codes of chunk c.
template <int BITS>
__device__ __forceinline__ void store_codes(uint8_t *__restrict__ codes, int64_t c, uint2 v) {
    if (BITS == 4) reinterpret_cast<uint32_t *>(codes)[c] = v.x;
    else reinterpret_cast<uint2 *>(codes)[c] = v;
}

// Codes of one chunk without a division per value.
//
// The definition's fp32 steps, u = fl(fl(x/S) + Z) and round-half-even(u),
// give the same integer as rounding the exact x/S + Z half-to-even: x and S
// are bf16, so write x = m_x 2^a, S = m_s 2^b with integer significands below
// 256.  Then x/S - (j + 1/2) = [2 m_x 2^(a-b) - (2j + 1) m_s] / (2 m_s).  For
// a >= b the numerator is an integer; for a < b it is an integer multiple of
// 2^(a-b+1), and |x/S| >= 0.49 (needed to be near a half-way point) forces
// 2^(a-b) >= 0.49 m_s / 255.  Either way x/S + Z is exactly half-way between
// two integers (a tie, which fp32 holds exactly) or at least 2^-10 from every
// half-way point, far more than fp32 rounding moves u.
//
// Here C = 1.5 * 2^7 (int4) or 1.5 * 2^9 (int8) puts T = x/S + Z + C inside
// one binade whose grid is 2^-16 (int4: T in [191.5, 207.5]) or 2^-14 (int8:
// T in [639.5, 895.5]).  With r = 1/S rounded to nearest, x*r is within
// |x/S| 2^-24 < 2^-16 (|x/S| <= 255) of x/S, which is under half a grid step,
// so y = fma(x, r, Z + C) rounds to T itself when T is a tie, and otherwise
// lands on T's side of its nearest half-way point (2^-10 away).  Adding
// 1.5 * 2^23 - C then rounds y - C to an integer, half to even, in one fp32
// add: the result is 1.5 * 2^23 + round_half_even(x/S + Z), with the code in
// its low mantissa bits.  Only a tie at q_max + 1/2 leaves the code range
// (x/S + Z stays within [q_min - 1/2, q_max + 1/2] and q_min is even), so the
// asymmetric formats clamp at the top.  If 1/S overflows (tiny subnormal S)
// the chunk falls back to the IEEE division.
template <int BITS, bool SYM, bool CLAMP = true>
__device__ __forceinline__ uint2 chunk_codes(const float (&x)[8], float s_f, float r, int z) {
    using R = Range<BITS, SYM>;
    constexpr float kC = BITS == 4 ? 192.0f : 768.0f;
    constexpr float kRound = 12582912.0f - kC;         // 1.5 * 2^23 - C, exact
    constexpr uint32_t kTop = 0x4B400000u + (uint32_t)R::qmax;   // bits of 1.5*2^23 + q_max
    if (!(r < __int_as_float(0x7F800000))) return chunk_codes_exact<BITS, SYM>(x, s_f, z);
    const float zc = __fadd_rn((float)z, kC);          // exact (small integers)
    uint32_t b[8];
    // two values per instruction: fma.rn.f32x2 and add.rn.f32x2 round each
    // lane exactly as the scalar fma and add do
#pragma unroll
    for (int i = 0; i < 8; i += 2) {
        asm("{\n\t.reg .b64 xx, rr, zz, kk, yy, uu;\n\t"
            "mov.b64 xx, {%2, %3};\n\t"
            "mov.b64 rr, {%4, %4};\n\t"
            "mov.b64 zz, {%5, %5};\n\t"
            "mov.b64 kk, {%6, %6};\n\t"
            "fma.rn.f32x2 yy, xx, rr, zz;\n\t"
            "add.rn.f32x2 uu, yy, kk;\n\t"
            "mov.b64 {%0, %1}, uu;\n\t}"
            : "=r"(b[i]), "=r"(b[i + 1])
            : "r"(__float_as_uint(x[i])), "r"(__float_as_uint(x[i + 1])), "r"(__float_as_uint(r)),
              "r"(__float_as_uint(zc)), "r"(__float_as_uint(kRound)));
    }
    if (!SYM && CLAMP) {
#pragma unroll
        for (int i = 0; i < 8; ++i) b[i] = min(b[i], kTop);
    }
    if (BITS == 4) {
        uint32_t p[4];
#pragma unroll
        for (int j = 0; j < 4; ++j)   // byte j: code 2j low nibble, code 2j+1 high nibble
            p[j] = dev::and_or<0x0Fu>(b[2 * j], b[2 * j + 1] << 4);   // only byte 0 is used
        const uint32_t lo = dev::prmt(p[0], p[1], 0x0040u);
        const uint32_t hi = dev::prmt(p[2], p[3], 0x0040u);
        return make_uint2(dev::prmt(lo, hi, 0x5410u), 0u);
    }
    const uint32_t w0 = dev::prmt(dev::prmt(b[0], b[1], 0x0040u), dev::prmt(b[2], b[3], 0x0040u), 0x5410u);
    const uint32_t w1 = dev::prmt(dev::prmt(b[4], b[5], 0x0040u), dev::prmt(b[6], b[7], 0x0040u), 0x5410u);
    return make_uint2(w0, w1);
}

// Whether any code of a group can exceed q_max: only a value at the group's
// maximum can land on the tie q_max + 1/2 (x/S + Z is monotone in x and at
// most q_max + 1/2), so the maximum's code, computed as chunk_codes computes
// it, decides.  Groups for which this is false skip the clamp.
template <int BITS, bool SYM>
__device__ __forceinline__ bool needs_clamp(float vmax, float r, int z) {
    if (SYM) return false;                             // |x/S| <= q_max
    using R = Range<BITS, SYM>;
    constexpr float kC = BITS == 4 ? 192.0f : 768.0f;
    constexpr float kRound = 12582912.0f - kC;
    constexpr uint32_t kTop = 0x4B400000u + (uint32_t)R::qmax;
    const float zc = __fadd_rn((float)z, kC);
    // a non-finite r (the IEEE fallback) compares greater as well
    return __float_as_uint(__fadd_rn(__fmaf_rn(vmax, r, zc), kRound)) > kTop;
}

template <int BITS, bool SYM>
__device__ __forceinline__ uint2 group_chunk_codes(const float (&x)[8], float s_f, float r, int z,
                                                   bool clamp) {
    return clamp ? chunk_codes<BITS, SYM, true>(x, s_f, r, z)
                 : chunk_codes<BITS, SYM, false>(x, s_f, r, z);
}

// Three-input fp32 max/min (sm_100); exact, they select one of their inputs.
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}
__device__ __forceinline__ float fmin3(float a, float b, float c) {
    float r;
    asm("min.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// Fold the 8 values of a chunk into a running range (asymmetric: min and
// max; symmetric: max |x| in vmax).
template <bool SYM>
__device__ __forceinline__ void fold_range(const float (&x)[8], float &vmin, float &vmax) {
    if (SYM) {
        const float a = fmax3(fabsf(x[0]), fabsf(x[1]), fabsf(x[2]));
        const float b = fmax3(fabsf(x[3]), fabsf(x[4]), fabsf(x[5]));
        vmax = fmax3(vmax, fmax3(a, b, fabsf(x[6])), fabsf(x[7]));
    } else {
        vmax = fmax3(vmax, fmax3(x[0], x[1], x[2]), fmax3(x[3], x[4], fmaxf(x[5], fmaxf(x[6], x[7]))));
        vmin = fmin3(vmin, fmin3(x[0], x[1], x[2]), fmin3(x[3], x[4], fminf(x[5], fminf(x[6], x[7]))));
    }
}

// ---------------------------------------------------------------------------
// Groups of 32..256 values: each lane owns 4 consecutive 16-byte chunks (32
// values) of one group, LPG = g/32 lanes share a group and combine their
// ranges with butterfly shuffles.  The per-group work (range, S, Z, 1/S) is
// done once per 32 values, and a lane writes its int4 codes with one 16-byte
// store.  The four 16-byte loads of a lane are L1-cached so that they merge
// into full sectors.  PREFETCH (chosen when a warp makes at least
// kPrefetchIters passes): the next pass's loads are issued before this pass
// is converted, at the cost of 16 registers per thread.
// ---------------------------------------------------------------------------
constexpr int kQuantThreads = 256;
constexpr int kPrefetchIters = 4;

template <int BITS, bool SYM, int LPG, bool PREFETCH>
__global__ void __launch_bounds__(kQuantThreads)
quantize_small_groups(const uint4 *__restrict__ w, int64_t total_chunks,
                      uint8_t *__restrict__ codes, uint16_t *__restrict__ scales,
                      uint8_t *__restrict__ zeros) {
    const int lane = threadIdx.x & 31;
    const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    uint4 nxt[4];
    if (PREFETCH) {
        const int64_t c0 = warp * 128 + 4 * lane;
#pragma unroll
        for (int u = 0; u < 4; ++u)
            nxt[u] = c0 < total_chunks ? __ldg(w + c0 + u) : make_uint4(0, 0, 0, 0);
    }
    for (int64_t base = warp * 128; base < total_chunks; base += nwarps * 128) {
        const int64_t c0 = base + 4 * lane;       // total_chunks is a multiple of 4
        const bool valid = c0 < total_chunks;
        float x[4][8];
        if (PREFETCH) {
#pragma unroll
            for (int u = 0; u < 4; ++u) unpack8(nxt[u], x[u]);
            const int64_t cn = c0 + nwarps * 128;
#pragma unroll
            for (int u = 0; u < 4; ++u)
                nxt[u] = cn < total_chunks ? __ldg(w + cn + u) : make_uint4(0, 0, 0, 0);
        } else {
#pragma unroll
            for (int u = 0; u < 4; ++u)
                unpack8(valid ? __ldg(w + c0 + u) : make_uint4(0, 0, 0, 0), x[u]);
        }
        float vmin = 0.0f, vmax = 0.0f;           // the range always contains 0
#pragma unroll
        for (int u = 0; u < 4; ++u) fold_range<SYM>(x[u], vmin, vmax);
#pragma unroll
        for (int o = LPG / 2; o >= 1; o >>= 1) {
            vmax = fmaxf(vmax, __shfl_xor_sync(0xFFFFFFFFu, vmax, o));
            if (!SYM) vmin = fminf(vmin, __shfl_xor_sync(0xFFFFFFFFu, vmin, o));
        }
        if (!valid) continue;                     // whole groups drop out together
        uint32_t s_bits; float s_f; int z;
        group_params<BITS, SYM>(vmin, vmax, vmax, s_bits, s_f, z);
        const float r = __frcp_rn(s_f);
        uint2 cw[4];
        const bool clamp = needs_clamp<BITS, SYM>(vmax, r, z);
#pragma unroll
        for (int u = 0; u < 4; ++u) cw[u] = group_chunk_codes<BITS, SYM>(x[u], s_f, r, z, clamp);
        if (BITS == 4) {
            reinterpret_cast<uint4 *>(codes)[c0 >> 2] = make_uint4(cw[0].x, cw[1].x, cw[2].x, cw[3].x);
        } else {
            uint4 *dst = reinterpret_cast<uint4 *>(codes) + (c0 >> 1);
            dst[0] = make_uint4(cw[0].x, cw[0].y, cw[1].x, cw[1].y);
            dst[1] = make_uint4(cw[2].x, cw[2].y, cw[3].x, cw[3].y);
        }
        if ((lane % LPG) == 0) {
            const int64_t gidx = c0 / (4 * LPG);
            scales[gidx] = (uint16_t)s_bits;
            if (!SYM) zeros[gidx] = (uint8_t)(int8_t)z;
        }
    }
}

// ---------------------------------------------------------------------------
// Groups of up to 65536 values (per-channel rows included): one block per
// group holds the whole group in registers (at most 8 chunks per thread), so
// the weights are read from HBM once; the range is combined with shuffles and
// one shared-memory step.
// ---------------------------------------------------------------------------
constexpr int kRowChunksPerThread = 8;

template <int BITS, bool SYM>
__global__ void __launch_bounds__(1024)
quantize_groups_block(const uint4 *__restrict__ w, int cpg, int64_t num_groups,
                      uint8_t *__restrict__ codes, uint16_t *__restrict__ scales,
                      uint8_t *__restrict__ zeros) {
    __shared__ float red[64];
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
    for (int64_t gidx = blockIdx.x; gidx < num_groups; gidx += gridDim.x) {
        const int64_t c0 = gidx * cpg;
        uint4 v[kRowChunksPerThread];
        float vmin = 0.0f, vmax = 0.0f;           // the range always contains 0
#pragma unroll
        for (int i = 0; i < kRowChunksPerThread; ++i) {
            const int c = threadIdx.x + i * blockDim.x;
            if (c < cpg) {
                v[i] = __ldcs(w + c0 + c);
                float x[8];
                unpack8(v[i], x);
                fold_range<SYM>(x, vmin, vmax);
            }
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) {
            vmax = fmaxf(vmax, __shfl_xor_sync(0xFFFFFFFFu, vmax, o));
            if (!SYM) vmin = fminf(vmin, __shfl_xor_sync(0xFFFFFFFFu, vmin, o));
        }
        if (lane == 0) { red[wid] = vmax; red[32 + wid] = vmin; }
        __syncthreads();
        vmax = red[0];
        vmin = red[32];
        for (int i = 1; i < nw; ++i) { vmax = fmaxf(vmax, red[i]); vmin = fminf(vmin, red[32 + i]); }
        __syncthreads();                          // red[] is reused by the next group
        uint32_t s_bits; float s_f; int z;
        group_params<BITS, SYM>(vmin, vmax, vmax, s_bits, s_f, z);
        const float r = __frcp_rn(s_f);
        const bool clamp = needs_clamp<BITS, SYM>(vmax, r, z);
#pragma unroll
        for (int i = 0; i < kRowChunksPerThread; ++i) {
            const int c = threadIdx.x + i * blockDim.x;
            if (c < cpg) {
                float x[8];
                unpack8(v[i], x);
                store_codes<BITS>(codes, c0 + c, group_chunk_codes<BITS, SYM>(x, s_f, r, z, clamp));
            }
        }
        if (threadIdx.x == 0) {
            scales[gidx] = (uint16_t)s_bits;
            if (!SYM) zeros[gidx] = (uint8_t)(int8_t)z;
        }
    }
}

// ---------------------------------------------------------------------------
// Groups of more than 65536 values: one block per group, two passes (the
// second re-reads the group from L2).
// ---------------------------------------------------------------------------
template <bool SYM>
__device__ __forceinline__ void block_reduce_stats(float &vmin, float &vmax, float &amax) {
    __shared__ float red[3][32];
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
        vmin = fminf(vmin, __shfl_xor_sync(0xFFFFFFFFu, vmin, o));
        vmax = fmaxf(vmax, __shfl_xor_sync(0xFFFFFFFFu, vmax, o));
        amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
    }
    if (lane == 0) { red[0][wid] = vmin; red[1][wid] = vmax; red[2][wid] = amax; }
    __syncthreads();
    const int nw = blockDim.x >> 5;
    vmin = 0.0f; vmax = 0.0f; amax = 0.0f;
    for (int i = 0; i < nw; ++i) {
        vmin = fminf(vmin, red[0][i]);
        vmax = fmaxf(vmax, red[1][i]);
        amax = fmaxf(amax, red[2][i]);
    }
    __syncthreads();
}

template <int BITS, bool SYM>
__global__ void __launch_bounds__(kQuantThreads)
quantize_large_groups(const uint4 *__restrict__ w, int64_t chunks_per_group,
                      int64_t num_groups, uint8_t *__restrict__ codes,
                      uint16_t *__restrict__ scales, uint8_t *__restrict__ zeros) {
    for (int64_t gidx = blockIdx.x; gidx < num_groups; gidx += gridDim.x) {
        const int64_t c0 = gidx * chunks_per_group;
        float vmin = 0.0f, vmax = 0.0f;           // the range always contains 0
        for (int64_t i = threadIdx.x; i < chunks_per_group; i += blockDim.x) {
            float x[8];
            unpack8(__ldcg(w + c0 + i), x);
            fold_range<SYM>(x, vmin, vmax);
        }
        float amax = vmax;
        block_reduce_stats<SYM>(vmin, vmax, amax);
        uint32_t s_bits; float s_f; int z;
        group_params<BITS, SYM>(vmin, vmax, amax, s_bits, s_f, z);
        const float r = __frcp_rn(s_f);
        const bool clamp = needs_clamp<BITS, SYM>(vmax, r, z);
        for (int64_t i = threadIdx.x; i < chunks_per_group; i += blockDim.x) {
            float x[8];
            unpack8(__ldcs(w + c0 + i), x);
            store_codes<BITS>(codes, c0 + i, group_chunk_codes<BITS, SYM>(x, s_f, r, z, clamp));
        }
        if (threadIdx.x == 0) {
            scales[gidx] = (uint16_t)s_bits;
            if (!SYM) zeros[gidx] = (uint8_t)(int8_t)z;
        }
    }
}

// ---------------------------------------------------------------------------
// Per-tensor: (1) range of the whole matrix into a 2-word workspace with
// atomic max on non-negative fp32 bit patterns (order-independent, exact),
// (2) quantize with the single scale, (3) publish scale/zero and clear the
// workspace for the next call.
// ---------------------------------------------------------------------------
template <bool SYM>
__global__ void __launch_bounds__(kQuantThreads)
tensor_range(const uint4 *__restrict__ w, int64_t total_chunks, uint32_t *__restrict__ ws) {
    float vmin = 0.0f, vmax = 0.0f, amax = 0.0f;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; c < total_chunks; c += stride) {
        float x[8];
        unpack8(dev::ld_stream_v4(w + c), x);
        accumulate_stats<SYM>(x, vmin, vmax, amax);
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
        vmin = fminf(vmin, __shfl_xor_sync(0xFFFFFFFFu, vmin, o));
        vmax = fmaxf(vmax, __shfl_xor_sync(0xFFFFFFFFu, vmax, o));
        amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
    }
    // The values are >= 0; fabsf also clears the sign of a -0.0 (from
    // negating +0.0 or from fmaxf(+0, -0)), whose bit pattern would otherwise
    // compare above every positive value.
    if ((threadIdx.x & 31) == 0) {
        if (SYM) {
            atomicMax(&ws[0], __float_as_uint(fabsf(amax)));
        } else {
            atomicMax(&ws[0], __float_as_uint(fabsf(vmax)));
            atomicMax(&ws[1], __float_as_uint(fabsf(vmin)));
        }
    }
}

template <int BITS, bool SYM>
__device__ __forceinline__ void tensor_params(const uint32_t *ws, uint32_t &s_bits,
                                              float &s_f, int &z) {
    const float a = __uint_as_float(__ldcg(&ws[0]));
    const float vmax = SYM ? 0.0f : a;
    const float vmin = SYM ? 0.0f : -__uint_as_float(__ldcg(&ws[1]));
    group_params<BITS, SYM>(vmin, vmax, a, s_bits, s_f, z);
}

template <int BITS, bool SYM>
__global__ void __launch_bounds__(kQuantThreads)
tensor_quantize(const uint4 *__restrict__ w, int64_t total_chunks,
                const uint32_t *__restrict__ ws, uint8_t *__restrict__ codes) {
    uint32_t s_bits; float s_f; int z;
    tensor_params<BITS, SYM>(ws, s_bits, s_f, z);
    const float r = __frcp_rn(s_f);
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; c < total_chunks; c += stride) {
        float x[8];
        unpack8(dev::ld_stream_v4(w + c), x);
        store_codes<BITS>(codes, c, chunk_codes<BITS, SYM>(x, s_f, r, z));
    }
}

template <int BITS, bool SYM>
__global__ void tensor_finish(uint32_t *__restrict__ ws, uint16_t *__restrict__ scales,
                              uint8_t *__restrict__ zeros) {
    uint32_t s_bits; float s_f; int z;
    tensor_params<BITS, SYM>(ws, s_bits, s_f, z);
    scales[0] = (uint16_t)s_bits;
    if (!SYM) zeros[0] = (uint8_t)(int8_t)z;
    ws[0] = 0u;
    ws[1] = 0u;
}

int grid_for(int64_t work_items, int per_block) {
    int64_t b = ceil_div(work_items, per_block);
    const int64_t cap = (int64_t)device_sm_count() * 16;
    if (b > cap) b = cap;
    if (b < 1) b = 1;
    return (int)b;
}

template <int BITS, bool SYM>
qz_status quantize_typed(const void *w, int64_t N, int64_t K, int64_t g, void *codes,
                         void *scales, void *zeros, void *workspace, cudaStream_t st) {
    const int64_t total = N * K / 8;
    auto *src = static_cast<const uint4 *>(w);
    auto *c8 = static_cast<uint8_t *>(codes);
    auto *s16 = static_cast<uint16_t *>(scales);
    auto *z8 = static_cast<uint8_t *>(zeros);
    if (g == 0) {
        auto *ws = static_cast<uint32_t *>(workspace);
        tensor_range<SYM><<<grid_for(total, kQuantThreads), kQuantThreads, 0, st>>>(src, total, ws);
        tensor_quantize<BITS, SYM><<<grid_for(total, kQuantThreads), kQuantThreads, 0, st>>>(
            src, total, ws, c8);
        tensor_finish<BITS, SYM><<<1, 1, 0, st>>>(ws, s16, z8);
        return launch_status();
    }
    const int grid = grid_for(total, kQuantThreads * 4);
    // passes per warp: each pass of a warp covers 128 chunks
    const bool prefetch = total >= (int64_t)grid * (kQuantThreads / 32) * 128 * kPrefetchIters;
    auto small = [&](auto lpg) {
        constexpr int LPG = decltype(lpg)::value;
        if (prefetch)
            quantize_small_groups<BITS, SYM, LPG, true><<<grid, kQuantThreads, 0, st>>>(
                src, total, c8, s16, z8);
        else
            quantize_small_groups<BITS, SYM, LPG, false><<<grid, kQuantThreads, 0, st>>>(
                src, total, c8, s16, z8);
        return launch_status();
    };
    switch (g) {
    case 32: return small(std::integral_constant<int, 1>{});
    case 64: return small(std::integral_constant<int, 2>{});
    case 128: return small(std::integral_constant<int, 4>{});
    case 256: return small(std::integral_constant<int, 8>{});
    default:
        break;
    }
    const int64_t groups = N * (K / g);
    const int64_t cpg = g / 8;
    if (cpg <= (int64_t)kRowChunksPerThread * 1024) {
        const int threads = (int)ceil_div(ceil_div(cpg, kRowChunksPerThread), 32) * 32;
        const int per_sm = std::max(1, 2048 / threads);
        const int blocks = (int)std::min<int64_t>(groups, (int64_t)device_sm_count() * per_sm * 4);
        quantize_groups_block<BITS, SYM><<<blocks, threads, 0, st>>>(src, (int)cpg, groups, c8,
                                                                      s16, z8);
        return launch_status();
    }
    const int blocks = (int)std::min<int64_t>(groups, (int64_t)device_sm_count() * 32);
    quantize_large_groups<BITS, SYM><<<blocks, kQuantThreads, 0, st>>>(src, cpg, groups, c8,
                                                                        s16, z8);
    return launch_status();
}

// ---------------------------------------------------------------------------
// Dequantize: w_hat = bf16_rne(S * (q - Z)).  The product of the bf16 scale
// (8-bit significand) and q - Z (at most 9 bits) is exact in fp32, so the
// only rounding is one round-to-nearest-even to bf16.  No integer-to-float
// conversion is used:
//   int4: byte i of the code word and of (word >> 4) hold codes 2i and 2i+1
//         in their low nibbles; one PRMT + LOP3 builds bf16(128 + q) for the
//         pair, sub.rn.bf16x2 removes (128 + Z) exactly and mul.rn.bf16x2 by
//         the scale rounds the product once (symmetric codes are first made
//         unsigned by XOR 8, with 8 added to Z).
//   int8: the byte (XOR 0x80) is placed in the mantissa of 2^23; one packed
//         fp32 add gives q - Z exactly, a packed fp32 multiply the exact
//         product, cvt.rn.bf16x2 rounds it once.
// One 16-byte output chunk (8 values) per thread per step.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t dq_pair_u4(uint32_t w, uint32_t w4, int i, uint32_t s2,
                                               uint32_t z2) {
    const uint32_t t = dev::prmt(w, w4, (uint32_t)i | ((uint32_t)(4 + i) << 8));
    const uint32_t x = dev::and_or<0x000F000Fu>(t, 0x43004300u);  // bf16(128 + q)
    return dev::bf16x2_mul(dev::bf16x2_sub(x, z2), s2);
}

__device__ __forceinline__ uint32_t dq_pair_i8(uint32_t word, int i, float off, float s) {
    // bytes 2i and 2i+1 (i = 0, 1) of `word` (already XORed with 0x80808080)
    const float f0 = __uint_as_float(dev::prmt(word, 0x4B000000u, (uint32_t)(2 * i) | 0x7540u));
    const float f1 = __uint_as_float(dev::prmt(word, 0x4B000000u, (uint32_t)(2 * i + 1) | 0x7540u));
    const float p0 = __fmul_rn(__fadd_rn(f0, off), s);             // q - Z exact, exact product
    const float p1 = __fmul_rn(__fadd_rn(f1, off), s);
    return dev::pack_bf16x2(p0, p1);
}

// Output chunk c (8 values) of the dequantized matrix from its code word(s).
template <int BITS, bool SYM>
__device__ __forceinline__ uint4 dequant_chunk(uint32_t w_lo, uint32_t w_hi,
                                               const uint16_t *__restrict__ scales,
                                               const uint8_t *__restrict__ zeros, int64_t gidx) {
    const uint32_t s_bits = __ldg(&scales[gidx]);
    uint32_t o[4];
    if (BITS == 4) {
        uint32_t w = w_lo;
        const uint32_t zb = SYM ? 8u : (uint32_t)__ldg(&zeros[gidx]);
        if (SYM) w ^= 0x88888888u;                              // two's complement -> q + 8
        const uint32_t s2 = s_bits * 0x00010001u;
        const uint32_t z2 = (0x4300u + zb) * 0x00010001u;
        const uint32_t w4 = w >> 4;
#pragma unroll
        for (int i = 0; i < 4; ++i) o[i] = dq_pair_u4(w, w4, i, s2, z2);
    } else {
        const int z = SYM ? 0 : (int)(int8_t)__ldg(&zeros[gidx]);
        const float off = -(8388736.0f + (float)z);              // -(2^23 + 128 + Z), exact
        const float s_f = __uint_as_float(s_bits << 16);
        const uint32_t lo = w_lo ^ 0x80808080u, hi = w_hi ^ 0x80808080u;
        o[0] = dq_pair_i8(lo, 0, off, s_f);
        o[1] = dq_pair_i8(lo, 1, off, s_f);
        o[2] = dq_pair_i8(hi, 0, off, s_f);
        o[3] = dq_pair_i8(hi, 1, off, s_f);
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}

__device__ __forceinline__ int64_t group_of_chunk(int64_t c, int64_t chunks_per_group,
                                                  int cpg_shift) {
    if (chunks_per_group == 0) return 0;
    return cpg_shift >= 0 ? (c >> cpg_shift) : c / chunks_per_group;
}

// A warp dequantizes 128 consecutive chunks per iteration, lane l taking
// chunks base + 32 i + l (i = 0..3): its four code loads are issued before any
// arithmetic (four loads in flight per thread), and every load and store
// instruction of the warp covers contiguous memory.
template <int BITS, bool SYM>
__global__ void __launch_bounds__(256)
dequantize_kernel(const uint8_t *__restrict__ codes, const uint16_t *__restrict__ scales,
                  const uint8_t *__restrict__ zeros, int64_t total_chunks,
                  int64_t chunks_per_group, int cpg_shift, uint4 *__restrict__ out) {
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x / 32);
    const int64_t warp = (int64_t)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
    for (int64_t base = warp * 128; base < total_chunks; base += warps * 128) {
        uint32_t wl[4], wh[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int64_t c = base + 32 * i + lane;
            wl[i] = wh[i] = 0u;
            if (c < total_chunks) {
                if (BITS == 4) {
                    wl[i] = __ldcs(reinterpret_cast<const unsigned int *>(codes) + c);
                } else {
                    const uint2 v = __ldcs(reinterpret_cast<const uint2 *>(codes) + c);
                    wl[i] = v.x; wh[i] = v.y;
                }
            }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int64_t c = base + 32 * i + lane;
            if (c < total_chunks)
                __stcs(out + c, dequant_chunk<BITS, SYM>(wl[i], wh[i], scales, zeros,
                                                         group_of_chunk(c, chunks_per_group, cpg_shift)));
        }
    }
}

template <int BITS, bool SYM>
qz_status dequantize_typed(const void *codes, const void *scales, const void *zeros,
                           int64_t N, int64_t K, int64_t g, void *w_hat, cudaStream_t st) {
    const int64_t total = N * K / 8;
    const int64_t cpg = (g == 0) ? 0 : g / 8;
    int shift = -1;
    if (cpg > 0 && (cpg & (cpg - 1)) == 0) {
        shift = 0;
        while ((int64_t(1) << shift) < cpg) ++shift;
    }
    dequantize_kernel<BITS, SYM><<<grid_for(ceil_div(total, 4), 256), 256, 0, st>>>(
        static_cast<const uint8_t *>(codes), static_cast<const uint16_t *>(scales),
        static_cast<const uint8_t *>(zeros), total, cpg, shift, static_cast<uint4 *>(w_hat));
    return launch_status();
}

}  // namespace

size_t quantize_workspace_bytes(int64_t group_size) {
    return group_size == 0 ? 2 * sizeof(uint32_t) : 0;
}

qz_status launch_quantize_pack(const void *w, int64_t N, int64_t K, int bits, int symmetric,
                               int64_t g, void *codes, void *scales, void *zeros,
                               void *workspace, cudaStream_t st) {
    if (bits == 4 && !symmetric) return quantize_typed<4, false>(w, N, K, g, codes, scales, zeros, workspace, st);
    if (bits == 4 && symmetric)  return quantize_typed<4, true>(w, N, K, g, codes, scales, zeros, workspace, st);
    if (bits == 8 && !symmetric) return quantize_typed<8, false>(w, N, K, g, codes, scales, zeros, workspace, st);
    return quantize_typed<8, true>(w, N, K, g, codes, scales, zeros, workspace, st);
}

qz_status launch_dequantize(const void *codes, const void *scales, const void *zeros,
                            int64_t N, int64_t K, int bits, int symmetric, int64_t g,
                            void *w_hat, cudaStream_t st) {
    if (bits == 4 && !symmetric) return dequantize_typed<4, false>(codes, scales, zeros, N, K, g, w_hat, st);
    if (bits == 4 && symmetric)  return dequantize_typed<4, true>(codes, scales, zeros, N, K, g, w_hat, st);
    if (bits == 8 && !symmetric) return dequantize_typed<8, false>(codes, scales, zeros, N, K, g, w_hat, st);
    return dequantize_typed<8, true>(codes, scales, zeros, N, K, g, w_hat, st);
}

}  // namespace qz
