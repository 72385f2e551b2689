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

// Quantize the 8 values of one chunk and write their codes (int4: one 32-bit
// word, int8: 8 bytes) at chunk index c.
template <int BITS, bool SYM>
__device__ __forceinline__ void quantize_chunk(const float (&x)[8], float s_f, int z,
                                               uint8_t *__restrict__ codes, int64_t c) {
    const float z_f = (float)z;
    if (BITS == 4) {
        uint32_t word = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i)
            word |= (uint32_t)(quantize_one<BITS, SYM>(x[i], s_f, z_f) & 0xF) << (4 * i);
        reinterpret_cast<uint32_t *>(codes)[c] = word;
    } else {
        uint32_t lo = 0, hi = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            lo |= (uint32_t)(quantize_one<BITS, SYM>(x[i], s_f, z_f) & 0xFF) << (8 * i);
            hi |= (uint32_t)(quantize_one<BITS, SYM>(x[i + 4], s_f, z_f) & 0xFF) << (8 * i);
        }
        reinterpret_cast<uint2 *>(codes)[c] = make_uint2(lo, hi);
    }
}

// ---------------------------------------------------------------------------
// Groups of 32..256 values: LPG = g/8 lanes own one group, one 16-byte chunk
// each, and reduce its range with butterfly shuffles.  Every warp-wide load
// instruction reads 512 contiguous bytes.
// ---------------------------------------------------------------------------
constexpr int kQuantThreads = 256;
constexpr int kQuantUnroll = 4;

template <int BITS, bool SYM, int LPG>
__global__ void __launch_bounds__(kQuantThreads)
quantize_small_groups(const uint4 *__restrict__ w, int64_t total_chunks,
                      uint8_t *__restrict__ codes, uint16_t *__restrict__ scales,
                      uint8_t *__restrict__ zeros) {
    const int lane = threadIdx.x & 31;
    const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    constexpr int64_t kSpan = 32 * kQuantUnroll;
    for (int64_t base = warp * kSpan; base < total_chunks; base += nwarps * kSpan) {
        uint4 v[kQuantUnroll];
#pragma unroll
        for (int u = 0; u < kQuantUnroll; ++u) {
            const int64_t c = base + u * 32 + lane;
            v[u] = (c < total_chunks) ? dev::ld_stream_v4(w + c) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < kQuantUnroll; ++u) {
            const int64_t c = base + u * 32 + lane;
            float x[8];
            unpack8(v[u], x);
            float vmin = 0.0f, vmax = 0.0f, amax = 0.0f;
            accumulate_stats<SYM>(x, vmin, vmax, amax);
#pragma unroll
            for (int o = LPG / 2; o >= 1; o >>= 1) {
                if (SYM) {
                    amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
                } else {
                    vmin = fminf(vmin, __shfl_xor_sync(0xFFFFFFFFu, vmin, o));
                    vmax = fmaxf(vmax, __shfl_xor_sync(0xFFFFFFFFu, vmax, o));
                }
            }
            if (c >= total_chunks) continue;   // whole groups drop out together
            uint32_t s_bits; float s_f; int z;
            group_params<BITS, SYM>(vmin, vmax, amax, s_bits, s_f, z);
            quantize_chunk<BITS, SYM>(x, s_f, z, codes, c);
            if ((lane % LPG) == 0) {
                const int64_t gidx = c / LPG;
                scales[gidx] = (uint16_t)s_bits;
                if (!SYM) zeros[gidx] = (uint8_t)(int8_t)z;
            }
        }
    }
}

// ---------------------------------------------------------------------------
// Any other group size (including per-channel, g == K): one block per group,
// two passes (the second re-reads the group from L2).
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
        float vmin = 0.0f, vmax = 0.0f, amax = 0.0f;
        for (int64_t i = threadIdx.x; i < chunks_per_group; i += blockDim.x) {
            float x[8];
            unpack8(__ldcg(w + c0 + i), x);
            accumulate_stats<SYM>(x, vmin, vmax, amax);
        }
        block_reduce_stats<SYM>(vmin, vmax, amax);
        uint32_t s_bits; float s_f; int z;
        group_params<BITS, SYM>(vmin, vmax, amax, s_bits, s_f, z);
        for (int64_t i = threadIdx.x; i < chunks_per_group; i += blockDim.x) {
            float x[8];
            unpack8(__ldcs(w + c0 + i), x);
            quantize_chunk<BITS, SYM>(x, s_f, z, codes, c0 + i);
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
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; c < total_chunks; c += stride) {
        float x[8];
        unpack8(dev::ld_stream_v4(w + c), x);
        quantize_chunk<BITS, SYM>(x, s_f, z, codes, c);
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
    const int64_t cap = (int64_t)kSmCount * 16;
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
    const int grid = grid_for(total, kQuantThreads * kQuantUnroll);
    switch (g) {
    case 32:
        quantize_small_groups<BITS, SYM, 4><<<grid, kQuantThreads, 0, st>>>(src, total, c8, s16, z8);
        return launch_status();
    case 64:
        quantize_small_groups<BITS, SYM, 8><<<grid, kQuantThreads, 0, st>>>(src, total, c8, s16, z8);
        return launch_status();
    case 128:
        quantize_small_groups<BITS, SYM, 16><<<grid, kQuantThreads, 0, st>>>(src, total, c8, s16, z8);
        return launch_status();
    case 256:
        quantize_small_groups<BITS, SYM, 32><<<grid, kQuantThreads, 0, st>>>(src, total, c8, s16, z8);
        return launch_status();
    default: {
        const int64_t groups = N * (K / g);
        const int blocks = (int)std::min<int64_t>(groups, (int64_t)kSmCount * 32);
        quantize_large_groups<BITS, SYM><<<blocks, kQuantThreads, 0, st>>>(
            src, g / 8, groups, c8, s16, z8);
        return launch_status();
    }
    }
}

// ---------------------------------------------------------------------------
// Dequantize: w_hat = bf16_rne(S * (q - Z)).  The fp32 product is exact (an
// 8-bit-significand scale times an integer of at most 8 bits), so the only
// rounding is the final conversion.  One 16-byte output chunk per thread.
// ---------------------------------------------------------------------------
template <int BITS, bool SYM>
__device__ __forceinline__ int code_at(uint32_t lo, uint32_t hi, int i) {
    if (BITS == 4) {
        const uint32_t nib = (lo >> (4 * i)) & 0xF;
        return SYM ? ((int)(nib << 28) >> 28) : (int)nib;
    }
    const uint32_t word = (i < 4) ? lo : hi;
    return (int)(int8_t)((word >> (8 * (i & 3))) & 0xFF);
}

template <int BITS, bool SYM>
__global__ void __launch_bounds__(256)
dequantize_kernel(const uint8_t *__restrict__ codes, const uint16_t *__restrict__ scales,
                  const uint8_t *__restrict__ zeros, int64_t total_chunks,
                  int64_t chunks_per_group, int cpg_shift, uint4 *__restrict__ out) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; c < total_chunks; c += stride) {
        int64_t gidx;
        if (chunks_per_group == 0) gidx = 0;
        else if (cpg_shift >= 0) gidx = c >> cpg_shift;
        else gidx = c / chunks_per_group;
        const float s_f = __uint_as_float((uint32_t)__ldg(&scales[gidx]) << 16);
        int z = 0;
        if (!SYM) z = (BITS == 4) ? (int)__ldg(&zeros[gidx]) : (int)(int8_t)__ldg(&zeros[gidx]);
        uint32_t lo, hi = 0;
        if (BITS == 4) {
            lo = __ldcs(reinterpret_cast<const unsigned int *>(codes) + c);
        } else {
            const uint2 p = __ldcs(reinterpret_cast<const uint2 *>(codes) + c);
            lo = p.x; hi = p.y;
        }
        uint32_t o[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float p0 = __fmul_rn(s_f, (float)(code_at<BITS, SYM>(lo, hi, 2 * j) - z));
            const float p1 = __fmul_rn(s_f, (float)(code_at<BITS, SYM>(lo, hi, 2 * j + 1) - z));
            o[j] = dev::pack_bf16x2(p0, p1);
        }
        __stcs(out + c, make_uint4(o[0], o[1], o[2], o[3]));
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
    dequantize_kernel<BITS, SYM><<<grid_for(total, 256), 256, 0, st>>>(
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
