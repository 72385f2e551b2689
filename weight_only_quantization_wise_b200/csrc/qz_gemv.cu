// qz_gemv.cu -- weight-only decode GEMV: y (M x N) = a (M x K) * w_hat^T, M <= 16.
//
// Quantization concepts guide, "Quantize weights or activations": weight-only
// methods keep activations in bf16 and dequantize the weights to the compute
// dtype before each matmul; when decoding one token at a time the GPU spends
// the step reading weights, so 4-bit weights move a quarter of the bytes.
// GPTQ explainer: the gain needs kernels that dequantize inside the matmul.
//
// Design (one warp = one 16-row tile of W over a K range):
//   * Each lane (g = lane/4, t = lane%4) streams 16 bytes of packed codes from
//     row g and from row g+8 per 128-wide K block (its 32 consecutive k), so a
//     warp-wide load covers 64 contiguous bytes of 8 rows.
//   * Codes are dequantized in registers to bf16 pairs exactly as
//     qz_dequantize forms them: an OR builds bf16(128 + q) for two nibbles,
//     sub.rn.bf16x2 removes (128 + Z) exactly, mul.rn.bf16x2 by the bf16
//     scale rounds S*(q - Z) once to nearest-even.  A byte of codes yields the
//     pairs (q_j, q_{j+4}), so the K axis is permuted consistently for both
//     MMA operands; the activations are permuted to match with PRMT.
//   * The pairs are the A operand (16 rows x 16 k) of mma.sync m16n8k16 with
//     fp32 accumulation; the activations (tokens as the 8 columns) are the B
//     operand.  For M > 8 a second MMA covers tokens 8..15.
//   * Split-K: blockIdx.y selects a K range.  With more than one split each
//     warp writes its fp32 partial tile into the workspace and bumps a
//     per-tile counter; the last warp to arrive adds the partials in split
//     order (deterministic), writes bf16 y and resets the counter to zero.
#include <cuda_runtime.h>

#include "qz_internal.cuh"

namespace qz {
namespace {

constexpr int kWarpsPerCta = 4;
constexpr int kThreads = 32 * kWarpsPerCta;

// bf16 pair (nibble j, nibble j+4) of a code word, dequantized:
// bf16_rne(S * (q - Z)) in each half.
__device__ __forceinline__ uint32_t dequant_pair_u4(uint32_t word, int j, uint32_t s2,
                                                    uint32_t z2) {
    const uint32_t x = ((word >> (4 * j)) & 0x000F000Fu) | 0x43004300u;  // bf16(128+q)
    return dev::bf16x2_mul(dev::bf16x2_sub(x, z2), s2);
}

// Activation operand for code word i (k = 8i..8i+7 of the lane's 32) and
// half h: b0 = (x[8i+2h], x[8i+2h+4]), b1 = (x[8i+2h+1], x[8i+2h+5]).
__device__ __forceinline__ void act_operand(const uint32_t (&x)[16], int i, int h,
                                            uint32_t &b0, uint32_t &b1) {
    const uint32_t lo = x[4 * i + h];       // k = 8i+2h, 8i+2h+1
    const uint32_t hi = x[4 * i + h + 2];   // k = 8i+2h+4, 8i+2h+5
    b0 = dev::prmt(lo, hi, 0x5410);
    b1 = dev::prmt(lo, hi, 0x7632);
}

__device__ __forceinline__ void load_act(const uint16_t *__restrict__ a, int K, int tok,
                                         int M, int k0, uint32_t (&x)[16]) {
    if (tok < M) {
        const uint4 *p = reinterpret_cast<const uint4 *>(a + (int64_t)tok * K + k0);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint4 v = __ldg(p + q);
            x[4 * q + 0] = v.x; x[4 * q + 1] = v.y; x[4 * q + 2] = v.z; x[4 * q + 3] = v.w;
        }
    } else {
#pragma unroll
        for (int q = 0; q < 16; ++q) x[q] = 0u;
    }
}

// Epilogue shared by the W4 and W8 kernels: acc[mb][j] holds
// y[tok = 8mb + 2t + (j&1)][row = n0 + g + 8(j>>1)].
template <int MB>
__device__ __forceinline__ void gemv_epilogue(float (&acc)[MB][4], int M, int N, int n0,
                                              int lane, int split, int splits, int tile,
                                              uint16_t *__restrict__ y,
                                              float *__restrict__ partials,
                                              uint32_t *__restrict__ counters) {
    const int g = lane >> 2, t = lane & 3;
    if (splits == 1) {
#pragma unroll
        for (int mb = 0; mb < MB; ++mb)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int row = n0 + g + 8 * (j >> 1);
                const int tok = 8 * mb + 2 * t + (j & 1);
                if (row < N && tok < M)
                    y[(int64_t)tok * N + row] = (uint16_t)dev::f32_to_bf16_rne(acc[mb][j]);
            }
        return;
    }
    const int64_t MN = (int64_t)M * N;
#pragma unroll
    for (int mb = 0; mb < MB; ++mb)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int row = n0 + g + 8 * (j >> 1);
            const int tok = 8 * mb + 2 * t + (j & 1);
            if (row < N && tok < M)
                __stcg(&partials[split * MN + (int64_t)tok * N + row], acc[mb][j]);
        }
    __threadfence();
    __syncwarp();
    uint32_t prev = 0;
    if (lane == 0) prev = atomicAdd(&counters[tile], 1u);
    prev = __shfl_sync(0xFFFFFFFFu, prev, 0);
    if (prev != (uint32_t)(splits - 1)) return;
    __threadfence();
#pragma unroll
    for (int mb = 0; mb < MB; ++mb)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int row = n0 + g + 8 * (j >> 1);
            const int tok = 8 * mb + 2 * t + (j & 1);
            if (row < N && tok < M) {
                float s = 0.0f;
                for (int sp = 0; sp < splits; ++sp)
                    s += __ldcg(&partials[sp * MN + (int64_t)tok * N + row]);
                y[(int64_t)tok * N + row] = (uint16_t)dev::f32_to_bf16_rne(s);
            }
        }
    if (lane == 0) counters[tile] = 0u;
}

// ---------------------------------------------------------------------------
// W4A16
// ---------------------------------------------------------------------------
template <int MB>
__global__ void __launch_bounds__(kThreads)
w4a16_gemv_kernel(const uint16_t *__restrict__ a, const uint8_t *__restrict__ codes,
                  const uint16_t *__restrict__ scales, const uint8_t *__restrict__ zeros,
                  int M, int N, int K, int group_size, int group_shift,
                  uint16_t *__restrict__ y, float *__restrict__ partials,
                  uint32_t *__restrict__ counters, int splits) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, t = lane & 3;
    const int tile = blockIdx.x * kWarpsPerCta + warp;
    const int n0 = tile * 16;
    if (n0 >= N) return;
    const int split = blockIdx.y;
    const int KB = K / 128;
    const int kb_begin = (int)((int64_t)split * KB / splits);
    const int kb_end = (int)((int64_t)(split + 1) * KB / splits);
    const int r0 = n0 + g, r1 = n0 + g + 8;
    const bool v0 = r0 < N, v1 = r1 < N;
    const int gpr = K / group_size;
    const uint8_t *row0 = codes + (int64_t)r0 * (K / 2) + t * 16;
    const uint8_t *row1 = codes + (int64_t)r1 * (K / 2) + t * 16;

    float acc[MB][4];
#pragma unroll
    for (int mb = 0; mb < MB; ++mb)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[mb][j] = 0.0f;

    const uint4 zero4 = make_uint4(0, 0, 0, 0);
    uint4 nw0 = zero4, nw1 = zero4;
    if (kb_begin < kb_end) {
        if (v0) nw0 = dev::ld_stream_v4(row0 + kb_begin * 64);
        if (v1) nw1 = dev::ld_stream_v4(row1 + kb_begin * 64);
    }
    for (int kb = kb_begin; kb < kb_end; ++kb) {
        const uint4 w0 = nw0, w1 = nw1;
        if (kb + 1 < kb_end) {
            if (v0) nw0 = dev::ld_stream_v4(row0 + (kb + 1) * 64);
            if (v1) nw1 = dev::ld_stream_v4(row1 + (kb + 1) * 64);
        }
        const int k0 = kb * 128 + t * 32;
        const int gi = group_shift >= 0 ? (k0 >> group_shift) : (k0 / group_size);
        uint32_t s0 = 0, s1 = 0, z0 = 0, z1 = 0;
        if (v0) { s0 = __ldg(&scales[(int64_t)r0 * gpr + gi]); z0 = __ldg(&zeros[(int64_t)r0 * gpr + gi]); }
        if (v1) { s1 = __ldg(&scales[(int64_t)r1 * gpr + gi]); z1 = __ldg(&zeros[(int64_t)r1 * gpr + gi]); }
        const uint32_t s2_0 = s0 | (s0 << 16), s2_1 = s1 | (s1 << 16);
        const uint32_t z2_0 = (0x4300u + z0) * 0x00010001u, z2_1 = (0x4300u + z1) * 0x00010001u;

        uint32_t x[MB][16];
#pragma unroll
        for (int mb = 0; mb < MB; ++mb) load_act(a, K, 8 * mb + g, M, k0, x[mb]);

        const uint32_t wa[4] = {w0.x, w0.y, w0.z, w0.w};
        const uint32_t wb[4] = {w1.x, w1.y, w1.z, w1.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const uint32_t a0 = dequant_pair_u4(wa[i], 2 * h, s2_0, z2_0);
                const uint32_t a1 = dequant_pair_u4(wb[i], 2 * h, s2_1, z2_1);
                const uint32_t a2 = dequant_pair_u4(wa[i], 2 * h + 1, s2_0, z2_0);
                const uint32_t a3 = dequant_pair_u4(wb[i], 2 * h + 1, s2_1, z2_1);
#pragma unroll
                for (int mb = 0; mb < MB; ++mb) {
                    uint32_t b0, b1;
                    act_operand(x[mb], i, h, b0, b1);
                    dev::mma_bf16_16816(acc[mb], a0, a1, a2, a3, b0, b1);
                }
            }
        }
    }
    gemv_epilogue<MB>(acc, M, N, n0, lane, split, splits, tile, y, partials, counters);
}

// ---------------------------------------------------------------------------
// W8A16 (symmetric per-channel): w_hat = bf16_rne(S * q).  A code byte is
// widened exactly: bits 0x4B000000 | (q ^ 0x80) is the fp32 2^23 + q + 128.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float code_i8_as_f32(uint32_t word_xor80, int byte) {
    // byte `byte` of the word into the low byte of fp32 2^23 (0x4B000000)
    const uint32_t sel = (uint32_t)byte | 0x7540u;
    const uint32_t bits = dev::prmt(word_xor80, 0x4B000000u, sel);
    return __fsub_rn(__uint_as_float(bits), 8388736.0f);   // - (2^23 + 128)
}

// bf16 pair (code c_j, code c_{j+4}) of 8 consecutive codes held in words
// lo (c0..c3) and hi (c4..c7), already XORed with 0x80808080.
__device__ __forceinline__ uint32_t dequant_pair_i8(uint32_t lo, uint32_t hi, int j, float s) {
    const float q0 = code_i8_as_f32(lo, j);
    const float q1 = code_i8_as_f32(hi, j);
    return dev::pack_bf16x2(__fmul_rn(q0, s), __fmul_rn(q1, s));
}

template <int MB>
__global__ void __launch_bounds__(kThreads)
w8a16_gemv_kernel(const uint16_t *__restrict__ a, const uint8_t *__restrict__ codes,
                  const uint16_t *__restrict__ scales, int M, int N, int K,
                  uint16_t *__restrict__ y, float *__restrict__ partials,
                  uint32_t *__restrict__ counters, int splits) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, t = lane & 3;
    const int tile = blockIdx.x * kWarpsPerCta + warp;
    const int n0 = tile * 16;
    if (n0 >= N) return;
    const int split = blockIdx.y;
    const int KB = K / 128;
    const int kb_begin = (int)((int64_t)split * KB / splits);
    const int kb_end = (int)((int64_t)(split + 1) * KB / splits);
    const int r0 = n0 + g, r1 = n0 + g + 8;
    const bool v0 = r0 < N, v1 = r1 < N;
    const uint8_t *row0 = codes + (int64_t)r0 * K + t * 32;
    const uint8_t *row1 = codes + (int64_t)r1 * K + t * 32;
    const float sf0 = v0 ? __uint_as_float((uint32_t)__ldg(&scales[r0]) << 16) : 0.0f;
    const float sf1 = v1 ? __uint_as_float((uint32_t)__ldg(&scales[r1]) << 16) : 0.0f;

    float acc[MB][4];
#pragma unroll
    for (int mb = 0; mb < MB; ++mb)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[mb][j] = 0.0f;

    const uint4 zero4 = make_uint4(0, 0, 0, 0);
    uint4 n0a = zero4, n0b = zero4, n1a = zero4, n1b = zero4;
    if (kb_begin < kb_end) {
        if (v0) { n0a = dev::ld_stream_v4(row0 + kb_begin * 128); n0b = dev::ld_stream_v4(row0 + kb_begin * 128 + 16); }
        if (v1) { n1a = dev::ld_stream_v4(row1 + kb_begin * 128); n1b = dev::ld_stream_v4(row1 + kb_begin * 128 + 16); }
    }
    for (int kb = kb_begin; kb < kb_end; ++kb) {
        const uint4 c0a = n0a, c0b = n0b, c1a = n1a, c1b = n1b;
        if (kb + 1 < kb_end) {
            const int off = (kb + 1) * 128;
            if (v0) { n0a = dev::ld_stream_v4(row0 + off); n0b = dev::ld_stream_v4(row0 + off + 16); }
            if (v1) { n1a = dev::ld_stream_v4(row1 + off); n1b = dev::ld_stream_v4(row1 + off + 16); }
        }
        const int k0 = kb * 128 + t * 32;
        uint32_t x[MB][16];
#pragma unroll
        for (int mb = 0; mb < MB; ++mb) load_act(a, K, 8 * mb + g, M, k0, x[mb]);
        // 32 codes per row: words 0..7, pair i covers codes 8i..8i+7 (words 2i, 2i+1)
        const uint32_t ra[8] = {c0a.x, c0a.y, c0a.z, c0a.w, c0b.x, c0b.y, c0b.z, c0b.w};
        const uint32_t rb[8] = {c1a.x, c1a.y, c1a.z, c1a.w, c1b.x, c1b.y, c1b.z, c1b.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t alo = ra[2 * i] ^ 0x80808080u, ahi = ra[2 * i + 1] ^ 0x80808080u;
            const uint32_t blo = rb[2 * i] ^ 0x80808080u, bhi = rb[2 * i + 1] ^ 0x80808080u;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const uint32_t a0 = dequant_pair_i8(alo, ahi, 2 * h, sf0);
                const uint32_t a1 = dequant_pair_i8(blo, bhi, 2 * h, sf1);
                const uint32_t a2 = dequant_pair_i8(alo, ahi, 2 * h + 1, sf0);
                const uint32_t a3 = dequant_pair_i8(blo, bhi, 2 * h + 1, sf1);
#pragma unroll
                for (int mb = 0; mb < MB; ++mb) {
                    uint32_t b0, b1;
                    act_operand(x[mb], i, h, b0, b1);
                    dev::mma_bf16_16816(acc[mb], a0, a1, a2, a3, b0, b1);
                }
            }
        }
    }
    gemv_epilogue<MB>(acc, M, N, n0, lane, split, splits, tile, y, partials, counters);
}

}  // namespace

// Split-K plan: enough warps for about 24 per SM, each with >= 2 K blocks.
GemvPlan gemv_plan(int64_t M, int64_t N, int64_t K) {
    GemvPlan p{};
    p.tiles = ceil_div(N, 16);
    const int64_t KB = K / 128;
    const int64_t target_warps = (int64_t)kSmCount * 24;
    int64_t s = ceil_div(target_warps, p.tiles);
    const int64_t max_s = KB >= 2 ? KB / 2 : 1;
    if (s > max_s) s = max_s;
    if (s < 1) s = 1;
    p.splits = (int)s;
    if (p.splits > 1) {
        p.partial_bytes = (size_t)p.splits * (size_t)M * (size_t)N * sizeof(float);
        p.partial_bytes = (p.partial_bytes + 255) & ~(size_t)255;
        p.counter_bytes = (size_t)ceil_div(p.tiles, 64) * 64 * sizeof(uint32_t);
    }
    p.total_bytes = p.partial_bytes + p.counter_bytes;
    return p;
}

static int group_shift_of(int64_t g) {
    if ((g & (g - 1)) != 0) return -1;
    int s = 0;
    while ((int64_t(1) << s) < g) ++s;
    return s;
}

qz_status launch_w4a16_gemv(const void *a, const void *codes, const void *scales,
                            const void *zeros, int64_t M, int64_t N, int64_t K,
                            int64_t group_size, void *y, void *workspace,
                            const GemvPlan &plan, cudaStream_t st) {
    float *partials = nullptr;
    uint32_t *counters = nullptr;
    if (plan.splits > 1) {
        partials = static_cast<float *>(workspace);
        counters = reinterpret_cast<uint32_t *>(static_cast<char *>(workspace) + plan.partial_bytes);
    }
    dim3 grid((unsigned)ceil_div(plan.tiles, kWarpsPerCta), (unsigned)plan.splits);
    const int shift = group_shift_of(group_size);
    auto *A = static_cast<const uint16_t *>(a);
    auto *C = static_cast<const uint8_t *>(codes);
    auto *S = static_cast<const uint16_t *>(scales);
    auto *Z = static_cast<const uint8_t *>(zeros);
    auto *Y = static_cast<uint16_t *>(y);
    if (M <= 8)
        w4a16_gemv_kernel<1><<<grid, kThreads, 0, st>>>(A, C, S, Z, (int)M, (int)N, (int)K,
                                                        (int)group_size, shift, Y, partials,
                                                        counters, plan.splits);
    else
        w4a16_gemv_kernel<2><<<grid, kThreads, 0, st>>>(A, C, S, Z, (int)M, (int)N, (int)K,
                                                        (int)group_size, shift, Y, partials,
                                                        counters, plan.splits);
    return launch_status();
}

qz_status launch_w8a16_gemv(const void *a, const void *codes, const void *scales,
                            int64_t M, int64_t N, int64_t K, void *y, void *workspace,
                            const GemvPlan &plan, cudaStream_t st) {
    float *partials = nullptr;
    uint32_t *counters = nullptr;
    if (plan.splits > 1) {
        partials = static_cast<float *>(workspace);
        counters = reinterpret_cast<uint32_t *>(static_cast<char *>(workspace) + plan.partial_bytes);
    }
    dim3 grid((unsigned)ceil_div(plan.tiles, kWarpsPerCta), (unsigned)plan.splits);
    auto *A = static_cast<const uint16_t *>(a);
    auto *C = static_cast<const uint8_t *>(codes);
    auto *S = static_cast<const uint16_t *>(scales);
    auto *Y = static_cast<uint16_t *>(y);
    if (M <= 8)
        w8a16_gemv_kernel<1><<<grid, kThreads, 0, st>>>(A, C, S, (int)M, (int)N, (int)K, Y,
                                                        partials, counters, plan.splits);
    else
        w8a16_gemv_kernel<2><<<grid, kThreads, 0, st>>>(A, C, S, (int)M, (int)N, (int)K, Y,
                                                        partials, counters, plan.splits);
    return launch_status();
}

}  // namespace qz
