// qz_gemv.cu -- weight-only decode GEMV: y (M x N) = a (M x K) * w_hat^T, M <= 16.
//
// Quantization concepts guide, "Quantize weights or activations": weight-only
// methods keep activations in bf16 and dequantize the weights to the compute
// dtype before each matmul; when decoding one token at a time the GPU spends
// the step reading weights, so 4-bit weights move a quarter of the bytes.
// GPTQ explainer: the gain needs kernels that dequantize inside the matmul.
//
// Design (one warp = 32 weight rows over a K range):
//   * Lane (g = lane/4, t = lane%4) streams, per 128-wide K block, its 32
//     consecutive k of rows g, g+8, g+16, g+24 (16 bytes of int4 codes or 32
//     bytes of int8 codes per row) with cp.async into a ring of kStages
//     blocks in the warp's own slice of shared memory, so that kStages-1
//     blocks are in flight while one is computed, without holding them in
//     registers.  The codes each lane copies are the ones it reads back.
//   * int4 with groups of 128 * 2^i: the scales and zeros of the
//     block ride in the same ring slot.  Lane (g, t) copies the aligned
//     32-bit words holding the scale and the zero of row g + 8t, so the 32
//     rows of the warp take two 4-byte copies per lane; after
//     cp.async.wait_group and a warp barrier every lane reads the words of
//     its four rows with two 16-byte shared loads and builds (S, S) and
//     bf16(-(128 + Z)) twice with one byte permute each.  Since the warp's
//     first row is a multiple of 32 and its rows differ by multiples of 8,
//     all four rows of a lane share the word offset of their entries.
//     Other group sizes load the lane's scales and zeros directly.
//   * Codes are dequantized in registers to bf16 exactly as qz_dequantize
//     forms them.  int4: a LOP3 builds bf16(128 + q) for two nibbles,
//     add.rn.bf16x2 of bf16(-(128 + Z)) leaves q - Z exactly, mul.rn.bf16x2
//     by the bf16 scale rounds S*(q - Z) once.  int8: the byte (XOR 0x80) is
//     placed in the mantissa of 2^23, one fp32 subtraction gives q exactly,
//     the pair is packed to bf16 exactly and mul.rn.bf16x2 rounds S*q once.
//   * A byte of codes yields the pairs (q_j, q_{j+4}), so the K axis is
//     permuted consistently for both MMA operands: the pairs are the A operand
//     (16 rows x 16 k) of mma.sync m16n8k16 with fp32 accumulation and the
//     activations (tokens as the 8 columns) are the B operand, permuted to
//     match with PRMT once per k for both 16-row tiles of the warp.  For
//     M > 8 a second MMA covers tokens 8..15.  Columns of tokens >= M read
//     token M-1's activations; their outputs are dropped.
//   * Stream-K: the (32-row task x 128-wide K block) units are divided into
//     equal contiguous ranges, one per launched warp, and exactly a whole
//     number of CTAs per SM is launched, so every SM gets the same work.  A
//     task covered by one warp is written directly; otherwise each
//     contributing warp writes its fp32 partial tile into the task's slot
//     and bumps the task's counter, and the last one to arrive adds the
//     slots in order (deterministic), one row per lane, writes bf16 y and
//     resets the counter.
#include <cuda_runtime.h>

#include "qz_internal.cuh"

namespace qz {
namespace {

constexpr int kWarpsPerCta = 4;
constexpr int kThreads = 32 * kWarpsPerCta;
constexpr int kRowsPerWarp = 32;                       // two 16-row MMA tiles

// bf16 pair (nibble j, nibble j+4) of a code word: bf16_rne(S * (q - Z)).
// nz2 holds bf16(-(128 + Z)) twice.
__device__ __forceinline__ uint32_t dequant_pair_u4(uint32_t word, int j, uint32_t s2,
                                                    uint32_t nz2) {
    const uint32_t x = dev::and_or<0x000F000Fu>(word >> (4 * j), 0x43004300u);   // bf16(128+q)
    return dev::bf16x2_mul(dev::bf16x2_add(x, nz2), s2);
}

// bf16 pair (code c_j, code c_{j+4}) of 8 consecutive int8 codes held in
// words lo (c0..c3) and hi (c4..c7), already XORed with 0x80808080:
// bits 0x4B000000 | byte is the fp32 2^23 + q + 128.  One subtraction leaves
// q exactly, the pair is packed to bf16 exactly (|q| <= 127), and
// mul.rn.bf16x2 by (S, S) rounds the exact product S*q once, as
// qz_dequantize does.
__device__ __forceinline__ uint32_t dequant_pair_i8(uint32_t lo, uint32_t hi, int j, uint32_t s2) {
    const uint32_t sel = (uint32_t)j | 0x7540u;
    const float f0 = __uint_as_float(dev::prmt(lo, 0x4B000000u, sel));
    const float f1 = __uint_as_float(dev::prmt(hi, 0x4B000000u, sel));
    const uint32_t q2 = dev::pack_bf16x2(__fsub_rn(f0, 8388736.0f), __fsub_rn(f1, 8388736.0f));
    return dev::bf16x2_mul(q2, s2);
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

template <int BITS>
struct RowWords {
    static constexpr int kWordsPerRow = BITS == 4 ? 4 : 8;
    uint32_t w[4][kWordsPerRow];   // rows g, g+8, g+16, g+24
};

struct RowParams {
    uint32_t s2[4], z2[4];         // int4, rows g + 8j: (S, S) and bf16(-(128 + Z)) twice
};

template <int MB>
struct Act {
    uint32_t x[MB][16];            // tokens g (+8): 32 bf16 each
};

template <int BITS>
constexpr int kStages = BITS == 4 ? 4 : 3;               // ring slots per warp
template <int BITS>
constexpr int kLaneRowBytes = BITS == 4 ? 16 : 32;     // codes of one row per lane per block
template <int BITS>
constexpr int kCodeBytes = 4 * 32 * kLaneRowBytes<BITS>;
constexpr int kSzBytes = 256;                          // 32 scale words + 32 zero words
template <int BITS>
constexpr int kSlotBytes = kCodeBytes<BITS> + (BITS == 4 ? kSzBytes : 0);
template <int BITS>
constexpr int kGemvSmemBytes = kWarpsPerCta * kStages<BITS> * kSlotBytes<BITS>;
// Resident CTAs per SM: registers allow five (int4, M <= 8: at most 102 per
// thread), four (int8, M <= 8: shared memory) or three (M > 8).
template <int BITS, int MB>
constexpr int kCtasPerSm = MB == 1 ? (BITS == 4 ? 5 : 4) : 3;

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async4(uint32_t dst, const void *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
    asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Byte offset, inside a warp's slot, of 16-byte piece `half` of row j for
// `lane`: pieces of 32 lanes are contiguous, so each 8-lane phase of a
// 16-byte shared load reads 128 consecutive bytes (no bank conflicts).
template <int BITS>
__device__ __forceinline__ uint32_t piece_offset(int j, int half, int lane) {
    return (uint32_t)(((j * (kLaneRowBytes<BITS> / 16) + half) * 32 + lane) * 16);
}

template <int BITS>
__device__ __forceinline__ void read_block(RowWords<BITS> &rw, const uint8_t *slot, int lane) {
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int h = 0; h < kLaneRowBytes<BITS> / 16; ++h) {
            const uint4 v = *reinterpret_cast<const uint4 *>(slot + piece_offset<BITS>(j, h, lane));
            rw.w[j][4 * h + 0] = v.x; rw.w[j][4 * h + 1] = v.y;
            rw.w[j][4 * h + 2] = v.z; rw.w[j][4 * h + 3] = v.w;
        }
}

struct GemvArgs {
    const uint16_t *a;
    const uint8_t *codes;
    const uint16_t *scales;
    const uint8_t *zeros;
    int M, N, K, group_size, group_shift;
    int bpg_shift;                     // log2(group_size / 128) (ring path), else -1
    uint16_t *y;
    float *partials;
    uint32_t *counters;
    int64_t units;        // tasks * kblocks
    int64_t warps;        // launched warps
    int kblocks, slots;
    int prefetch_early;   // launch overlap: first blocks' weights before the grid wait
};

// Group index of 128-wide block kb when the group size is 128 * 2^bpg_shift
// (the ring path's condition).
__device__ __forceinline__ int group_of_block(const GemvArgs &p, int kb) {
    return kb >> p.bpg_shift;
}

// Scales and zeros of the lane's four rows for block kb, loaded directly
// (group sizes below 128, or scale/zero arrays the ring cannot copy).
__device__ __forceinline__ void load_params_direct(RowParams &rp, const GemvArgs &p,
                                                   const bool (&valid)[4], const int (&rows)[4],
                                                   int kb, int t) {
    const int k0 = kb * 128 + t * 32;
    const int64_t gpr = p.K / p.group_size;
    const int gi = p.group_shift >= 0 ? (k0 >> p.group_shift) : (k0 / p.group_size);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint32_t s = valid[j] ? __ldg(&p.scales[(int64_t)rows[j] * gpr + gi]) : 0u;
        const uint32_t z = valid[j] ? __ldg(&p.zeros[(int64_t)rows[j] * gpr + gi]) : 0u;
        rp.s2[j] = s * 0x00010001u;                      // (S, S)
        rp.z2[j] = (0xC300u + z) * 0x00010001u;          // bf16(-(128 + Z)) twice
    }
}

// Activations of one block for tokens g (and g + 8), clamped to M - 1: read
// from L1/L2 (the vector is shared by every warp) right before the block is
// computed.
template <int MB>
__device__ __forceinline__ void load_act(Act<MB> &ac, const GemvArgs &p, int kb, int g, int t) {
    const int k0 = kb * 128 + t * 32;
#pragma unroll
    for (int mb = 0; mb < MB; ++mb) {
        const int tok = min(8 * mb + g, p.M - 1);
        const uint4 *src = reinterpret_cast<const uint4 *>(p.a + (int64_t)tok * p.K + k0);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint4 v = __ldg(src + q);
            ac.x[mb][4 * q + 0] = v.x; ac.x[mb][4 * q + 1] = v.y;
            ac.x[mb][4 * q + 2] = v.z; ac.x[mb][4 * q + 3] = v.w;
        }
    }
}

template <int BITS, int MB>
__device__ __forceinline__ void compute_block(const RowParams &rp, const Act<MB> &ac,
                                              const RowWords<BITS> &rw, const uint32_t (&s8)[4],
                                              float (&acc)[2][MB][4]) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        uint32_t lo8[4], hi8[4];
        if (BITS == 8) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                lo8[j] = rw.w[j][2 * i] ^ 0x80808080u;
                hi8[j] = rw.w[j][2 * i + 1] ^ 0x80808080u;
            }
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            uint32_t b0[MB], b1[MB];
#pragma unroll
            for (int mb = 0; mb < MB; ++mb) act_operand(ac.x[mb], i, h, b0[mb], b1[mb]);
#pragma unroll
            for (int rt = 0; rt < 2; ++rt) {
                const int ja = 2 * rt, jb = 2 * rt + 1;     // rows g(+16), g+8(+16)
                uint32_t a0, a1, a2, a3;
                if (BITS == 4) {
                    a0 = dequant_pair_u4(rw.w[ja][i], 2 * h, rp.s2[ja], rp.z2[ja]);
                    a1 = dequant_pair_u4(rw.w[jb][i], 2 * h, rp.s2[jb], rp.z2[jb]);
                    a2 = dequant_pair_u4(rw.w[ja][i], 2 * h + 1, rp.s2[ja], rp.z2[ja]);
                    a3 = dequant_pair_u4(rw.w[jb][i], 2 * h + 1, rp.s2[jb], rp.z2[jb]);
                } else {
                    a0 = dequant_pair_i8(lo8[ja], hi8[ja], 2 * h, s8[ja]);
                    a1 = dequant_pair_i8(lo8[jb], hi8[jb], 2 * h, s8[jb]);
                    a2 = dequant_pair_i8(lo8[ja], hi8[ja], 2 * h + 1, s8[ja]);
                    a3 = dequant_pair_i8(lo8[jb], hi8[jb], 2 * h + 1, s8[jb]);
                }
#pragma unroll
                for (int mb = 0; mb < MB; ++mb)
                    dev::mma_bf16_16816(acc[rt][mb], a0, a1, a2, a3, b0[mb], b1[mb]);
            }
        }
    }
}

// Programmatic dependent launch: let the next kernel on the stream be
// scheduled; wait until the previous one has completed and its writes are
// visible (a no-op when this grid was not launched as a dependent).
__device__ __forceinline__ void allow_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void wait_for_previous_grid() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

// First warp whose unit range contains unit u (ranges: [w*U/W, (w+1)*U/W)).
__device__ __forceinline__ int64_t warp_of_unit(int64_t u, int64_t U, int64_t W) {
    return ((u + 1) * W - 1) / U;
}

// Deterministic split-K sum: y[t][row] = sum over slots c = 0, 1, ... of
// base[c * slot_elems + t * ROWS + r], for the M <= MAXTOK tokens, added in
// slot order.  The loads of two slots for every token (eight slots when
// M = 1) are issued together.
template <int MAXTOK, int ROWS>
__device__ __forceinline__ void reduce_slots(const float *base, int64_t slot_elems,
                                             int contributors, int M, int r, int64_t row,
                                             int N, uint16_t *y) {
    if (M == 1) {                      // one token: eight slots' loads per round trip
        float sum = 0.0f;
        for (int c0 = 0; c0 < contributors; c0 += 8) {
            float v[8];
#pragma unroll
            for (int cc = 0; cc < 8; ++cc)
                v[cc] = c0 + cc < contributors ? __ldcg(base + (int64_t)(c0 + cc) * slot_elems + r)
                                               : 0.0f;
#pragma unroll
            for (int cc = 0; cc < 8; ++cc)
                if (c0 + cc < contributors) sum += v[cc];
        }
        if (row < N) y[row] = (uint16_t)dev::f32_to_bf16_rne(sum);
        return;
    }
    float sum[MAXTOK];
#pragma unroll
    for (int t = 0; t < MAXTOK; ++t) sum[t] = 0.0f;
    for (int c = 0; c < contributors; c += 2) {
        float x0[MAXTOK], x1[MAXTOK];
        const float *s0 = base + (int64_t)c * slot_elems + r;
        const bool two = c + 1 < contributors;
#pragma unroll
        for (int t = 0; t < MAXTOK; ++t) {
            x0[t] = t < M ? __ldcg(s0 + t * ROWS) : 0.0f;
            x1[t] = (t < M && two) ? __ldcg(s0 + slot_elems + t * ROWS) : 0.0f;
        }
#pragma unroll
        for (int t = 0; t < MAXTOK; ++t) {
            sum[t] += x0[t];
            if (two) sum[t] += x1[t];
        }
    }
    if (row < N) {
#pragma unroll
        for (int t = 0; t < MAXTOK; ++t)
            if (t < M) y[(int64_t)t * N + row] = (uint16_t)dev::f32_to_bf16_rne(sum[t]);
    }
}

// acc[rt][mb][j] holds y[tok = 8mb + 2t + (j&1)][row = n0 + 16rt + g + 8(j>>1)].
// `whole`: this warp covered every K block of the task.  Otherwise the
// partial goes to slot (this warp - the task's first warp) and the last of
// the task's contributors adds the slots in order, lane l summing row l.
template <int MB>
__device__ __forceinline__ void gemv_flush(float (&acc)[2][MB][4], const GemvArgs &p, int task,
                                           bool whole, int64_t w, int lane) {
    const int g = lane >> 2, t = lane & 3;
    const int n0 = task * kRowsPerWarp;
    if (whole) {
#pragma unroll
        for (int rt = 0; rt < 2; ++rt)
#pragma unroll
            for (int mb = 0; mb < MB; ++mb)
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int row = n0 + 16 * rt + g + 8 * (j >> 1);
                    const int tok = 8 * mb + 2 * t + (j & 1);
                    if (row < p.N && tok < p.M)
                        p.y[(int64_t)tok * p.N + row] = (uint16_t)dev::f32_to_bf16_rne(acc[rt][mb][j]);
                }
        return;
    }
    const int64_t first = warp_of_unit((int64_t)task * p.kblocks, p.units, p.warps);
    const int64_t last = warp_of_unit((int64_t)(task + 1) * p.kblocks - 1, p.units, p.warps);
    const int contributors = (int)(last - first + 1);
    const int64_t slot_elems = (int64_t)p.M * kRowsPerWarp;
    float *base = p.partials + ((int64_t)task * p.slots) * slot_elems;
    float *mine = base + (w - first) * slot_elems;
#pragma unroll
    for (int rt = 0; rt < 2; ++rt)
#pragma unroll
        for (int mb = 0; mb < MB; ++mb)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int rl = 16 * rt + g + 8 * (j >> 1);
                const int tok = 8 * mb + 2 * t + (j & 1);
                if (tok < p.M) __stcg(&mine[tok * kRowsPerWarp + rl], acc[rt][mb][j]);
            }
    __threadfence();
    __syncwarp();
    uint32_t prev = 0;
    if (lane == 0) prev = atomicAdd(&p.counters[task], 1u);
    prev = __shfl_sync(0xFFFFFFFFu, prev, 0);
    if (prev != (uint32_t)(contributors - 1)) return;
    __threadfence();
    // The last contributor: lane l adds row l of every slot in slot order,
    // for all tokens at once (two slots' loads in flight per round trip).
    reduce_slots<8 * MB, kRowsPerWarp>(base, slot_elems, contributors, p.M, lane, n0 + lane,
                                       p.N, p.y);
    if (lane == 0) p.counters[task] = 0u;
}

// RING_SZ: int4 scales and zeros travel through the cp.async ring (group
// size a multiple of 128, 4-byte aligned arrays whose 4-byte words stay
// inside them).
template <int BITS, int MB, bool RING_SZ>
__global__ void __launch_bounds__(kThreads, kCtasPerSm<BITS, MB>)
gemv_kernel(const GemvArgs p) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, t = lane & 3;
    const int64_t w = (int64_t)blockIdx.x * kWarpsPerCta + warp;
    if (w >= p.warps) return;                      // the last CTA of a short grid
    int64_t u = w * p.units / p.warps;
    const int64_t u_end = (w + 1) * p.units / p.warps;
    // With launch overlap, only the first ring fill of weights (which the
    // caller guarantees the previous kernel does not write) precedes the
    // wait for the previous grid; every other global access follows it.
    allow_dependents();
    bool waited = !p.prefetch_early;

    constexpr int S = kStages<BITS>;
    constexpr int kSlot = kSlotBytes<BITS>;
    extern __shared__ __align__(16) uint8_t gemv_smem[];
    uint8_t *ring = gemv_smem + warp * S * kSlot;
    const uint32_t ring_u32 = (uint32_t)__cvta_generic_to_shared(ring);
    const int64_t gpr = BITS == 4 ? p.K / p.group_size : 1;
    const uint32_t *scale_words = reinterpret_cast<const uint32_t *>(p.scales);
    const uint32_t *zero_words = reinterpret_cast<const uint32_t *>(p.zeros);
    // (row * gpr) mod 4 is the same for rows g, g+8, g+16, g+24 of any task
    const int word_phase = (int)(((int64_t)g * gpr) & 3);

    while (u < u_end) {
        const int task = (int)(u / p.kblocks);
        const int kb_begin = (int)(u - (int64_t)task * p.kblocks);
        const int64_t kb_lim = kb_begin + (u_end - u);
        const int kb_end = (int)(kb_lim < p.kblocks ? kb_lim : (int64_t)p.kblocks);
        const int nkb = kb_end - kb_begin;
        const int n0 = task * kRowsPerWarp;

        int rows[4];
        bool valid[4];
        const uint8_t *rowp[4];
        uint32_t s8[4];                              // int8: (S, S) of rows g + 8j
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            rows[j] = n0 + g + 8 * j;
            valid[j] = rows[j] < p.N;
            rowp[j] = p.codes + (int64_t)(valid[j] ? rows[j] : 0) * (BITS == 4 ? p.K / 2 : p.K) +
                      t * (BITS == 4 ? 16 : 32);
            s8[j] = (BITS == 8 && valid[j]) ? (uint32_t)__ldg(&p.scales[rows[j]]) * 0x00010001u : 0u;
        }
        // the row whose scale and zero words this lane copies
        const int row_c = n0 + g + 8 * t;
        const bool valid_c = RING_SZ && row_c < p.N;
        const int64_t entry_c = (int64_t)(valid_c ? row_c : 0) * gpr;
        const uint32_t sz_dst = kCodeBytes<BITS> + 4u * (uint32_t)(4 * g + t);

        auto issue = [&](int kb, uint32_t slot) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                if (!valid[j]) continue;
#pragma unroll
                for (int h = 0; h < kLaneRowBytes<BITS> / 16; ++h)
                    cp_async16(slot + piece_offset<BITS>(j, h, lane),
                               rowp[j] + kb * (BITS == 4 ? 64 : 128) + 16 * h);
            }
            if (RING_SZ && valid_c) {
                const int64_t e = entry_c + group_of_block(p, kb);
                cp_async4(slot + sz_dst, scale_words + (e >> 1));
                cp_async4(slot + sz_dst + 128u, zero_words + (e >> 2));
            }
        };

        float acc[2][MB][4];
#pragma unroll
        for (int rt = 0; rt < 2; ++rt)
#pragma unroll
            for (int mb = 0; mb < MB; ++mb)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[rt][mb][j] = 0.0f;

#pragma unroll
        for (int q = 0; q < S - 1; ++q) {
            if (q < nkb) issue(kb_begin + q, ring_u32 + q * kSlot);
            cp_async_commit();
        }
        if (!waited) {
            wait_for_previous_grid();
            waited = true;
        }
        int slot = 0;
#pragma unroll 2
        for (int ii = 0; ii < nkb; ++ii) {
            cp_async_wait<S - 2>();                  // block ii has landed in its slot
            if (RING_SZ) __syncwarp();               // ... every lane's copies of it, too
            const int refill = ii + S - 1;           // into the slot read one block ago
            const int rslot = slot == 0 ? S - 1 : slot - 1;
            if (refill < nkb) issue(kb_begin + refill, ring_u32 + rslot * kSlot);
            cp_async_commit();
            const int kb = kb_begin + ii;
            const uint8_t *cur = ring + slot * kSlot;
            Act<MB> ac;
            load_act(ac, p, kb, g, t);
            RowWords<BITS> rw;
            read_block<BITS>(rw, cur, lane);
            RowParams rp;
            if (BITS == 4) {
                if (RING_SZ) {
                    const uint4 ws = *reinterpret_cast<const uint4 *>(cur + kCodeBytes<BITS> + 16 * g);
                    const uint4 wz =
                        *reinterpret_cast<const uint4 *>(cur + kCodeBytes<BITS> + 128 + 16 * g);
                    const int phase = word_phase + group_of_block(p, kb);
                    const uint32_t os = (uint32_t)(phase & 1) * 2u, oz = (uint32_t)(phase & 3);
                    const uint32_t sel_s = os * 0x0101u + (os + 1u) * 0x1010u;   // (S, S)
                    const uint32_t sel_z = oz * 0x0101u + 0x4040u;               // (0xC3, Z) x 2
                    const uint32_t wsv[4] = {ws.x, ws.y, ws.z, ws.w};
                    const uint32_t wzv[4] = {wz.x, wz.y, wz.z, wz.w};
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        rp.s2[j] = dev::prmt(wsv[j], 0u, sel_s);
                        rp.z2[j] = dev::prmt(wzv[j], 0xC3C3C3C3u, sel_z);
                    }
                } else {
                    load_params_direct(rp, p, valid, rows, kb, t);
                }
            }
            compute_block<BITS, MB>(rp, ac, rw, s8, acc);
            slot = slot == S - 1 ? 0 : slot + 1;
        }
        cp_async_wait<0>();
        __syncwarp();                                // the ring is reused by the next task
        gemv_flush<MB>(acc, p, task, nkb == p.kblocks, w, lane);
        u += nkb;
    }
}

int log2_exact(int64_t v) {
    if (v <= 0 || (v & (v - 1)) != 0) return -1;
    int s = 0;
    while ((int64_t(1) << s) < v) ++s;
    return s;
}

template <int BITS, int MB, bool RING_SZ>
qz_status launch_variant(const GemvArgs &args, dim3 grid, int overlap, cudaStream_t st) {
    constexpr int smem = kGemvSmemBytes<BITS>;
    static DeviceOnce attr_once;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return QZ_ERR_CUDA;
    }
    if (attr_once.run(dev, [] {
            return cudaFuncSetAttribute(gemv_kernel<BITS, MB, RING_SZ>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        }) != cudaSuccess)
        return QZ_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = overlap > 0 ? 1 : 0;
    cudaLaunchKernelEx(&cfg, gemv_kernel<BITS, MB, RING_SZ>, args);
    return launch_status();
}

template <int BITS>
qz_status launch_gemv(const void *a, const void *codes, const void *scales, const void *zeros,
                      int64_t M, int64_t N, int64_t K, int64_t group_size, void *y,
                      void *workspace, const GemvPlan &plan, int overlap, cudaStream_t st) {
    GemvArgs args;
    args.a = static_cast<const uint16_t *>(a);
    args.codes = static_cast<const uint8_t *>(codes);
    args.scales = static_cast<const uint16_t *>(scales);
    args.zeros = static_cast<const uint8_t *>(zeros);
    args.M = (int)M; args.N = (int)N; args.K = (int)K;
    args.group_size = (int)group_size;
    args.group_shift = log2_exact(group_size);
    args.bpg_shift = group_size % 128 == 0 ? log2_exact(group_size / 128) : -1;
    args.y = static_cast<uint16_t *>(y);
    args.partials = nullptr;
    args.counters = nullptr;
    if (plan.total_bytes > 0) {
        args.partials = static_cast<float *>(workspace);
        args.counters =
            reinterpret_cast<uint32_t *>(static_cast<char *>(workspace) + plan.partial_bytes);
    }
    args.units = plan.tasks * plan.kblocks;
    args.warps = plan.warps;
    args.kblocks = (int)plan.kblocks;
    args.slots = (int)plan.slots;
    args.prefetch_early = overlap;
    const dim3 grid((unsigned)ceil_div(plan.warps, (int64_t)kWarpsPerCta));

    // The ring copies the aligned 4-byte words holding each scale and zero;
    // they stay inside the arrays when N * K / g is a multiple of 4.
    if constexpr (BITS == 4) {
        const int64_t entries = N * (K / group_size);
        const bool ring_sz = args.bpg_shift >= 0 && aligned(scales, 4) && aligned(zeros, 4) &&
                             entries % 4 == 0;
        if (M <= 8)
            return ring_sz ? launch_variant<4, 1, true>(args, grid, overlap, st)
                           : launch_variant<4, 1, false>(args, grid, overlap, st);
        return ring_sz ? launch_variant<4, 2, true>(args, grid, overlap, st)
                       : launch_variant<4, 2, false>(args, grid, overlap, st);
    } else {
        return M <= 8 ? launch_variant<8, 1, false>(args, grid, overlap, st)
                      : launch_variant<8, 2, false>(args, grid, overlap, st);
    }
}

}  // namespace

// Stream-K plan.  Up to kCtasPerSm 4-warp CTAs are resident on an SM (the
// ring of a CTA takes 36 KB (int4) or 48 KB (int8) of shared memory), and
// the same number k runs on every SM.
//   M = 1: a warp streams its ceil(U / W) K blocks one after another, and a
//   block takes longer the more warps share an SM sub-partition: about
//   (0.40 + 0.33 k) us with k CTAs per SM, fitted to the decode layers.  k
//   minimises ceil(U / W) * (40 + 33 k); ties go to the smaller k.
//   M > 1: the split-K partials grow with M, so k is the largest that gives
//   each warp at least kGemvMinBlocksPerWarp blocks (fewer contributors).
constexpr int kBlockCostBase = 40, kBlockCostPerCta = 33;
constexpr int kGemvMinBlocksPerWarp = 4;

GemvPlan gemv_plan(int64_t M, int64_t N, int64_t K, int bits, int sms) {
    GemvPlan p{};
    p.tasks = ceil_div(N, kRowsPerWarp);
    p.kblocks = K / 128;
    const int64_t units = p.tasks * p.kblocks;
    const int64_t max_per_sm = M <= 8 ? (bits == 4 ? kCtasPerSm<4, 1> : kCtasPerSm<8, 1>)
                                      : kCtasPerSm<4, 2>;
    int64_t per_sm = 1;
    if (M == 1) {
        int64_t best_cost = -1;
        for (int64_t k = 1; k <= max_per_sm; ++k) {
            const int64_t cost = ceil_div(units, (int64_t)sms * kWarpsPerCta * k) *
                                 (kBlockCostBase + kBlockCostPerCta * k);
            if (best_cost < 0 || cost < best_cost) {
                best_cost = cost;
                per_sm = k;
            }
        }
    } else {
        per_sm = units / ((int64_t)sms * kWarpsPerCta * kGemvMinBlocksPerWarp);
        if (per_sm > max_per_sm) per_sm = max_per_sm;
        if (per_sm < 1) per_sm = 1;
    }
    p.warps = (int64_t)sms * per_sm * kWarpsPerCta;
    // Fewer units than warps: one unit per warp.  Every warp must own at
    // least one unit, or a split task would count a contributor that never
    // arrives.
    if (p.warps > units) p.warps = units;
    // contributors of one task: at most ceil(KB / floor(U/W)) + 1
    const int64_t per_warp = units / p.warps;
    p.slots = per_warp >= 1 ? ceil_div(p.kblocks, per_warp) + 1 : p.kblocks + 1;
    if (p.slots > p.kblocks) p.slots = p.kblocks;
    p.partial_bytes = (size_t)p.tasks * p.slots * (size_t)M * kRowsPerWarp * sizeof(float);
    p.partial_bytes = (p.partial_bytes + 255) & ~(size_t)255;
    p.counter_bytes = (size_t)ceil_div(p.tasks, 64) * 64 * sizeof(uint32_t);
    p.total_bytes = p.partial_bytes + p.counter_bytes;
    return p;
}

// The plan's workspace is not monotone in the SM count (fewer SMs can pick
// more CTAs per SM), so the size callers allocate is the largest over every
// count up to kSmCount.
size_t gemv_workspace_bound(int64_t M, int64_t N, int64_t K, int bits) {
    size_t most = 0;
    for (int sms = 1; sms <= kSmCount; ++sms) {
        const size_t b = gemv_plan(M, N, K, bits, sms).total_bytes;
        if (b > most) most = b;
    }
    return most;
}

qz_status launch_w4a16_gemv(const void *a, const void *codes, const void *scales,
                            const void *zeros, int64_t M, int64_t N, int64_t K,
                            int64_t group_size, void *y, void *workspace,
                            const GemvPlan &plan, int overlap, cudaStream_t st) {
    return launch_gemv<4>(a, codes, scales, zeros, M, N, K, group_size, y, workspace, plan,
                          overlap, st);
}

qz_status launch_w8a16_gemv(const void *a, const void *codes, const void *scales,
                            int64_t M, int64_t N, int64_t K, void *y, void *workspace,
                            const GemvPlan &plan, int overlap, cudaStream_t st) {
    return launch_gemv<8>(a, codes, scales, nullptr, M, N, K, K, y, workspace, plan, overlap,
                          st);
}

}  // namespace qz
