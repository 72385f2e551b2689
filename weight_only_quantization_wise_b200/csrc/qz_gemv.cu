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
//     bytes of int8 codes per row) with cp.async into a ring of STAGES blocks
//     in the warp's own slice of shared memory, so that STAGES-1 blocks are in
//     flight while one is computed without holding them in registers.  Each
//     lane reads back only what it copied, so the ring needs no barrier:
//     cp.async.wait_group orders it.  Scales and zeros are prefetched one
//     block ahead in registers; the activation vector, which every warp
//     reads, is loaded from L1 when its block is computed.
//   * Codes are dequantized in registers to bf16 exactly as qz_dequantize
//     forms them.  int4: a LOP3 builds bf16(128 + q) for two nibbles,
//     sub.rn.bf16x2 removes (128 + Z) exactly, mul.rn.bf16x2 by the bf16 scale
//     rounds S*(q - Z) once.  int8: the byte (XOR 0x80) is placed in the
//     mantissa of 2^23, one packed fp32 subtraction gives q exactly, a packed
//     fp32 multiply gives the exact S*q, cvt.rn.bf16x2 rounds it once.
//     The subtraction adds a precomputed -(128 + Z) so that no per-pair
//     negation is needed.
//   * A byte of codes yields the pairs (q_j, q_{j+4}), so the K axis is
//     permuted consistently for both MMA operands: the pairs are the A operand
//     (16 rows x 16 k) of mma.sync m16n8k16 with fp32 accumulation and the
//     activations (tokens as the 8 columns) are the B operand, permuted to
//     match with PRMT once per k for both 16-row tiles of the warp.  For
//     M > 8 a second MMA covers tokens 8..15.
//   * Stream-K: the (32-row task x 128-wide K block) units are divided into
//     equal contiguous ranges, one per launched warp, and exactly a whole
//     number of CTAs per SM is launched, so every SM gets the same work.  A
//     task covered by one warp is written directly; otherwise each
//     contributing warp writes its fp32 partial tile into the task's slot
//     and bumps the task's counter, and the last one to arrive adds the
//     slots in order (deterministic), writes bf16 y and resets the counter.
#include <cuda_runtime.h>

#include "qz_internal.cuh"

namespace qz {
namespace {

constexpr int kWarpsPerCta = 4;
constexpr int kThreads = 32 * kWarpsPerCta;
constexpr int kRowsPerWarp = 32;                       // two 16-row MMA tiles
constexpr int kRowsPerCta = kRowsPerWarp * kWarpsPerCta;

// bf16 pair (nibble j, nibble j+4) of a code word: bf16_rne(S * (q - Z)).
// nz2 holds bf16(-(128 + Z)) twice.
__device__ __forceinline__ uint32_t dequant_pair_u4(uint32_t word, int j, uint32_t s2,
                                                    uint32_t nz2) {
    const uint32_t x = ((word >> (4 * j)) & 0x000F000Fu) | 0x43004300u;   // bf16(128+q)
    return dev::bf16x2_mul(dev::bf16x2_add(x, nz2), s2);
}

// bf16 pair (code c_j, code c_{j+4}) of 8 consecutive int8 codes held in
// words lo (c0..c3) and hi (c4..c7), already XORed with 0x80808080:
// bits 0x4B000000 | byte is the fp32 2^23 + q + 128.
__device__ __forceinline__ uint32_t dequant_pair_i8(uint32_t lo, uint32_t hi, int j, float s) {
    const uint32_t sel = (uint32_t)j | 0x7540u;
    const float f0 = __uint_as_float(dev::prmt(lo, 0x4B000000u, sel));
    const float f1 = __uint_as_float(dev::prmt(hi, 0x4B000000u, sel));
    const float p0 = __fmul_rn(__fsub_rn(f0, 8388736.0f), s);     // - (2^23 + 128): exact
    const float p1 = __fmul_rn(__fsub_rn(f1, 8388736.0f), s);     // then the exact product
    return dev::pack_bf16x2(p0, p1);
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

template <int BITS, int MB>
struct Stage {
    uint32_t s[4], z[4];           // int4: per-row scale bits and zero of this block
};

template <int MB>
struct Act {
    uint32_t x[MB][16];            // tokens g (+8): 32 bf16 each
};

template <int BITS>
constexpr int kGemvStages = BITS == 4 ? 8 : 4;           // a power of two
template <int BITS>
constexpr int kLaneRowBytes = BITS == 4 ? 16 : 32;     // codes of one row per lane per block
template <int BITS>
constexpr int kWarpStageBytes = 4 * 32 * kLaneRowBytes<BITS>;
template <int BITS>
constexpr int kGemvSmemBytes = kWarpsPerCta * kGemvStages<BITS> * kWarpStageBytes<BITS>;

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
    asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Byte offset, inside a warp's stage, of 16-byte piece `half` of row j for
// `lane`: pieces of 32 lanes are contiguous, so each 8-lane phase of a
// 16-byte shared load reads 128 consecutive bytes (no bank conflicts).
template <int BITS>
__device__ __forceinline__ uint32_t piece_offset(int j, int half, int lane) {
    return (uint32_t)(((j * (kLaneRowBytes<BITS> / 16) + half) * 32 + lane) * 16);
}

template <int BITS>
__device__ __forceinline__ void issue_block(uint32_t stage_base, const uint8_t *const (&rowp)[4],
                                            const bool (&valid)[4], int kb, int lane) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        if (!valid[j]) continue;
#pragma unroll
        for (int h = 0; h < kLaneRowBytes<BITS> / 16; ++h)
            cp_async16(stage_base + piece_offset<BITS>(j, h, lane),
                       rowp[j] + kb * (BITS == 4 ? 64 : 128) + 16 * h);
    }
}

template <int BITS>
__device__ __forceinline__ void read_block(RowWords<BITS> &rw, const uint8_t *stage, int lane) {
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int h = 0; h < kLaneRowBytes<BITS> / 16; ++h) {
            const uint4 v = *reinterpret_cast<const uint4 *>(stage + piece_offset<BITS>(j, h, lane));
            rw.w[j][4 * h + 0] = v.x; rw.w[j][4 * h + 1] = v.y;
            rw.w[j][4 * h + 2] = v.z; rw.w[j][4 * h + 3] = v.w;
        }
}

template <int BITS, int MB>
struct GemvArgs {
    const uint16_t *a;
    const uint8_t *codes;
    const uint16_t *scales;
    const uint8_t *zeros;
    int M, N, K, group_size, group_shift;
    uint16_t *y;
    float *partials;
    uint32_t *counters;
    int64_t units;        // tasks * kblocks
    int64_t warps;        // launched warps
    int kblocks, slots;
};

template <int BITS, int MB>
__device__ __forceinline__ void load_stage(Stage<BITS, MB> &st, const GemvArgs<BITS, MB> &p,
                                           const bool (&valid)[4], const int (&rows)[4], int kb,
                                           int g, int t) {
    const int k0 = kb * 128 + t * 32;
    if (BITS == 4) {
        const int gpr = p.K / p.group_size;
        const int gi = p.group_shift >= 0 ? (k0 >> p.group_shift) : (k0 / p.group_size);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            st.s[j] = valid[j] ? __ldg(&p.scales[(int64_t)rows[j] * gpr + gi]) : 0u;
            st.z[j] = valid[j] ? __ldg(&p.zeros[(int64_t)rows[j] * gpr + gi]) : 0u;
        }
    }
}

// Activations of one block for tokens g (and g + 8): read from L1/L2 (the
// vector is shared by every warp) right before the block is computed.
template <int BITS, int MB>
__device__ __forceinline__ void load_act(Act<MB> &ac, const GemvArgs<BITS, MB> &p, int kb, int g,
                                         int t) {
    const int k0 = kb * 128 + t * 32;
#pragma unroll
    for (int mb = 0; mb < MB; ++mb) {
        const int tok = 8 * mb + g;
        if (tok < p.M) {
            const uint4 *src = reinterpret_cast<const uint4 *>(p.a + (int64_t)tok * p.K + k0);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const uint4 v = __ldg(src + q);
                ac.x[mb][4 * q + 0] = v.x; ac.x[mb][4 * q + 1] = v.y;
                ac.x[mb][4 * q + 2] = v.z; ac.x[mb][4 * q + 3] = v.w;
            }
        } else {
#pragma unroll
            for (int q = 0; q < 16; ++q) ac.x[mb][q] = 0u;
        }
    }
}

template <int BITS, int MB>
__device__ __forceinline__ void compute_stage(const Stage<BITS, MB> &st, const Act<MB> &ac,
                                              const RowWords<BITS> &rw, const float (&sf)[4],
                                              float (&acc)[2][MB][4]) {
    uint32_t s2[4], z2[4];
    if (BITS == 4) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            s2[j] = st.s[j] * 0x00010001u;                  // (S, S)
            z2[j] = (0xC300u + st.z[j]) * 0x00010001u;      // bf16(-(128 + Z)) twice
        }
    }
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
                    a0 = dequant_pair_u4(rw.w[ja][i], 2 * h, s2[ja], z2[ja]);
                    a1 = dequant_pair_u4(rw.w[jb][i], 2 * h, s2[jb], z2[jb]);
                    a2 = dequant_pair_u4(rw.w[ja][i], 2 * h + 1, s2[ja], z2[ja]);
                    a3 = dequant_pair_u4(rw.w[jb][i], 2 * h + 1, s2[jb], z2[jb]);
                } else {
                    a0 = dequant_pair_i8(lo8[ja], hi8[ja], 2 * h, sf[ja]);
                    a1 = dequant_pair_i8(lo8[jb], hi8[jb], 2 * h, sf[jb]);
                    a2 = dequant_pair_i8(lo8[ja], hi8[ja], 2 * h + 1, sf[ja]);
                    a3 = dequant_pair_i8(lo8[jb], hi8[jb], 2 * h + 1, sf[jb]);
                }
#pragma unroll
                for (int mb = 0; mb < MB; ++mb)
                    dev::mma_bf16_16816(acc[rt][mb], a0, a1, a2, a3, b0[mb], b1[mb]);
            }
        }
    }
}

// First warp whose unit range contains unit u (ranges: [w*U/W, (w+1)*U/W)).
__device__ __forceinline__ int64_t warp_of_unit(int64_t u, int64_t U, int64_t W) {
    return ((u + 1) * W - 1) / U;
}

// acc[rt][mb][j] holds y[tok = 8mb + 2t + (j&1)][row = n0 + 16rt + g + 8(j>>1)].
// `whole`: this warp covered every K block of the task.  Otherwise the
// partial goes to slot (this warp - the task's first warp) and the last of
// the task's contributors adds the slots in order.
template <int BITS, int MB>
__device__ __forceinline__ void gemv_flush(float (&acc)[2][MB][4], const GemvArgs<BITS, MB> &p,
                                           int task, bool whole, int64_t w, int lane) {
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
    // Add the slots in order; four contributors' values are loaded at a time
    // so that the L2 round trips overlap.
    float sum[2][MB][4];
#pragma unroll
    for (int rt = 0; rt < 2; ++rt)
#pragma unroll
        for (int mb = 0; mb < MB; ++mb)
#pragma unroll
            for (int j = 0; j < 4; ++j) sum[rt][mb][j] = 0.0f;
    for (int c0 = 0; c0 < contributors; c0 += 4) {
        float v[4][2][MB][4];
#pragma unroll
        for (int cc = 0; cc < 4; ++cc)
#pragma unroll
            for (int rt = 0; rt < 2; ++rt)
#pragma unroll
                for (int mb = 0; mb < MB; ++mb)
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int rl = 16 * rt + g + 8 * (j >> 1);
                        const int tok = 8 * mb + 2 * t + (j & 1);
                        v[cc][rt][mb][j] = (c0 + cc < contributors && tok < p.M)
                            ? __ldcg(&base[(c0 + cc) * slot_elems + tok * kRowsPerWarp + rl])
                            : 0.0f;
                    }
#pragma unroll
        for (int cc = 0; cc < 4; ++cc)
#pragma unroll
            for (int rt = 0; rt < 2; ++rt)
#pragma unroll
                for (int mb = 0; mb < MB; ++mb)
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        if (c0 + cc < contributors) sum[rt][mb][j] += v[cc][rt][mb][j];
    }
#pragma unroll
    for (int rt = 0; rt < 2; ++rt)
#pragma unroll
        for (int mb = 0; mb < MB; ++mb)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int row = n0 + 16 * rt + g + 8 * (j >> 1);
                const int tok = 8 * mb + 2 * t + (j & 1);
                if (row < p.N && tok < p.M)
                    p.y[(int64_t)tok * p.N + row] = (uint16_t)dev::f32_to_bf16_rne(sum[rt][mb][j]);
            }
    if (lane == 0) p.counters[task] = 0u;
}

template <int BITS, int MB>
__global__ void __launch_bounds__(kThreads)
gemv_kernel(const GemvArgs<BITS, MB> p) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, t = lane & 3;
    const int64_t w = (int64_t)blockIdx.x * kWarpsPerCta + warp;
    int64_t u = w * p.units / p.warps;
    const int64_t u_end = (w + 1) * p.units / p.warps;

    constexpr int S = kGemvStages<BITS>;
    extern __shared__ __align__(16) uint8_t gemv_smem[];
    uint8_t *ring = gemv_smem + warp * S * kWarpStageBytes<BITS>;
    const uint32_t ring_u32 = (uint32_t)__cvta_generic_to_shared(ring);

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
        float sf[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            rows[j] = n0 + g + 8 * j;
            valid[j] = rows[j] < p.N;
            rowp[j] = p.codes + (int64_t)(valid[j] ? rows[j] : 0) * (BITS == 4 ? p.K / 2 : p.K) +
                      t * (BITS == 4 ? 16 : 32);
            sf[j] = 0.0f;
            if (BITS == 8 && valid[j])
                sf[j] = __uint_as_float((uint32_t)__ldg(&p.scales[rows[j]]) << 16);
        }
        float acc[2][MB][4];
#pragma unroll
        for (int rt = 0; rt < 2; ++rt)
#pragma unroll
            for (int mb = 0; mb < MB; ++mb)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[rt][mb][j] = 0.0f;

#pragma unroll
        for (int q = 0; q < S - 1; ++q) {
            if (q < nkb) issue_block<BITS>(ring_u32 + q * kWarpStageBytes<BITS>, rowp, valid,
                                           kb_begin + q, lane);
            cp_async_commit();
        }
        Stage<BITS, MB> sa, sb;
        load_stage(sa, p, valid, rows, kb_begin, g, t);
        for (int i = 0; i < nkb; i += 2) {
#pragma unroll
            for (int v = 0; v < 2; ++v) {
                const int ii = i + v;
                if (ii >= nkb) break;
                Stage<BITS, MB> &cur = v == 0 ? sa : sb;
                Stage<BITS, MB> &nxt = v == 0 ? sb : sa;
                cp_async_wait<S - 2>();               // block ii has landed in its slot
                const int refill = ii + S - 1;       // into the slot read one block ago
                if (refill < nkb)
                    issue_block<BITS>(ring_u32 + (refill & (S - 1)) * kWarpStageBytes<BITS>, rowp,
                                      valid, kb_begin + refill, lane);
                cp_async_commit();
                Act<MB> ac;
                load_act(ac, p, kb_begin + ii, g, t);
                RowWords<BITS> rw;
                read_block<BITS>(rw, ring + (ii & (S - 1)) * kWarpStageBytes<BITS>, lane);
                if (ii + 1 < nkb) load_stage(nxt, p, valid, rows, kb_begin + ii + 1, g, t);
                compute_stage(cur, ac, rw, sf, acc);
            }
        }
        cp_async_wait<0>();
        __syncwarp();                                // the ring is reused by the next task
        gemv_flush<BITS, MB>(acc, p, task, nkb == p.kblocks, w, lane);
        u += nkb;
    }
}

int group_shift_of(int64_t g) {
    if (g <= 0 || (g & (g - 1)) != 0) return -1;
    int s = 0;
    while ((int64_t(1) << s) < g) ++s;
    return s;
}

template <int BITS, int MB>
void set_smem_once() {
    static bool done[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !done[dev]) {
        cudaFuncSetAttribute(gemv_kernel<BITS, MB>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kGemvSmemBytes<BITS>);
        done[dev] = true;
    }
}

template <int BITS>
qz_status launch_gemv(const void *a, const void *codes, const void *scales, const void *zeros,
                      int64_t M, int64_t N, int64_t K, int64_t group_size, void *y,
                      void *workspace, const GemvPlan &plan, cudaStream_t st) {
    float *partials = nullptr;
    uint32_t *counters = nullptr;
    if (plan.total_bytes > 0) {
        partials = static_cast<float *>(workspace);
        counters = reinterpret_cast<uint32_t *>(static_cast<char *>(workspace) + plan.partial_bytes);
    }
    const dim3 grid((unsigned)(plan.warps / kWarpsPerCta));
    auto fill = [&](auto &args) {
        args.a = static_cast<const uint16_t *>(a);
        args.codes = static_cast<const uint8_t *>(codes);
        args.scales = static_cast<const uint16_t *>(scales);
        args.zeros = static_cast<const uint8_t *>(zeros);
        args.M = (int)M; args.N = (int)N; args.K = (int)K;
        args.group_size = (int)group_size;
        args.group_shift = group_shift_of(group_size);
        args.y = static_cast<uint16_t *>(y);
        args.partials = partials;
        args.counters = counters;
        args.units = plan.tasks * plan.kblocks;
        args.warps = plan.warps;
        args.kblocks = (int)plan.kblocks;
        args.slots = (int)plan.slots;
    };
    constexpr int smem = kGemvSmemBytes<BITS>;
    if (M <= 8) {
        GemvArgs<BITS, 1> args;
        fill(args);
        set_smem_once<BITS, 1>();
        gemv_kernel<BITS, 1><<<grid, kThreads, smem, st>>>(args);
    } else {
        GemvArgs<BITS, 2> args;
        fill(args);
        set_smem_once<BITS, 2>();
        gemv_kernel<BITS, 2><<<grid, kThreads, smem, st>>>(args);
    }
    return launch_status();
}

}  // namespace

// Stream-K plan.  Three 4-warp CTAs fit on an SM (64 KB of cp.async ring
// each), so 1, 2 or 3 CTAs per SM are launched -- always the same number on
// every SM -- with at least about four K blocks per warp.
constexpr int kGemvCtasPerSm = 3;

GemvPlan gemv_plan(int64_t M, int64_t N, int64_t K) {
    GemvPlan p{};
    p.tasks = ceil_div(N, kRowsPerWarp);
    p.kblocks = K / 128;
    const int64_t units = p.tasks * p.kblocks;
    int64_t per_sm = units / ((int64_t)kSmCount * kWarpsPerCta * 4);
    if (per_sm > kGemvCtasPerSm) per_sm = kGemvCtasPerSm;
    if (per_sm < 1) per_sm = 1;
    p.warps = (int64_t)kSmCount * per_sm * kWarpsPerCta;
    if (p.warps > units) p.warps = ceil_div(units, kWarpsPerCta) * kWarpsPerCta;
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

qz_status launch_w4a16_gemv(const void *a, const void *codes, const void *scales,
                            const void *zeros, int64_t M, int64_t N, int64_t K,
                            int64_t group_size, void *y, void *workspace,
                            const GemvPlan &plan, cudaStream_t st) {
    return launch_gemv<4>(a, codes, scales, zeros, M, N, K, group_size, y, workspace, plan, st);
}

qz_status launch_w8a16_gemv(const void *a, const void *codes, const void *scales,
                            int64_t M, int64_t N, int64_t K, void *y, void *workspace,
                            const GemvPlan &plan, cudaStream_t st) {
    return launch_gemv<8>(a, codes, scales, nullptr, M, N, K, K, y, workspace, plan, st);
}

}  // namespace qz
