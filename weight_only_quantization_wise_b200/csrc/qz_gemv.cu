// qz_gemv.cu -- weight-only decode GEMV: y (M x N) = a (M x K) * w_hat^T, M <= 16.
//
// Quantization concepts guide, "Quantize weights or activations": weight-only
// methods keep activations in bf16 and dequantize the weights to the compute
// dtype before each matmul; when decoding one token at a time the GPU spends
// the step reading weights, so 4-bit weights move a quarter of the bytes.
// GPTQ explainer: the gain needs kernels that dequantize inside the matmul.
//
// Design: each CTA is one producer warp and four consumer warps around a
// ring of shared-memory stages; a stage is one unit of work, 128 weight rows
// x 128 k (8 KB of int4 codes, 16 KB of int8).
//   * Producer (warp 0).  One lane issues a TMA 2D copy of the unit's codes
//     into the stage (completing on the stage's "full" mbarrier with a
//     transaction count).  For int4 with groups of 128 * 2^i the 32 lanes
//     also gather, with 4-byte cp.async copies, the aligned words that hold
//     the scale and the zero of each of the 128 rows and signal the same
//     barrier when they land (cp.async.mbarrier.arrive.noinc), so codes,
//     scales and zeros of a unit arrive together.  The producer waits on a
//     stage's "empty" barrier before refilling it; it never touches
//     activations, outputs or the workspace.
//   * Consumers (warps 1..4).  Warp w owns rows 32w..32w+31 of each unit.
//     Lane (g = lane/4, t = lane%4) reads the 16 (int4) or 32 (int8) code
//     bytes of k = 32t..32t+31 of rows g, g+8, g+16, g+24 from the stage with
//     16-byte shared loads (int8 rows are 128 B, loaded with the 128-byte
//     swizzle so that those loads are free of bank conflicts), reads the
//     four rows' scale and zero words with one 16-byte load each, releases
//     the stage, and dequantizes in registers to bf16 exactly as
//     qz_dequantize forms each weight.  int4: a LOP3 builds bf16(128 + q) for
//     two nibbles, add.rn.bf16x2 of bf16(-(128 + Z)) leaves q - Z exactly,
//     mul.rn.bf16x2 by the bf16 scale rounds S*(q - Z) once.  int8: the byte
//     (XOR 0x80) is placed in the mantissa of 2^23, one fp32 subtraction
//     gives q exactly, the pair is packed to bf16 exactly and mul.rn.bf16x2
//     rounds S*q once.
//   * A byte of codes yields the pairs (q_j, q_{j+4}), so the K axis is
//     permuted consistently for both MMA operands: the pairs are the A
//     operand (16 rows x 16 k) of mma.sync m16n8k16 with fp32 accumulation
//     and the activations (tokens as the 8 columns, read through L1) are the
//     B operand, permuted to match with PRMT once per k for both 16-row tiles
//     of the warp.  For M > 8 a second MMA covers tokens 8..15.  Columns of
//     tokens >= M read token M-1's activations; their outputs are dropped.
//   * Stream-K: the units, in (row task, k block) order, are divided into
//     equal contiguous ranges, one per CTA, with the same number of CTAs on
//     every SM, so every SM streams the same number of bytes.  A 32-row
//     subtask covered by one CTA is written directly; otherwise each
//     contributing CTA's warp writes its fp32 partial tile into the
//     subtask's slot and bumps the subtask's counter, and the last one to
//     arrive adds the slots in order (deterministic), one row per lane,
//     writes bf16 y and resets the counter.
//   * Every mbarrier wait is bounded (wall time, qz_set_device_wait_limit):
//     on expiry the waiting warp records the fault in the device error word
//     and a CTA-local abort flag, the producer stops issuing, waits (again
//     bounded) for every copy it issued to land, and the CTA exits.
#include <cuda.h>
#include <cuda_runtime.h>

#include "qz_sm100.cuh"

namespace qz {
namespace {

using namespace sm100;

constexpr int kConsumerWarps = 4;
constexpr int kRowsPerWarp = 32;                               // two 16-row MMA tiles
constexpr int kTileRows = kConsumerWarps * kRowsPerWarp;       // rows of a unit
constexpr int kThreads = 32 * (1 + kConsumerWarps);
constexpr int kBlockK = 128;                                   // k of a unit
template <int BITS>
constexpr int kRowBytes = kBlockK * BITS / 8;                  // code bytes of a row in a unit
template <int BITS>
constexpr int kCodeStage = kTileRows * kRowBytes<BITS>;        // 8 KB (int4), 16 KB (int8)
constexpr int kSzStage = kTileRows * 8;                        // 128 scale words + 128 zero words
template <int BITS>
constexpr int kStages = BITS == 4 ? 8 : 4;
constexpr int kMaxCtasPerSm = 3;

// Shared-memory layout (offsets from the 1024-byte aligned base).
template <int BITS>
struct Layout {
    static constexpr int S = kStages<BITS>;
    static constexpr uint32_t codes = 0;
    static constexpr uint32_t sz = codes + S * kCodeStage<BITS>;
    static constexpr uint32_t full = sz + (BITS == 4 ? S * kSzStage : 0);
    static constexpr uint32_t empty = full + 8 * S;
    static constexpr uint32_t abort_flag = empty + 8 * S;
    static constexpr uint32_t end = abort_flag + 16;
    static constexpr uint32_t bytes = end + 1024;                // + alignment slack
};
static_assert(kMaxCtasPerSm * (Layout<4>::bytes + 1024) <= 228 * 1024, "int4 ring fits 3 CTAs");
static_assert(kMaxCtasPerSm * (Layout<8>::bytes + 1024) <= 228 * 1024, "int8 ring fits 3 CTAs");

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

__device__ __forceinline__ void cp_async4(uint32_t dst, const void *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
// Arrive on `bar` once every cp.async this thread issued so far has landed
// (the arrival is counted in the barrier's expected count: no increment).
__device__ __forceinline__ void cp_async_arrive_noinc(uint32_t bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(addr));
    return v;
}

// Codes of the lane's four rows from a stage.  int4: row r at 64 r, lane t
// reads bytes 16t..16t+15 (rows g and g+1 of an 8-lane phase are adjacent:
// 128 consecutive bytes).  int8: row r at 128 r with the 128-byte swizzle
// (16-byte chunk c stored at chunk c ^ (r & 7)); lane t reads chunks 2t and
// 2t+1, and r & 7 == g for every row of the lane.
template <int BITS>
__device__ __forceinline__ void read_codes(RowWords<BITS> &rw, uint32_t stage, int row0, int g,
                                           int t) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint32_t row = stage + (uint32_t)(row0 + 8 * j) * kRowBytes<BITS>;
        if (BITS == 4) {
            const uint4 v = lds128(row + 16u * t);
            rw.w[j][0] = v.x; rw.w[j][1] = v.y; rw.w[j][2] = v.z; rw.w[j][3] = v.w;
        } else {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const uint4 v = lds128(row + 16u * ((2 * t + h) ^ g));
                rw.w[j][4 * h + 0] = v.x; rw.w[j][4 * h + 1] = v.y;
                rw.w[j][4 * h + 2] = v.z; rw.w[j][4 * h + 3] = v.w;
            }
        }
    }
}

struct GemvArgs {
    const uint16_t *a;
    const uint16_t *scales;
    const uint8_t *zeros;
    int M, N, K, group_size, group_shift;
    int bpg_shift;             // log2(group_size / 128) (ring path), else -1
    int kblocks;               // K / 128
    uint16_t *y;
    float *partials;
    uint32_t *counters;
    int64_t units;             // tasks * kblocks
    int64_t ctas;              // launched CTAs (each owns at least one unit)
    int slots;
    int prefetch_early;        // launch overlap: weights may be read before the grid wait
    uint64_t wait_limit;
    unsigned int *err_word;    // device error word (set when a bounded wait runs out)
};

// Scales and zeros of the lane's four rows for block kb, loaded directly
// (group sizes below 128, or scale/zero arrays the ring cannot gather).
__device__ __forceinline__ void load_params_direct(RowParams &rp, const GemvArgs &p,
                                                   const bool (&valid)[4], const int (&rows)[4],
                                                   int kb, int t) {
    const int k0 = kb * kBlockK + t * 32;
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
// through L1 (the vector is shared by every warp of the SM).
template <int MB>
__device__ __forceinline__ void load_act(Act<MB> &ac, const GemvArgs &p, int kb, int g, int t) {
    const int k0 = kb * kBlockK + t * 32;
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

// First CTA whose unit range contains unit u (ranges: [c*U/C, (c+1)*U/C)).
__device__ __forceinline__ int64_t cta_of_unit(int64_t u, int64_t U, int64_t C) {
    return ((u + 1) * C - 1) / U;
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

// acc[rt][mb][j] holds y[tok = 8mb + 2t + (j&1)][row = n0 + 16rt + g + 8(j>>1)]
// for the warp's 32 rows n0.. of task `task`.  `whole`: this CTA covered
// every K block of the task.  Otherwise the partial goes to slot (this CTA -
// the task's first CTA) of the warp's subtask and the last of the
// subtask's contributors adds the slots in order, lane l summing row l.
template <int MB>
__device__ __forceinline__ void gemv_flush(float (&acc)[2][MB][4], const GemvArgs &p, int task,
                                           int w, bool whole, int64_t cta, int lane) {
    const int g = lane >> 2, t = lane & 3;
    const int n0 = task * kTileRows + w * kRowsPerWarp;
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
                        p.y[(int64_t)tok * p.N + row] =
                            (uint16_t)dev::f32_to_bf16_rne(acc[rt][mb][j]);
                }
        return;
    }
    const int64_t first = cta_of_unit((int64_t)task * p.kblocks, p.units, p.ctas);
    const int64_t last = cta_of_unit((int64_t)(task + 1) * p.kblocks - 1, p.units, p.ctas);
    const int contributors = (int)(last - first + 1);
    const int64_t slot_elems = (int64_t)p.M * kRowsPerWarp;
    const int64_t sub = (int64_t)task * kConsumerWarps + w;
    float *base = p.partials + (sub * p.slots) * slot_elems;
    float *mine = base + (cta - first) * slot_elems;
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
    if (lane == 0) prev = atomicAdd(&p.counters[sub], 1u);
    prev = __shfl_sync(0xFFFFFFFFu, prev, 0);
    if (prev != (uint32_t)(contributors - 1)) return;
    __threadfence();
    // The last contributor: lane l adds row l of every slot in slot order,
    // for all tokens at once.
    reduce_slots<8 * MB, kRowsPerWarp>(base, slot_elems, contributors, p.M, lane, n0 + lane,
                                       p.N, p.y);
    if (lane == 0) p.counters[sub] = 0u;
}

// RING_SZ: int4 scales and zeros travel with the codes (group size a
// multiple of 128, 4-byte aligned arrays whose 4-byte words stay inside
// them).
template <int BITS, int MB, bool RING_SZ>
__global__ void __launch_bounds__(kThreads, kMaxCtasPerSm)
gemv_kernel(const __grid_constant__ CUtensorMap code_map, const GemvArgs p) {
    using L = Layout<BITS>;
    constexpr int S = L::S;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    volatile uint32_t *abort_flag = reinterpret_cast<volatile uint32_t *>(smem + L::abort_flag);
    auto full_bar = [&](int s) { return sbase + L::full + 8u * s; };
    auto empty_bar = [&](int s) { return sbase + L::empty + 8u * s; };

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t cta = blockIdx.x;
    const int64_t u_begin = cta * p.units / p.ctas;
    const int64_t u_end = (cta + 1) * p.units / p.ctas;
    const int KB = p.kblocks;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(full_bar(s), RING_SZ ? 1 + 32 : 1);   // TMA arrive + 32 gather arrivals
            mbar_init(empty_bar(s), kConsumerWarps);
        }
        *abort_flag = 0u;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&code_map))
                     : "memory");
    }
    __syncthreads();
    allow_dependents();

    if (warp == 0) {
        // ---------------- producer ----------------
        // Weights only: with launch overlap this may run before the previous
        // grid completes (the caller guarantees it does not write them).
        const int64_t gpr = p.K / p.group_size;
        const uint32_t *scale_words = reinterpret_cast<const uint32_t *>(p.scales);
        const uint32_t *zero_words = reinterpret_cast<const uint32_t *>(p.zeros);
        // the rows whose scale and zero words this lane gathers: rows
        // 32 (lane / 8) + (lane % 8) + 8j of the unit, into words 4 lane + j
        // of the stage's scale area (and of its zero area, 512 bytes on)
        const int prow = 32 * (lane >> 3) + (lane & 7);
        int task = (int)(u_begin / KB);
        int kb = (int)(u_begin - (int64_t)task * KB);
        int s = 0, r = 0;
        int64_t issued = 0;
        for (int64_t u = u_begin; u < u_end; ++u) {
            if (r > 0 && !mbar_wait(empty_bar(s), (r - 1) & 1, p.wait_limit, abort_flag,
                                    p.err_word))
                break;
            if (lane == 0) {
                mbar_arrive_expect_tx(full_bar(s), kCodeStage<BITS>);
                tma_load_2d(sbase + L::codes + s * kCodeStage<BITS>, &code_map,
                            kb * kRowBytes<BITS>, task * kTileRows, full_bar(s));
            }
            if (RING_SZ) {
                const uint32_t dst = sbase + L::sz + s * kSzStage + 16u * lane;
                const int gi = kb >> p.bpg_shift;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int row = task * kTileRows + prow + 8 * j;
                    if (row < p.N) {
                        const int64_t e = (int64_t)row * gpr + gi;
                        cp_async4(dst + 4u * j, scale_words + (e >> 1));
                        cp_async4(dst + 512u + 4u * j, zero_words + (e >> 2));
                    }
                }
                cp_async_arrive_noinc(full_bar(s));
            }
            ++issued;
            if (++kb == KB) {
                kb = 0;
                ++task;
            }
            if (++s == S) {
                s = 0;
                ++r;
            }
        }
        // every issued copy must have landed before the CTA may exit: the
        // last unit issued into stage q < issued is unit q + S * rq
#pragma unroll
        for (int q = 0; q < S; ++q)
            if (q < issued) {
                const int64_t rq = (issued - 1 - q) / S;
                mbar_drain(full_bar(q), (uint32_t)(rq & 1), p.err_word);
            }
        return;
    }

    // ---------------- consumers ----------------
    const int w = warp - 1;
    const int g = lane >> 2, t = lane & 3;
    if (p.prefetch_early) wait_for_previous_grid();   // before activations, y and workspace
    int task = (int)(u_begin / KB);
    int kb0 = (int)(u_begin - (int64_t)task * KB);
    int s = 0, r = 0;
    const int word_phase = (int)(((int64_t)g * (p.K / p.group_size)) & 3);
    for (int64_t u = u_begin; u < u_end;) {
        const int64_t kb_lim = kb0 + (u_end - u);
        const int kb_end = (int)(kb_lim < KB ? kb_lim : (int64_t)KB);
        const int nkb = kb_end - kb0;
        const int n0 = task * kTileRows + w * kRowsPerWarp;
        int rows[4];
        bool valid[4];
        uint32_t s8[4];                              // int8: (S, S) of rows g + 8j
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            rows[j] = n0 + g + 8 * j;
            valid[j] = rows[j] < p.N;
            s8[j] = (BITS == 8 && valid[j]) ? (uint32_t)__ldg(&p.scales[rows[j]]) * 0x00010001u
                                            : 0u;
        }
        float acc[2][MB][4];
#pragma unroll
        for (int rt = 0; rt < 2; ++rt)
#pragma unroll
            for (int mb = 0; mb < MB; ++mb)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[rt][mb][j] = 0.0f;

        for (int kb = kb0; kb < kb_end; ++kb) {
            Act<MB> ac;
            load_act(ac, p, kb, g, t);
            if (!mbar_wait(full_bar(s), r & 1, p.wait_limit, abort_flag, p.err_word)) return;
            const uint32_t stage = sbase + L::codes + s * kCodeStage<BITS>;
            RowWords<BITS> rw;
            read_codes<BITS>(rw, stage, w * kRowsPerWarp + g, g, t);
            RowParams rp;
            if (BITS == 4 && RING_SZ) {
                const uint32_t sz = sbase + L::sz + s * kSzStage + 16u * (8 * w + g);
                const uint4 ws = lds128(sz);
                const uint4 wz = lds128(sz + 512u);
                const int phase = word_phase + (kb >> p.bpg_shift);
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
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(empty_bar(s));   // the stage's data is in registers
            if (BITS == 4 && !RING_SZ) load_params_direct(rp, p, valid, rows, kb, t);
            compute_block<BITS, MB>(rp, ac, rw, s8, acc);
            if (++s == S) {
                s = 0;
                ++r;
            }
        }
        gemv_flush<MB>(acc, p, task, w, nkb == KB, cta, lane);
        u += nkb;
        ++task;
        kb0 = 0;
    }
}

int log2_exact(int64_t v) {
    if (v <= 0 || (v & (v - 1)) != 0) return -1;
    int s = 0;
    while ((int64_t(1) << s) < v) ++s;
    return s;
}

template <int BITS, int MB, bool RING_SZ>
qz_status launch_variant(const CUtensorMap &map, const GemvArgs &args, dim3 grid, int overlap,
                         cudaStream_t st) {
    constexpr int smem = Layout<BITS>::bytes;
    static DeviceOnce attr_once;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return QZ_ERR_CUDA;
    }
    if (attr_once.run(dev, [] {
            cudaError_t e = cudaFuncSetAttribute(gemv_kernel<BITS, MB, RING_SZ>,
                                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 smem);
            // three rings per SM need (nearly) all of the unified memory as
            // shared memory
            if (e == cudaSuccess)
                e = cudaFuncSetAttribute(gemv_kernel<BITS, MB, RING_SZ>,
                                         cudaFuncAttributePreferredSharedMemoryCarveout, 100);
            return e;
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
    cudaLaunchKernelEx(&cfg, gemv_kernel<BITS, MB, RING_SZ>, map, args);
    return launch_status();
}

template <int BITS>
qz_status launch_gemv(const void *a, const void *codes, const void *scales, const void *zeros,
                      int64_t M, int64_t N, int64_t K, int64_t group_size, void *y,
                      void *workspace, const GemvPlan &plan, int overlap, cudaStream_t st) {
    GemvArgs args;
    args.a = static_cast<const uint16_t *>(a);
    args.scales = static_cast<const uint16_t *>(scales);
    args.zeros = static_cast<const uint8_t *>(zeros);
    args.M = (int)M; args.N = (int)N; args.K = (int)K;
    args.group_size = (int)group_size;
    args.group_shift = log2_exact(group_size);
    args.bpg_shift = group_size % kBlockK == 0 ? log2_exact(group_size / kBlockK) : -1;
    args.kblocks = (int)(K / kBlockK);
    args.y = static_cast<uint16_t *>(y);
    args.partials = nullptr;
    args.counters = nullptr;
    if (plan.total_bytes > 0) {
        args.partials = static_cast<float *>(workspace);
        args.counters =
            reinterpret_cast<uint32_t *>(static_cast<char *>(workspace) + plan.partial_bytes);
    }
    args.units = plan.tasks * plan.kblocks;
    args.ctas = plan.ctas;
    args.slots = (int)plan.slots;
    args.prefetch_early = overlap;
    args.wait_limit = device_wait_limit();
    args.err_word = device_error_word();
    if (args.err_word == nullptr) return QZ_ERR_CUDA;

    CUtensorMap map;
    const uint64_t row_bytes = (uint64_t)K * BITS / 8;
    if (!make_map_2d(&map, CU_TENSOR_MAP_DATA_TYPE_UINT8, codes, row_bytes, (uint64_t)N,
                     row_bytes, kRowBytes<BITS>, kTileRows,
                     BITS == 4 ? CU_TENSOR_MAP_SWIZZLE_NONE : CU_TENSOR_MAP_SWIZZLE_128B))
        return QZ_ERR_CUDA;
    const dim3 grid((unsigned)plan.ctas);

    // The ring gathers the aligned 4-byte words holding each scale and zero;
    // they stay inside the arrays when N * K / g is a multiple of 4.
    if constexpr (BITS == 4) {
        const int64_t entries = N * (K / group_size);
        const bool ring_sz = args.bpg_shift >= 0 && aligned(scales, 4) && aligned(zeros, 4) &&
                             entries % 4 == 0;
        if (M <= 8)
            return ring_sz ? launch_variant<4, 1, true>(map, args, grid, overlap, st)
                           : launch_variant<4, 1, false>(map, args, grid, overlap, st);
        return ring_sz ? launch_variant<4, 2, true>(map, args, grid, overlap, st)
                       : launch_variant<4, 2, false>(map, args, grid, overlap, st);
    } else {
        return M <= 8 ? launch_variant<8, 1, false>(map, args, grid, overlap, st)
                      : launch_variant<8, 2, false>(map, args, grid, overlap, st);
    }
}

}  // namespace

// Stream-K plan.  Units are (128-row task x 128-wide K block); up to
// kMaxCtasPerSm CTAs run on an SM (their rings take 74 KB (int4) or 66 KB
// (int8) of shared memory each), and the same number k runs on every SM.
// k is the largest that still gives each CTA at least kMinUnitsPerCta units
// (more CTAs per SM keep more consumer warps issuing; fewer keep short
// layers from splitting every task over many CTAs).
constexpr int64_t kMinUnitsPerCta = 4;

GemvPlan gemv_plan(int64_t M, int64_t N, int64_t K, int bits, int sms) {
    (void)bits;
    GemvPlan p{};
    p.tasks = ceil_div(N, kTileRows);
    p.kblocks = K / kBlockK;
    const int64_t units = p.tasks * p.kblocks;
    int64_t per_sm = kMaxCtasPerSm;
    while (per_sm > 1 && units < (int64_t)sms * per_sm * kMinUnitsPerCta) --per_sm;
    p.ctas = (int64_t)sms * per_sm;
    // Fewer units than CTAs: one unit per CTA.  Every CTA must own at least
    // one unit, or a split task would count a contributor that never
    // arrives.
    if (p.ctas > units) p.ctas = units;
    // contributors of one task: at most ceil(KB / floor(U/C)) + 1
    const int64_t per_cta = units / p.ctas;
    p.slots = per_cta >= 1 ? ceil_div(p.kblocks, per_cta) + 1 : p.kblocks + 1;
    if (p.slots > p.kblocks) p.slots = p.kblocks;
    const int64_t subtasks = p.tasks * kConsumerWarps;
    p.partial_bytes = (size_t)subtasks * p.slots * (size_t)M * kRowsPerWarp * sizeof(float);
    p.partial_bytes = (p.partial_bytes + 255) & ~(size_t)255;
    p.counter_bytes = (size_t)ceil_div(subtasks, 64) * 64 * sizeof(uint32_t);
    p.total_bytes = p.partial_bytes + p.counter_bytes;
    return p;
}

// The plan's workspace is not monotone in the SM count, so the size callers
// allocate is the largest over every count up to kSmCount.
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
