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
// x 128 k (8 KB of int4 codes, 16 KB of int8) plus the unit's activations
// (M rows x 128 bf16).
//   * Producer (warp 0).  One lane issues TMA 2D copies of the unit's codes
//     and activations into the stage, completing on the stage's "full"
//     mbarrier with a transaction count.  Scales and zeros of int4 groups of
//     128 * 2^i reach shared memory in one of two ways.  When their rows are
//     16-byte multiples (K / g a multiple of 16), a TMA copy brings eight
//     groups of scales (and sixteen of zeros) for all 128 rows into one of
//     two "meta" slots with their own full/empty barriers, once per eight
//     groups.  Otherwise the 32 lanes gather, with 4-byte cp.async copies,
//     the aligned words holding each row's scale and zero into the stage and
//     signal its barrier when they land (cp.async.mbarrier.arrive.noinc).
//     The producer waits on a stage's (or meta slot's) "empty" barrier before
//     refilling it.  With launch overlap it copies weights before the
//     previous grid completes and activations only after.
//   * Consumers (warps 1..4).  Warp w owns rows 32w..32w+31 of each unit.
//     Lane (g = lane/4, t = lane%4) reads the 16 (int4) or 32 (int8) code
//     bytes of k = 32t..32t+31 of rows g, g+8, g+16, g+24 from the stage with
//     16-byte shared loads (int8 rows are 128 B, loaded with the 128-byte
//     swizzle so that those loads are free of bank conflicts), its tokens'
//     activations of the same k, and the four rows' scales and zeros,
//     dequantizes in registers to bf16 exactly as qz_dequantize forms each
//     weight, and releases the stage once its MMAs have consumed every
//     loaded register (a release right after the loads let a refill
//     overwrite a stage whose loads had not yet returned, seen with fewer
//     registers per thread).  int4: a LOP3 builds bf16(128 + q) for
//     two nibbles, add.rn.bf16x2 of bf16(-(128 + Z)) leaves q - Z exactly,
//     mul.rn.bf16x2 by the bf16 scale rounds S*(q - Z) once.  int8: the byte
//     (XOR 0x80) is placed in the mantissa of 2^23, one packed fp32
//     subtraction gives a pair of q exactly, the pair is packed to bf16
//     exactly and mul.rn.bf16x2 rounds S*q once.
//   * A byte of codes yields the pairs (q_j, q_{j+4}), so the K axis is
//     permuted consistently for both MMA operands: the pairs are the A
//     operand (16 rows x 16 k) of mma.sync m16n8k16 with fp32 accumulation
//     and the activations (tokens as the 8 columns) are the B operand,
//     permuted to match with PRMT once per k for both 16-row tiles of the
//     warp.  For M > 8 a second MMA covers tokens 8..15.  Columns of tokens
//     >= M read token M-1's activations; their outputs are dropped.
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
constexpr int kMaxCtasPerSm = 3;
// CTAs per SM of a variant: tokens in groups of 8 (MB groups); M > 16
// (integer formats) takes larger stages and more registers: two CTAs per SM
// for MB = 4, one for MB = 8 (64 accumulators per thread).
template <int MB, int HALVES = 1>
constexpr int kCtasPerSm = MB <= 2 ? (HALVES == 2 && MB == 2 ? 2 : kMaxCtasPerSm)
                                   : (MB == 4 ? 2 : 1);
// Independent MMA accumulator chains per 16-row tile for M <= 8: the MMAs of
// even and odd code words accumulate separately (summed at the flush), so a
// warp has twice as many MMAs in flight.
constexpr int kAccChains = 2;
template <int MB>
constexpr int kChains = MB == 1 ? kAccChains : 1;
// Shared memory one CTA may use so that kCtasPerSm fit on an SM (228 KB,
// 1 KB of it reserved per CTA), less the slack for aligning the base.
template <int MB, int HALVES = 1>
constexpr int kCtaSmemBudget = 228 * 1024 / kCtasPerSm<MB, HALVES> - 1024 - 1024;

// How int4 scales and zeros reach shared memory (see the header comment).
enum Meta { kMetaNone = 0, kMetaGather = 1, kMetaTma = 2 };
// Weight format: integer codes with scale (and zero), or FP4 (E2M1) codes
// with MXFP4 (32-value blocks, E8M0 scales) or NVFP4 (16-value blocks, E4M3
// scales and one fp32 tensor scale) block scales.
enum Fmt { kFmtInt = 0, kFmtMx = 1, kFmtNv = 2 };
constexpr int kFp4MetaBytes = kTileRows * 32;                  // 32 scale bytes per row
constexpr int kMetaGroups = 8;                                 // scale groups per meta slot
constexpr int kMetaScaleBytes = kTileRows * 16;                // 8 bf16 scales per row
constexpr int kMetaZeroBytes = kTileRows * 16;                 // 16 zeros per row

// Shared-memory layout (offsets from the 1024-byte aligned base): S stages
// of [codes | activations (8 MB rows) | gathered scale/zero words], then the
// two meta slots [scales | zeros], then the barriers.
template <int BITS, int MB, int META, int FMT = kFmtInt, int HALVES = 1>
struct Layout {
    static constexpr int code = kCodeStage<BITS> * HALVES;              // code bytes per stage
    static constexpr int act = 8 * MB * kBlockK * HALVES * 2;           // bytes per stage
    static constexpr int stage = code + act + (META == kMetaGather ? kSzStage : 0);
    static constexpr int meta = META == kMetaTma ? 2 * (kMetaScaleBytes + kMetaZeroBytes) : 0;
    static constexpr int lut = FMT == kFmtNv ? 512 : 0;                 // E4M3 -> bf16 table
    static constexpr int S = (kCtaSmemBudget<MB, HALVES> - meta - lut - 256) / stage;
    static constexpr uint32_t codes = 0;                                 // + s * stage
    static constexpr uint32_t act_off = code;                            // within a stage
    static constexpr uint32_t sz_off = code + act;                       // within a stage
    static constexpr uint32_t meta_base = S * stage;
    static constexpr uint32_t lut_base = meta_base + meta;
    static constexpr uint32_t full = lut_base + lut;
    static constexpr uint32_t empty = full + 8 * S;
    static constexpr uint32_t meta_full = empty + 8 * S;
    static constexpr uint32_t meta_empty = meta_full + 16;
    static constexpr uint32_t abort_flag = meta_empty + 16;
    static constexpr uint32_t end = abort_flag + 16;
    static constexpr uint32_t bytes = end + 1024;                        // + alignment slack
    static_assert(stage % 1024 == 0, "stages keep the 1024-byte alignment of the swizzled codes");
    static_assert(S >= 3, "at least three stages in flight");
    static_assert(end + 1024 <= kCtaSmemBudget<MB, HALVES> + 1024, "the CTAs fit on an SM");
};

// bf16 pair (nibble j, nibble j+4) of a code word: bf16_rne(S * (q - Z)).
// nz2 holds bf16(-(128 + Z)) twice.
__device__ __forceinline__ uint32_t dequant_pair_u4(uint32_t word, int j, uint32_t s2,
                                                    uint32_t nz2) {
    const uint32_t x = dev::and_or<0x000F000Fu>(word >> (4 * j), 0x43004300u);   // bf16(128+q)
    return dev::bf16x2_mul(dev::bf16x2_add(x, nz2), s2);
}

// bf16 pair (code c_j, code c_{j+4}) of 8 consecutive int8 codes held in
// words lo (c0..c3) and hi (c4..c7), already XORed with 0x80808080: both
// bytes go into the mantissa of 2^23, one packed subtraction gives the pair
// of q exactly (dev::i8_codes_bf16x2), and mul.rn.bf16x2 by (S, S) rounds
// S*q once, as qz_dequantize does.
__device__ __forceinline__ uint32_t dequant_pair_i8(uint32_t lo, uint32_t hi, int j, uint32_t s2) {
    const uint32_t sel = (uint32_t)j | 0x7540u;            // bytes: byte j, 0, 0, 0x4B
    return dev::bf16x2_mul(
        dev::i8_codes_bf16x2(dev::prmt(lo, 0x4B000000u, sel), dev::prmt(hi, 0x4B000000u, sel)), s2);
}

// FP4: the four natural-order bf16 pairs (q0,q1), (q2,q3), (q4,q5), (q6,q7)
// of the E2M1 values of a code word (code k in bits 4k..4k+3: sign in bit 3,
// magnitude index in bits 0..2).  Two 8-entry byte tables (PRMT) give the low
// and high byte of bf16(|v|) for the magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6;
// PRMT's sign-replicate mode spreads each code's sign bit over a byte mask,
// merged into the high bytes; two more PRMTs interleave low and high bytes.
__device__ __forceinline__ void fp4_pairs(uint32_t w, uint32_t (&p)[4]) {
    constexpr uint32_t kLo0 = 0xC0800000u, kLo1 = 0xC0804000u;   // low bytes, magnitudes 0..7
    constexpr uint32_t kHi0 = 0x3F3F3F00u, kHi1 = 0x40404040u;   // high bytes
    const uint32_t mag = w & 0x77777777u;
    const uint32_t mag_hi = mag >> 16;
    const uint32_t w4 = w << 4;                      // code 2i's sign at bit 7 of byte i
    const uint32_t lo_a = dev::prmt(kLo0, kLo1, mag), lo_b = dev::prmt(kLo0, kLo1, mag_hi);
    uint32_t hi_a = dev::prmt(kHi0, kHi1, mag), hi_b = dev::prmt(kHi0, kHi1, mag_hi);
    // byte k of the mask: 0xFF when code k (k = 0..3, then 4..7) is negative
    hi_a = dev::and_or<0x80808080u>(dev::prmt(w4, w, 0xD9C8u), hi_a);
    hi_b = dev::and_or<0x80808080u>(dev::prmt(w4, w, 0xFBEAu), hi_b);
    p[0] = dev::prmt(lo_a, hi_a, 0x5140u);
    p[1] = dev::prmt(lo_a, hi_a, 0x7362u);
    p[2] = dev::prmt(lo_b, hi_b, 0x5140u);
    p[3] = dev::prmt(lo_b, hi_b, 0x7362u);
}

// E8M0 byte -> (2^(b-127), 2^(b-127)) as bf16 bits (b = 0 is the subnormal 2^-127).
__device__ __forceinline__ uint32_t e8m0_pair(uint32_t b) {
    const uint32_t h = b == 0u ? 0x0040u : (b << 7);
    return h * 0x00010001u;
}

// E4M3 byte (non-negative scale) -> bf16 bits (exact).
__device__ __forceinline__ uint32_t e4m3_bf16(uint32_t b) {
    const uint32_t e = (b >> 3) & 15u, m = b & 7u;
    if (e == 0) return __float_as_uint((float)m * 0.001953125f) >> 16;   // m * 2^-9
    return ((e + 120u) << 7) | (m << 4);
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
    // FP4, rows g + 8j: (s, s) of the lane's first and second 16-value block
    // (MXFP4: both the one 32-value block)
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

// Activations of one 128-wide half h of a two-half unit for tokens g (and
// g + 8), clamped to M - 1.  The unit's 256 k arrive as four boxes of 64 k
// (128-byte token rows, 128-byte swizzle: 16-byte chunk c of token row r at
// chunk c ^ (r % 8)), box b at act + b * MB KB; lane t reads k = 32t..32t+31
// of the half: chunks 4(t % 2)..4(t % 2)+3 of box 2h + t / 2.  Tokens g of a
// warp then spread over all banks (unswizzled 512-byte rows put the eight
// tokens' chunks in the same banks).
template <int MB>
__device__ __forceinline__ void load_act_sw(Act<MB> &ac, uint32_t act, int M, int g, int t,
                                            int h) {
    const uint32_t box = act + (uint32_t)(2 * h + (t >> 1)) * (MB * 1024u);
#pragma unroll
    for (int mb = 0; mb < MB; ++mb) {
        const int tok = min(8 * mb + g, M - 1);
        const uint32_t row = box + (uint32_t)tok * 128u;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint4 v = lds128(row + 16u * (uint32_t)((((t & 1) * 4) + q) ^ (tok & 7)));
            ac.x[mb][4 * q + 0] = v.x; ac.x[mb][4 * q + 1] = v.y;
            ac.x[mb][4 * q + 2] = v.z; ac.x[mb][4 * q + 3] = v.w;
        }
    }
}

// int4 units of two 128-wide halves: 128-byte rows stored with the 128-byte
// swizzle (16-byte chunk c of row r at chunk c ^ (r % 8)); half h of lane t is
// chunk 4h + t, and r % 8 == g for the lane's four rows.
__device__ __forceinline__ void read_codes_half(RowWords<4> &rw, uint32_t stage, int row0, int g,
                                                int t, int h) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint32_t row = stage + (uint32_t)(row0 + 8 * j) * 128u;
        const uint4 v = lds128(row + 16u * (uint32_t)((4 * h + t) ^ g));
        rw.w[j][0] = v.x; rw.w[j][1] = v.y; rw.w[j][2] = v.z; rw.w[j][3] = v.w;
    }
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
    const uint16_t *scales;
    const uint8_t *fp4_scales;  // FP4 block scales (N x K / block bytes)
    const float *tensor_scale;  // NVFP4 tensor scale
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
    int meta_span_shift;       // log2(units per meta slot) (kMetaTma)
    int fp4_bpu_shift;         // FP4: log2(scale blocks per 128-wide unit)
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

// Activations of one unit for tokens g (and g + 8), clamped to M - 1, from
// the stage: token rows of 256 bytes, lane t reading bytes 64t..64t+63.
template <int MB>
__device__ __forceinline__ void load_act(Act<MB> &ac, uint32_t act, int M, int g, int t,
                                         uint32_t pitch = kBlockK * 2) {
#pragma unroll
    for (int mb = 0; mb < MB; ++mb) {
        const int tok = min(8 * mb + g, M - 1);
        const uint32_t src = act + (uint32_t)tok * pitch + 64u * t;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint4 v = lds128(src + 16u * q);
            ac.x[mb][4 * q + 0] = v.x; ac.x[mb][4 * q + 1] = v.y;
            ac.x[mb][4 * q + 2] = v.z; ac.x[mb][4 * q + 3] = v.w;
        }
    }
}

template <int BITS, int MB>
__device__ __forceinline__ void compute_block(const RowParams &rp, const Act<MB> &ac,
                                              const RowWords<BITS> &rw, const uint32_t (&s8)[4],
                                              float (&acc)[kChains<MB>][2][MB][4]) {
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
                    dev::mma_bf16_16816(acc[i % kChains<MB>][rt][mb], a0, a1, a2, a3, b0[mb],
                                        b1[mb]);
            }
        }
    }
}

// M > 16: the activations stay in the stage.  Per code word i the A
// fragments of both halves and both 16-row tiles are formed once; then, per
// group of 8 tokens (g + 8mb, clamped to M - 1), one 16-byte shared load
// gives that token's 8 activations of the word, so only one group's worth is
// live in registers.
template <int BITS, int MB>
__device__ __forceinline__ void compute_block_wide(const RowParams &rp, uint32_t act, int M,
                                                   int g, int t, const RowWords<BITS> &rw,
                                                   const uint32_t (&s8)[4],
                                                   float (&acc)[1][2][MB][4]) {
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
        uint32_t af[2][2][4];                      // [h][rt][a0..a3]
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int rt = 0; rt < 2; ++rt) {
                const int ja = 2 * rt, jb = 2 * rt + 1;
                if (BITS == 4) {
                    af[h][rt][0] = dequant_pair_u4(rw.w[ja][i], 2 * h, rp.s2[ja], rp.z2[ja]);
                    af[h][rt][1] = dequant_pair_u4(rw.w[jb][i], 2 * h, rp.s2[jb], rp.z2[jb]);
                    af[h][rt][2] = dequant_pair_u4(rw.w[ja][i], 2 * h + 1, rp.s2[ja], rp.z2[ja]);
                    af[h][rt][3] = dequant_pair_u4(rw.w[jb][i], 2 * h + 1, rp.s2[jb], rp.z2[jb]);
                } else {
                    af[h][rt][0] = dequant_pair_i8(lo8[ja], hi8[ja], 2 * h, s8[ja]);
                    af[h][rt][1] = dequant_pair_i8(lo8[jb], hi8[jb], 2 * h, s8[jb]);
                    af[h][rt][2] = dequant_pair_i8(lo8[ja], hi8[ja], 2 * h + 1, s8[ja]);
                    af[h][rt][3] = dequant_pair_i8(lo8[jb], hi8[jb], 2 * h + 1, s8[jb]);
                }
            }
#pragma unroll
        for (int mb = 0; mb < MB; ++mb) {
            const int tok = min(8 * mb + g, M - 1);
            const uint4 v = lds128(act + (uint32_t)tok * (kBlockK * 2) + 64u * t + 16u * i);
            const uint32_t x[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const uint32_t b0 = dev::prmt(x[h], x[h + 2], 0x5410);
                const uint32_t b1 = dev::prmt(x[h], x[h + 2], 0x7632);
#pragma unroll
                for (int rt = 0; rt < 2; ++rt)
                    dev::mma_bf16_16816(acc[0][rt][mb], af[h][rt][0], af[h][rt][1],
                                        af[h][rt][2], af[h][rt][3], b0, b1);
            }
        }
    }
}

// FP4 codes, natural k order: for word i and half h the MMA's k are
// 8i + 4h .. 8i + 4h + 3 of the lane's 32 for both operands, so the
// activations need no permute.  The block scale multiplies exactly (a bf16
// E2M1 value times an E8M0 or E4M3 scale has at most 6 significant bits).
template <int MB>
__device__ __forceinline__ void compute_block_fp4(const uint32_t (&sa)[4], const uint32_t (&sb)[4],
                                                  const Act<MB> &ac, const RowWords<4> &rw,
                                                  float (&acc)[kChains<MB>][2][MB][4]) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        uint32_t pr[4][4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            fp4_pairs(rw.w[j][i], pr[j]);
            const uint32_t sc = i < 2 ? sa[j] : sb[j];
#pragma unroll
            for (int q = 0; q < 4; ++q) pr[j][q] = dev::bf16x2_mul(pr[j][q], sc);
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
#pragma unroll
            for (int rt = 0; rt < 2; ++rt) {
                const int ja = 2 * rt, jb = 2 * rt + 1;
#pragma unroll
                for (int mb = 0; mb < MB; ++mb)
                    dev::mma_bf16_16816(acc[i % kChains<MB>][rt][mb], pr[ja][2 * h],
                                        pr[jb][2 * h], pr[ja][2 * h + 1], pr[jb][2 * h + 1],
                                        ac.x[mb][4 * i + 2 * h], ac.x[mb][4 * i + 2 * h + 1]);
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
                                             int N, uint16_t *y, float out_scale) {
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
        if (row < N) y[row] = (uint16_t)dev::f32_to_bf16_rne(sum * out_scale);
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
            if (t < M) y[(int64_t)t * N + row] = (uint16_t)dev::f32_to_bf16_rne(sum[t] * out_scale);
    }
}

// acc[rt][mb][j] holds y[tok = 8mb + 2t + (j&1)][row = n0 + 16rt + g + 8(j>>1)]
// for the warp's 32 rows n0.. of task `task`.  `whole`: this CTA covered
// every K block of the task.  Otherwise the partial goes to slot (this CTA -
// the task's first CTA) of the warp's subtask and the last of the
// subtask's contributors adds the slots in order, lane l summing row l.
// `out_scale` multiplies the sums before the bf16 rounding (NVFP4's tensor
// scale; 1 otherwise, which changes nothing).
template <int MB>
__device__ __forceinline__ void gemv_flush(float (&acc)[2][MB][4], const GemvArgs &p, int task,
                                           int w, bool whole, int64_t cta, int lane,
                                           float out_scale) {
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
                            (uint16_t)dev::f32_to_bf16_rne(acc[rt][mb][j] * out_scale);
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
                                       p.N, p.y, out_scale);
    if (lane == 0) p.counters[sub] = 0u;
}

// The kernel.  META: how int4 scales and zeros arrive (kMetaNone: int8's
// per-row scales, or int4 groups loaded directly by the consumers).  HALVES:
// 128-wide K blocks per unit (2: int4 units of 128 rows x 256 k, one
// 128-byte row of codes per weight row, consumed as two halves).  ACTSW
// (two-half units): activations as four swizzled 64-k boxes (load_act_sw),
// else one box of 256 k (one token: its lanes of equal t read the same words).
template <int BITS, int MB, int META, int FMT, int HALVES = 1, bool ACTSW = true>
__global__ void __launch_bounds__(kThreads, (kCtasPerSm<MB, HALVES>))
gemv_kernel(const __grid_constant__ CUtensorMap code_map,
            const __grid_constant__ CUtensorMap act_map,
            const __grid_constant__ CUtensorMap scale_map,
            const __grid_constant__ CUtensorMap zero_map, const GemvArgs p) {
    using L = Layout<BITS, MB, META, FMT, HALVES>;
    static_assert(HALVES == 1 ||
                      (BITS == 4 && MB <= 2 &&
                       (META == kMetaTma || (FMT == kFmtInt && META == kMetaGather))),
                  "two-half units: 4-bit codes with scales by TMA (int4 also by gathered "
                  "words), up to 16 tokens");
    constexpr int S = L::S;
    constexpr bool kFp4 = FMT != kFmtInt;
    constexpr uint32_t kMetaBytes = kFp4 ? kFp4MetaBytes : kMetaScaleBytes + kMetaZeroBytes;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    volatile uint32_t *abort_flag = reinterpret_cast<volatile uint32_t *>(smem + L::abort_flag);
    auto full_bar = [&](int s) { return sbase + L::full + 8u * s; };
    auto empty_bar = [&](int s) { return sbase + L::empty + 8u * s; };
    auto meta_full_bar = [&](int m) { return sbase + L::meta_full + 8u * m; };
    auto meta_empty_bar = [&](int m) { return sbase + L::meta_empty + 8u * m; };
    auto stage_addr = [&](int s) { return sbase + L::codes + (uint32_t)s * L::stage; };
    auto meta_addr = [&](int m) { return sbase + L::meta_base + (uint32_t)m * kMetaBytes; };

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t cta = blockIdx.x;
    const int64_t u_begin = cta * p.units / p.ctas;
    const int64_t u_end = (cta + 1) * p.units / p.ctas;
    const int KB = p.kblocks;
    const uint32_t act_bytes = (uint32_t)p.M * kBlockK * HALVES * 2;
    // a meta slot holds 8 groups: 8 << bpg_shift units of one task
    const int span_mask = META == kMetaTma ? (1 << p.meta_span_shift) - 1 : 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(full_bar(s), META == kMetaGather ? 1 + 32 : 1);   // + 32 gather arrivals
            mbar_init(empty_bar(s), kConsumerWarps);
        }
        for (int m = 0; m < 2; ++m) {
            mbar_init(meta_full_bar(m), 1);
            mbar_init(meta_empty_bar(m), kConsumerWarps);
        }
        *abort_flag = 0u;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&code_map))
                     : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&act_map))
                     : "memory");
    }
    if (FMT == kFmtNv)        // E4M3 byte -> bf16 bits
        for (int b = threadIdx.x; b < 256; b += blockDim.x)
            reinterpret_cast<uint16_t *>(smem + L::lut_base)[b] = (uint16_t)e4m3_bf16((uint32_t)b);
    __syncthreads();
    allow_dependents();

    if (warp == 0) {
        // ---------------- producer ----------------
        const int64_t gpr = p.K / p.group_size;
        const uint32_t *scale_words = reinterpret_cast<const uint32_t *>(p.scales);
        const uint32_t *zero_words = reinterpret_cast<const uint32_t *>(p.zeros);
        // gather path: rows 32 (lane / 8) + (lane % 8) + 8j of the unit, into
        // words 4 lane + j of the stage's scale area (and zero area, +512)
        const int prow = 32 * (lane >> 3) + (lane & 7);
        int task = (int)(u_begin / KB);
        int kb = (int)(u_begin - (int64_t)task * KB);
        int s = 0, r = 0, spans = 0;
        int64_t issued = 0;
        // Launch overlap: the first units' weights may be fetched while the
        // previous grid finishes, their activations only once it has
        // completed.  The early phase ends before the producer's first
        // blocking wait (a stage or meta slot to refill), which needs the
        // consumers to have used units whose activations are still to come.
        bool early_phase = p.prefetch_early != 0;
        int64_t no_act = 0;                          // early units without activations
        const int task0 = (int)(u_begin / KB);
        const int kb_first = (int)(u_begin - (int64_t)task0 * KB);
        // a unit's activations: one box of 128 k (256 k: two-half units
        // without ACTSW), or four swizzled boxes of 64 k (load_act_sw)
        auto load_unit_act = [&](int st, int kbx) {
            if constexpr (HALVES == 2 && ACTSW) {
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    tma_load_2d(stage_addr(st) + L::act_off + (uint32_t)i * (MB * 1024u), &act_map,
                                kbx * kBlockK * HALVES + 64 * i, 0, full_bar(st));
            } else {
                tma_load_2d(stage_addr(st) + L::act_off, &act_map, kbx * kBlockK * HALVES, 0,
                            full_bar(st));
            }
        };
        auto finish_early = [&]() {
            if (!early_phase) return;
            early_phase = false;
            wait_for_previous_grid();
            if (lane == 0) {
                int kb2 = kb_first;
                for (int64_t i = 0; i < no_act; ++i) {
                    load_unit_act((int)i, kb2);
                    if (++kb2 == KB) kb2 = 0;
                }
            }
        };
        bool ok = true;
        for (int64_t u = u_begin; u < u_end && ok; ++u) {
            if (META == kMetaTma && (u == u_begin || (kb & span_mask) == 0)) {
                const int m = spans & 1;
                if (spans >= 2) {
                    finish_early();
                    if (!mbar_wait(meta_empty_bar(m), ((spans >> 1) - 1) & 1, p.wait_limit,
                                   abort_flag, p.err_word)) {
                        ok = false;
                        break;
                    }
                }
                if (lane == 0) {
                    mbar_arrive_expect_tx(meta_full_bar(m), kMetaBytes);
                    if (kFp4) {
                        // 32 scale bytes (blocks) of each of the 128 rows
                        tma_load_2d(meta_addr(m), &scale_map,
                                    ((kb * HALVES) << p.fp4_bpu_shift) & ~31,
                                    task * kTileRows, meta_full_bar(m));
                    } else {
                        const int gi = (kb * HALVES) >> p.bpg_shift;
                        tma_load_2d(meta_addr(m), &scale_map, gi & ~(kMetaGroups - 1),
                                    task * kTileRows, meta_full_bar(m));
                        tma_load_2d(meta_addr(m) + kMetaScaleBytes, &zero_map, gi & ~15,
                                    task * kTileRows, meta_full_bar(m));
                    }
                }
                ++spans;
            }
            if (r > 0) {
                finish_early();
                if (!mbar_wait(empty_bar(s), (r - 1) & 1, p.wait_limit, abort_flag, p.err_word)) {
                    ok = false;
                    break;
                }
            }
            if (lane == 0) {
                mbar_arrive_expect_tx(full_bar(s), (uint32_t)L::code + act_bytes);
                tma_load_2d(stage_addr(s), &code_map, kb * kRowBytes<BITS> * HALVES,
                            task * kTileRows, full_bar(s));
                if (!early_phase) load_unit_act(s, kb);
            }
            if (META == kMetaGather) {
                const uint32_t dst = stage_addr(s) + L::sz_off + 16u * lane;
                // two-half units: the first half's group; the second half's
                // scale and zero share its words (even groups per row)
                const int gi = (kb * HALVES) >> p.bpg_shift;
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
            if (early_phase) ++no_act;
            if (++kb == KB) {
                kb = 0;
                ++task;
            }
            if (++s == S) {
                s = 0;
                ++r;
            }
        }
        finish_early();                              // ranges shorter than the ring
        // every issued copy must have landed before the CTA may exit: the
        // last unit issued into stage q < issued is unit q + S * rq
#pragma unroll 1
        for (int q = 0; q < S; ++q)
            if (q < issued) {
                const int64_t rq = (issued - 1 - q) / S;
                mbar_drain(full_bar(q), (uint32_t)(rq & 1), p.err_word);
            }
        if (META == kMetaTma)
            for (int m = 0; m < 2; ++m)
                if (m < spans) mbar_drain(meta_full_bar(m), (uint32_t)(((spans - 1 - m) >> 1) & 1),
                                          p.err_word);
        return;
    }

    // ---------------- consumers ----------------
    const int w = warp - 1;
    const int g = lane >> 2, t = lane & 3;
    if (p.prefetch_early) wait_for_previous_grid();   // before y and the workspace
    int task = (int)(u_begin / KB);
    int kb0 = (int)(u_begin - (int64_t)task * KB);
    int s = 0, r = 0, spans = 0;
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
        float acc[kChains<MB>][2][MB][4];
#pragma unroll
        for (int c = 0; c < kChains<MB>; ++c)
#pragma unroll
            for (int rt = 0; rt < 2; ++rt)
#pragma unroll
                for (int mb = 0; mb < MB; ++mb)
#pragma unroll
                    for (int j = 0; j < 4; ++j) acc[c][rt][mb][j] = 0.0f;

        for (int kb = kb0; kb < kb_end; ++kb) {
            int m = 0;
            if (META == kMetaTma) {
                m = (spans - 1) & 1;
                if (kb == kb0 && u == u_begin ? true : (kb & span_mask) == 0) {
                    m = spans & 1;
                    if (!mbar_wait(meta_full_bar(m), (spans >> 1) & 1, p.wait_limit, abort_flag,
                                   p.err_word))
                        return;
                    ++spans;
                }
            }
            if (!mbar_wait(full_bar(s), r & 1, p.wait_limit, abort_flag, p.err_word)) return;
            if constexpr (HALVES == 2) {
                // two 128-wide halves: each its own codes, activations and
                // group scale/zero; the stage is released after both halves'
                // MMAs
                const uint32_t stage = stage_addr(s);
                const uint32_t ms = meta_addr(m) + 16u * (uint32_t)(w * kRowsPerWarp + g);
                uint4 gs = make_uint4(0u, 0u, 0u, 0u), gz = gs;     // gathered words
                if constexpr (META == kMetaGather) {
                    const uint32_t sz = stage + L::sz_off + 16u * (8 * w + g);
                    gs = lds128(sz);
                    gz = lds128(sz + 512u);
                }
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    Act<MB> ac;
                    if constexpr (ACTSW)
                        load_act_sw(ac, stage + L::act_off, p.M, g, t, h);
                    else
                        load_act(ac, stage + L::act_off + (uint32_t)h * (kBlockK * 2), p.M, g, t,
                                 kBlockK * 2 * HALVES);
                    RowWords<4> rw;
                    read_codes_half(rw, stage, w * kRowsPerWarp + g, g, t, h);
                    RowParams rp;
                    uint32_t fa[4], fb[4];                   // FP4 block scales, rows g + 8j
                    const int gi = (kb * 2 + h) >> p.bpg_shift;
                    if constexpr (kFp4) {
                        // the half's blocks in the meta slot (32 scale bytes per row)
                        const int blk = ((kb * 2 + h) << p.fp4_bpu_shift) +
                                        (FMT == kFmtMx ? t : 2 * t);
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const uint32_t a = meta_addr(m) +
                                               32u * (uint32_t)(w * kRowsPerWarp + g + 8 * j) +
                                               (uint32_t)(blk & 31);
                            uint32_t b0, b1 = 0u;
                            asm volatile("ld.shared.u8 %0, [%1];" : "=r"(b0) : "r"(a));
                            if (FMT == kFmtNv)
                                asm volatile("ld.shared.u8 %0, [%1];" : "=r"(b1) : "r"(a + 1u));
                            if (FMT == kFmtMx) {
                                fa[j] = fb[j] = e8m0_pair(b0);
                            } else {
                                const uint16_t *lut =
                                    reinterpret_cast<const uint16_t *>(smem + L::lut_base);
                                fa[j] = (uint32_t)lut[b0] * 0x00010001u;
                                fb[j] = (uint32_t)lut[b1] * 0x00010001u;
                            }
                        }
                    } else if constexpr (META == kMetaGather) {
                        // the group's position in the words the producer
                        // gathered for the unit's first group
                        const int phase = word_phase + gi;
                        const uint32_t os = (uint32_t)(phase & 1) * 2u, oz = (uint32_t)(phase & 3);
                        const uint32_t sel_s = os * 0x0101u + (os + 1u) * 0x1010u;   // (S, S)
                        const uint32_t sel_z = oz * 0x0101u + 0x4040u;               // (0xC3, Z) x 2
                        const uint32_t wsv[4] = {gs.x, gs.y, gs.z, gs.w};
                        const uint32_t wzv[4] = {gz.x, gz.y, gz.z, gz.w};
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            rp.s2[j] = dev::prmt(wsv[j], 0u, sel_s);
                            rp.z2[j] = dev::prmt(wzv[j], 0xC3C3C3C3u, sel_z);
                        }
                    } else {
                        const uint32_t sc = ms + 2u * (uint32_t)(gi & (kMetaGroups - 1));
                        const uint32_t zc = ms + kMetaScaleBytes + (uint32_t)(gi & 15);
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            uint32_t sv, zv;
                            asm volatile("ld.shared.u16 %0, [%1];" : "=r"(sv) : "r"(sc + 128u * j));
                            asm volatile("ld.shared.u8 %0, [%1];" : "=r"(zv) : "r"(zc + 128u * j));
                            rp.s2[j] = sv * 0x00010001u;
                            rp.z2[j] = (0xC300u + zv) * 0x00010001u;
                        }
                    }
                    if constexpr (kFp4)
                        compute_block_fp4<MB>(fa, fb, ac, rw, acc);
                    else
                        compute_block<4, MB>(rp, ac, rw, s8, acc);
                }
                // Both halves' registers have been consumed by their MMAs, so
                // every shared-memory load of the stage (and of the meta
                // slot, on its last unit) has returned: only now may the
                // producer refill them.
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(empty_bar(s));
                    if (META == kMetaTma && (kb + 1 == KB || ((kb + 1) & span_mask) == 0 ||
                                             u + (kb - kb0) + 1 == u_end))
                        mbar_arrive(meta_empty_bar(m));
                }
            } else {
            const uint32_t stage = stage_addr(s);
            constexpr bool kWide = MB > 2;
            Act<kWide ? 1 : MB> ac;
            if constexpr (!kWide) load_act(ac, stage + L::act_off, p.M, g, t);
            RowWords<BITS> rw;
            read_codes<BITS>(rw, stage, w * kRowsPerWarp + g, g, t);
            RowParams rp;
            if (BITS == 4 && !kFp4 && META == kMetaGather) {
                const uint32_t sz = stage + L::sz_off + 16u * (8 * w + g);
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
            uint32_t fa[4], fb[4];                       // FP4 block scales, rows g + 8j
            if constexpr (kFp4) {
                const int blk = (kb << p.fp4_bpu_shift) + (FMT == kFmtMx ? t : 2 * t);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int r_in = w * kRowsPerWarp + g + 8 * j;
                    uint32_t b0, b1;
                    if (META == kMetaTma) {
                        const uint32_t a = meta_addr(m) + 32u * (uint32_t)r_in + (uint32_t)(blk & 31);
                        asm volatile("ld.shared.u8 %0, [%1];" : "=r"(b0) : "r"(a));
                        if (FMT == kFmtNv)
                            asm volatile("ld.shared.u8 %0, [%1];" : "=r"(b1) : "r"(a + 1u));
                    } else {
                        const int64_t e = (int64_t)rows[j] * (p.K >> (7 - p.fp4_bpu_shift)) + blk;
                        b0 = valid[j] ? __ldg(p.fp4_scales + e) : 0u;
                        if (FMT == kFmtNv) b1 = valid[j] ? __ldg(p.fp4_scales + e + 1) : 0u;
                    }
                    if (FMT == kFmtMx) {
                        fa[j] = fb[j] = e8m0_pair(b0);
                    } else {
                        const uint16_t *lut = reinterpret_cast<const uint16_t *>(smem + L::lut_base);
                        fa[j] = (uint32_t)lut[b0] * 0x00010001u;
                        fb[j] = (uint32_t)lut[b1] * 0x00010001u;
                    }
                }
            }
            if (BITS == 4 && !kFp4 && META == kMetaTma) {
                // row r's eight scales (16 B) at meta + 16 r, its sixteen
                // zeros at meta + 2048 + 16 r
                const int gi = kb >> p.bpg_shift;
                const uint32_t ms = meta_addr(m) + 16u * (uint32_t)(w * kRowsPerWarp + g);
                const uint32_t sc = ms + 2u * (uint32_t)(gi & (kMetaGroups - 1));
                const uint32_t zc = ms + kMetaScaleBytes + (uint32_t)(gi & 15);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    uint32_t sv, zv;
                    asm volatile("ld.shared.u16 %0, [%1];" : "=r"(sv) : "r"(sc + 128u * j));
                    asm volatile("ld.shared.u8 %0, [%1];" : "=r"(zv) : "r"(zc + 128u * j));
                    rp.s2[j] = sv * 0x00010001u;                      // (S, S)
                    rp.z2[j] = (0xC300u + zv) * 0x00010001u;          // bf16(-(128 + Z)) twice
                }
            }
            if constexpr (kFp4) {
                compute_block_fp4<MB>(fa, fb, ac, rw, acc);
            } else if constexpr (kWide) {
                if (BITS == 4 && META == kMetaNone) load_params_direct(rp, p, valid, rows, kb, t);
                compute_block_wide<BITS, MB>(rp, stage + L::act_off, p.M, g, t, rw, s8, acc);
            } else {
                if (BITS == 4 && META == kMetaNone) load_params_direct(rp, p, valid, rows, kb, t);
                compute_block<BITS, MB>(rp, ac, rw, s8, acc);
            }
            // The MMAs have consumed every register loaded from the stage
            // (and from the meta slot), so those loads have returned: the
            // producer may refill them.  On the meta slot's last unit the
            // next unit starts a new slot.
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(empty_bar(s));
                if (META == kMetaTma && (kb + 1 == KB || ((kb + 1) & span_mask) == 0 ||
                                         u + (kb - kb0) + 1 == u_end))
                    mbar_arrive(meta_empty_bar(m));
            }
            }
            if (++s == S) {
                s = 0;
                ++r;
            }
        }
#pragma unroll
        for (int c = 1; c < kChains<MB>; ++c)
#pragma unroll
            for (int rt = 0; rt < 2; ++rt)
#pragma unroll
                for (int mb = 0; mb < MB; ++mb)
#pragma unroll
                    for (int j = 0; j < 4; ++j) acc[0][rt][mb][j] += acc[c][rt][mb][j];
        gemv_flush<MB>(acc[0], p, task, w, nkb == KB, cta, lane,
                       FMT == kFmtNv ? __ldg(p.tensor_scale) : 1.0f);
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

struct Maps {
    CUtensorMap code, act, scale, zero;
};

template <int BITS, int MB, int META, int FMT, int HALVES = 1, bool ACTSW = true>
qz_status launch_variant(const Maps &maps, const GemvArgs &args, dim3 grid, int overlap,
                         cudaStream_t st) {
    constexpr int smem = Layout<BITS, MB, META, FMT, HALVES>::bytes;
    static DeviceOnce attr_once;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return QZ_ERR_CUDA;
    }
    if (attr_once.run(dev, [] {
            cudaError_t e = cudaFuncSetAttribute(gemv_kernel<BITS, MB, META, FMT, HALVES, ACTSW>,
                                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 smem);
            // three rings per SM need (nearly) all of the unified memory as
            // shared memory
            if (e == cudaSuccess)
                e = cudaFuncSetAttribute(gemv_kernel<BITS, MB, META, FMT, HALVES, ACTSW>,
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
    cudaLaunchKernelEx(&cfg, gemv_kernel<BITS, MB, META, FMT, HALVES, ACTSW>, maps.code, maps.act,
                       maps.scale, maps.zero, args);
    return launch_status();
}

template <int BITS, int META, int FMT = kFmtInt>
qz_status launch_mb(const Maps &maps, const GemvArgs &args, dim3 grid, int overlap,
                    cudaStream_t st) {
    if (args.M <= 8) return launch_variant<BITS, 1, META, FMT>(maps, args, grid, overlap, st);
    if (args.M <= 16 || FMT != kFmtInt)
        return launch_variant<BITS, 2, META, FMT>(maps, args, grid, overlap, st);
    if (args.M <= 32) return launch_variant<BITS, 4, META, kFmtInt>(maps, args, grid, overlap, st);
    return launch_variant<BITS, 8, META, kFmtInt>(maps, args, grid, overlap, st);
}

// How the int4 GEMV's scales and zeros reach shared memory: as TMA tiles
// (groups a multiple of 128, K/g a multiple of 16, both arrays 16-byte
// aligned), as gathered 4-byte words (groups a multiple of 128, arrays 4-byte
// aligned, N * K / g a multiple of 4 so every word lies inside its array), or
// loaded by the consumers.
int int4_meta(int64_t N, int64_t K, int64_t group_size, const void *scales, const void *zeros) {
    const int64_t gpr = K / group_size;
    const bool ring = group_size % kBlockK == 0 && log2_exact(group_size / kBlockK) >= 0;
    if (ring && gpr % 16 == 0 && aligned(scales, 16) && aligned(zeros, 16)) return kMetaTma;
    if (ring && aligned(scales, 4) && aligned(zeros, 4) && (N * gpr) % 4 == 0) return kMetaGather;
    return kMetaNone;
}

// Two-half units (256 k) need a ring metadata path, K % 256 == 0, and, with
// gathered words, the second half's scale and zero in the words of the
// first: the two halves share a group (g >= 256), or the row's group count
// is even (g = 128: the pair 2j, 2j+1 never straddles a scale or zero word).
bool two_half_ok(int64_t M, int64_t N, int64_t K, int64_t group_size, const void *scales,
                 const void *zeros) {
    if (M > 16 || K % (2 * kBlockK) != 0) return false;
    const int meta = int4_meta(N, K, group_size, scales, zeros);
    if (meta == kMetaTma) return true;
    return meta == kMetaGather && (group_size > kBlockK || (K / group_size) % 2 == 0);
}

template <int BITS>
qz_status launch_gemv(const void *a, const void *codes, const void *scales, const void *zeros,
                      int64_t M, int64_t N, int64_t K, int64_t group_size, void *y,
                      void *workspace, const GemvPlan &plan, int overlap, cudaStream_t st) {
    GemvArgs args;
    args.scales = static_cast<const uint16_t *>(scales);
    args.fp4_scales = nullptr;
    args.tensor_scale = nullptr;
    args.fp4_bpu_shift = 0;
    args.zeros = static_cast<const uint8_t *>(zeros);
    args.M = (int)M; args.N = (int)N; args.K = (int)K;
    args.group_size = (int)group_size;
    args.group_shift = log2_exact(group_size);
    args.bpg_shift = group_size % kBlockK == 0 ? log2_exact(group_size / kBlockK) : -1;
    // a meta slot holds 8 groups: 8 << bpg_shift blocks of 128 k, half as
    // many units when a unit is two blocks
    const int halves = plan.unit_k / kBlockK;
    args.meta_span_shift = args.bpg_shift >= 0 ? args.bpg_shift + 3 - (halves - 1) : 0;
    args.kblocks = (int)(K / plan.unit_k);
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

    Maps maps;
    const bool act_sw = halves == 2 && M > 1;      // see gemv_kernel's ACTSW
    const uint64_t row_bytes = (uint64_t)K * BITS / 8;
    // 128-byte code rows (int8, and int4 two-half units) take the 128-byte swizzle
    const bool swizzle = BITS == 8 || halves == 2;
    if (!make_map_2d_cached(&maps.code, CU_TENSOR_MAP_DATA_TYPE_UINT8, codes, row_bytes,
                            (uint64_t)N, row_bytes, kRowBytes<BITS> * halves, kTileRows,
                            swizzle ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !make_map_2d_cached(&maps.act, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a, (uint64_t)K,
                            (uint64_t)M, (uint64_t)K * 2, act_sw ? 64 : kBlockK * halves,
                            (uint32_t)M,
                            act_sw ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE))
        return QZ_ERR_CUDA;
    maps.scale = maps.code;   // unused unless kMetaTma
    maps.zero = maps.code;
    const dim3 grid((unsigned)plan.ctas);

    if constexpr (BITS == 4) {
        const int64_t gpr = K / group_size;
        const int meta = int4_meta(N, K, group_size, scales, zeros);
        if (halves == 2 && !two_half_ok(M, N, K, group_size, scales, zeros))
            return QZ_ERR_UNSUPPORTED;   // the plan's units need a ring metadata path
        if (meta == kMetaTma) {
            // eight groups of scales and sixteen of zeros per row, 128 rows
            if (!make_map_2d_cached(&maps.scale, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, scales,
                                    (uint64_t)gpr, (uint64_t)N, (uint64_t)gpr * 2, kMetaGroups,
                                    kTileRows, CU_TENSOR_MAP_SWIZZLE_NONE) ||
                !make_map_2d_cached(&maps.zero, CU_TENSOR_MAP_DATA_TYPE_UINT8, zeros,
                                    (uint64_t)gpr, (uint64_t)N, (uint64_t)gpr, 16, kTileRows,
                                    CU_TENSOR_MAP_SWIZZLE_NONE))
                return QZ_ERR_CUDA;
            if (halves == 2)
                return M == 1   ? launch_variant<4, 1, kMetaTma, kFmtInt, 2, false>(maps, args, grid,
                                                                                   overlap, st)
                       : M <= 8 ? launch_variant<4, 1, kMetaTma, kFmtInt, 2>(maps, args, grid,
                                                                          overlap, st)
                              : launch_variant<4, 2, kMetaTma, kFmtInt, 2>(maps, args, grid,
                                                                          overlap, st);
            return launch_mb<4, kMetaTma>(maps, args, grid, overlap, st);
        }
        // The gather path copies the aligned 4-byte words holding each scale
        // and zero.
        if (meta == kMetaGather) {
            if (halves == 2)
                return M == 1   ? launch_variant<4, 1, kMetaGather, kFmtInt, 2, false>(maps, args, grid,
                                                                                   overlap, st)
                       : M <= 8 ? launch_variant<4, 1, kMetaGather, kFmtInt, 2>(maps, args, grid,
                                                                          overlap, st)
                              : launch_variant<4, 2, kMetaGather, kFmtInt, 2>(maps, args, grid,
                                                                             overlap, st);
            return launch_mb<4, kMetaGather>(maps, args, grid, overlap, st);
        }
        return launch_mb<4, kMetaNone>(maps, args, grid, overlap, st);
    } else {
        return launch_mb<8, kMetaNone>(maps, args, grid, overlap, st);
    }
}

qz_status launch_fp4_gemv(const void *a, const void *codes, const void *scales,
                          const void *tensor_scale, int64_t M, int64_t N, int64_t K, int kind,
                          void *y, void *workspace, const GemvPlan &plan, int overlap,
                          cudaStream_t st) {
    GemvArgs args{};
    args.fp4_scales = static_cast<const uint8_t *>(scales);
    args.tensor_scale = static_cast<const float *>(tensor_scale);
    args.fp4_bpu_shift = kind == 0 ? 2 : 3;             // 4 or 8 scale blocks per 128 k
    const int halves = plan.unit_k / kBlockK;
    // 32 scale bytes per meta slot: 8 (MXFP4) or 4 (NVFP4) blocks of 128 k,
    // half as many units when a unit is two blocks
    args.meta_span_shift = 5 - args.fp4_bpu_shift - (halves - 1);
    args.M = (int)M; args.N = (int)N; args.K = (int)K;
    args.group_size = (int)K;                           // unused by the FP4 path
    args.group_shift = -1;
    args.bpg_shift = 0;
    args.kblocks = (int)(K / plan.unit_k);
    args.y = static_cast<uint16_t *>(y);
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
    Maps maps;
    const bool act_sw = halves == 2 && M > 1;      // see gemv_kernel's ACTSW
    const uint64_t row_bytes = (uint64_t)K / 2;
    if (!make_map_2d_cached(&maps.code, CU_TENSOR_MAP_DATA_TYPE_UINT8, codes, row_bytes,
                            (uint64_t)N, row_bytes, kRowBytes<4> * halves, kTileRows,
                            halves == 2 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !make_map_2d_cached(&maps.act, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a, (uint64_t)K,
                            (uint64_t)M, (uint64_t)K * 2, act_sw ? 64 : kBlockK * halves,
                            (uint32_t)M,
                            act_sw ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE))
        return QZ_ERR_CUDA;
    maps.scale = maps.code;
    maps.zero = maps.code;
    const dim3 grid((unsigned)plan.ctas);
    const int64_t blocks_per_row = K >> (7 - args.fp4_bpu_shift);
    const bool tma_meta = blocks_per_row % 16 == 0 && aligned(scales, 16);
    if (tma_meta &&
        !make_map_2d_cached(&maps.scale, CU_TENSOR_MAP_DATA_TYPE_UINT8, scales,
                            (uint64_t)blocks_per_row, (uint64_t)N, (uint64_t)blocks_per_row, 32,
                            kTileRows, CU_TENSOR_MAP_SWIZZLE_NONE))
        return QZ_ERR_CUDA;
    if (halves == 2) {
        if (!tma_meta || K % (2 * kBlockK) != 0) return QZ_ERR_UNSUPPORTED;
        if (kind == 0)
            return M == 1   ? launch_variant<4, 1, kMetaTma, kFmtMx, 2, false>(maps, args, grid, overlap, st)
                   : M <= 8 ? launch_variant<4, 1, kMetaTma, kFmtMx, 2>(maps, args, grid, overlap, st)
                          : launch_variant<4, 2, kMetaTma, kFmtMx, 2>(maps, args, grid, overlap, st);
        return M == 1   ? launch_variant<4, 1, kMetaTma, kFmtNv, 2, false>(maps, args, grid, overlap, st)
                   : M <= 8 ? launch_variant<4, 1, kMetaTma, kFmtNv, 2>(maps, args, grid, overlap, st)
                      : launch_variant<4, 2, kMetaTma, kFmtNv, 2>(maps, args, grid, overlap, st);
    }
    if (kind == 0)
        return tma_meta ? launch_mb<4, kMetaTma, kFmtMx>(maps, args, grid, overlap, st)
                        : launch_mb<4, kMetaNone, kFmtMx>(maps, args, grid, overlap, st);
    return tma_meta ? launch_mb<4, kMetaTma, kFmtNv>(maps, args, grid, overlap, st)
                    : launch_mb<4, kMetaNone, kFmtNv>(maps, args, grid, overlap, st);
}

}  // namespace

// Stream-K plan.  Units are (128-row task x unit_k-wide K block); up to
// kMaxCtasPerSm CTAs run on an SM (their rings take 74 KB (int4) or 66 KB
// (int8) of shared memory each), and the same number k runs on every SM.
// k is the largest that still gives each CTA at least kMinUnitsPerCta units
// (more CTAs per SM keep more consumer warps issuing; fewer keep short
// layers from splitting every task over many CTAs).
constexpr int64_t kMinUnitsPerCta = 4;

GemvPlan gemv_plan(int64_t M, int64_t N, int64_t K, int bits, int sms, int unit_k) {
    (void)bits;
    GemvPlan p{};
    p.unit_k = unit_k;
    p.tasks = ceil_div(N, kTileRows);
    p.kblocks = K / unit_k;
    const int64_t units = p.tasks * p.kblocks;
    // the minimum counts 128-wide blocks: two-half units count twice
    const int64_t min_units = kMinUnitsPerCta * kBlockK / unit_k;
    // (9..16 tokens in two-half units: two CTAs per SM, for four stages)
    int64_t per_sm = M <= 8 ? kMaxCtasPerSm
                            : M <= 16 ? (unit_k > kBlockK ? 2 : kMaxCtasPerSm) : (M <= 32 ? 2 : 1);
    while (per_sm > 1 && units < (int64_t)sms * per_sm * min_units) --per_sm;
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
// allocate is the largest over every count up to kSmCount, and over the unit
// widths up to max_unit_k (a call planned for 256-wide units falls back to
// 128 when its scale or zero array is not 16-byte aligned).
size_t gemv_workspace_bound(int64_t M, int64_t N, int64_t K, int bits, int max_unit_k) {
    (void)bits;
    size_t most = 0;
    for (int unit_k = kBlockK; unit_k <= max_unit_k; unit_k += kBlockK) {
        for (int sms = 1; sms <= kSmCount; ++sms) {
            const size_t b = gemv_plan(M, N, K, bits, sms, unit_k).total_bytes;
            if (b > most) most = b;
        }
    }
    return most;
}

// K per unit of the integer decode GEMV: 256 (two 128-wide halves, one
// 128-byte row of codes per weight row and half the per-unit overhead) for
// int4 with at most 16 tokens when K is a multiple of 256 and the groups'
// scales and zeros come through the ring (two_half_ok); otherwise 128.
// K per unit of the FP4A16 GEMV: 256 when K is a multiple of 512 (both
// kinds then get their block scales as TMA tiles: K/32 and K/16 multiples of
// 16) and the block-scale array is 16-byte aligned; otherwise 128.
int gemv_fp4_unit_k(int64_t M, int64_t K, const void *scales) {
    return M <= 16 && K % 512 == 0 && aligned(scales, 16) ? 2 * kBlockK : kBlockK;
}

int gemv_unit_k(int bits, int64_t M, int64_t N, int64_t K, int64_t group_size,
                const void *scales, const void *zeros) {
    if (bits != 4 || group_size <= 0 || K % group_size != 0) return kBlockK;
    return two_half_ok(M, N, K, group_size, scales, zeros) ? 2 * kBlockK : kBlockK;
}

qz_status launch_w4a16_gemv(const void *a, const void *codes, const void *scales,
                            const void *zeros, int64_t M, int64_t N, int64_t K,
                            int64_t group_size, void *y, void *workspace,
                            const GemvPlan &plan, int overlap, cudaStream_t st) {
    return launch_gemv<4>(a, codes, scales, zeros, M, N, K, group_size, y, workspace, plan,
                          overlap, st);
}

qz_status launch_fp4a16_gemv(const void *a, const void *codes, const void *scales,
                             const void *tensor_scale, int64_t M, int64_t N, int64_t K, int kind,
                             void *y, void *workspace, const GemvPlan &plan, int overlap,
                             cudaStream_t st) {
    return launch_fp4_gemv(a, codes, scales, tensor_scale, M, N, K, kind, y, workspace, plan,
                           overlap, st);
}

qz_status launch_w8a16_gemv(const void *a, const void *codes, const void *scales,
                            int64_t M, int64_t N, int64_t K, void *y, void *workspace,
                            const GemvPlan &plan, int overlap, cudaStream_t st) {
    return launch_gemv<8>(a, codes, scales, nullptr, M, N, K, K, y, workspace, plan, overlap,
                          st);
}

}  // namespace qz
