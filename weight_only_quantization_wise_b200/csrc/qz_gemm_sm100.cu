// qz_gemm_sm100.cu -- W4A16 and W8A16 prefill GEMMs on the sm_100a (tcgen05)
// tensor cores, and the device error word used by bounded device-side waits.
//
// Quantization concepts guide, "Quantize weights or activations": weight-only
// methods dequantize the weights to the compute dtype before each matmul;
// prefill and large batches are compute-bound, so this path must keep the
// tensor cores busy.  The GPTQ explainer: the dequantization happens inside
// the matmul kernel, with no separate conversion pass.
//
// y (M x N) = a (M x K) * w_hat^T with w_hat = bf16_rne(S * (q - Z)) (int4,
// group-wise scales and zeros) or w_hat = bf16_rne(S * q) (int8, symmetric,
// one scale per weight row).
//
// Persistent kernel: each CTA loops over tiles of 128 weight rows x 256
// tokens (tile t = blockIdx.x + i * gridDim.x).  The roles:
//   warp 0       TMA producer: per 64-wide K step, the activation tile
//                (256 tokens x 64 bf16, 128-byte swizzle) and the codes
//                (128 rows x 32 bytes of int4, or x 64 bytes of int8) into a
//                STAGES-deep shared-memory ring.
//   warp 1       allocates tensor memory; one lane issues tcgen05.mma.
//   warps 2..9   dequantize: warp w owns weight rows 32*(w%4) .. +31 (the
//                tensor-memory lane quarter that warp may access) and half of
//                the stage's K (warps 2..5 the first 32 k, 6..9 the second);
//                each thread turns 32 codes of its row into bf16 exactly as
//                qz_dequantize does and stores them with tcgen05.st as the A
//                operand of the MMA (A = weights in tensor memory, K-major,
//                2 bf16 per 32-bit column).
//   warps 10..13 epilogue: read the fp32 accumulators with tcgen05.ld, release
//                the accumulator for the next tile, round to bf16 into a
//                shared staging tile and write it with one TMA 2D store that
//                overlaps the next tile's main loop.
// The MMA is M = 128 (weight rows), N = 256 (tokens), K = 16, fp32
// accumulation in tensor memory (256 columns); B = activations from shared
// memory.  Each weight tile is dequantized once per 256 tokens.
//
// Every mbarrier wait is bounded by a caller-set time limit; on expiry
// the thread records the fault in g_device_error_word and in a CTA-local
// abort flag, every role stops issuing work, in-flight copies and MMAs are
// drained (with bounded waits), tensor memory is released and the CTA exits.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "qz_sm100.cuh"

namespace qz {

// Set (atomicOr) by a kernel whose bounded wait ran out.
__device__ unsigned int g_device_error_word = 0;

namespace {

using namespace sm100;

constexpr int kTileN = 128;               // weight rows per tile (MMA M)
constexpr int kTileM = 256;               // tokens per tile (MMA N)
constexpr int kTileK = 64;                // K per stage
template <int BITS>
constexpr int kPackStageBytes = kTileN * kTileK * BITS / 8;   // 4 KB (int4), 8 KB (int8)
constexpr int kACols = kTileK / 2;                       // A columns per stage (bf16 pairs)
constexpr int kTmemCols = 512;
constexpr int kDequantWarps = 8;
constexpr int kMetaFifo = 2;              // groups of scales/zeros loaded ahead
constexpr int kMaxSplits = 4;             // split-K ranges per tile at most
constexpr int kMaxStages = 16;            // ring depth at most
constexpr int kEpilogueWarps = 4;
constexpr int kFirstEpilogueWarp = 2 + kDequantWarps;
constexpr int kThreads = 32 * (2 + kDequantWarps + kEpilogueWarps);
constexpr int kSmemLimit = 227 * 1024;    // dynamic shared memory of one CTA
constexpr int kSmemPerSm = 228 * 1024;    // shared memory of an SM (1 KB of it reserved per CTA)
// Short token tiles (at most kPairMaxRows tokens) run two CTAs per SM, each
// with half of the tensor memory, so that twice as many warps dequantize.
constexpr int kPairMaxRows = 64;

// Shared- and tensor-memory layout of one launch.  The activation box holds
// act_rows tokens (a multiple of 16, at most 256), so a stage takes
// act_rows x 128 bytes of activations plus the codes of 128 rows, and the
// ring is as deep as shared memory (and the A slots in tensor memory) allow:
// short token tiles get more stages in flight to cover the memory latency.
struct GemmLayout {
    int stages;
    uint32_t act_stage, pack_stage;
    // byte offsets from the 1024-aligned base
    uint32_t act, pack, staging, full, empty, afull, dfull, dempty, drain, tmem_slot,
        abort_flag, epi_decision, epi_last, end;
    uint32_t a_col0;   // first tensor-memory column of the A slots (accumulator at 0)
};

__host__ __device__ constexpr GemmLayout gemm_layout(int bits, int act_rows, int stages) {
    GemmLayout L{};
    L.stages = stages;
    L.act_stage = (uint32_t)act_rows * kTileK * 2;
    L.pack_stage = (uint32_t)(kTileN * kTileK * bits / 8);
    L.act = 0;
    L.pack = L.act + stages * L.act_stage;
    L.staging = L.pack + stages * L.pack_stage;
    L.full = L.staging + (uint32_t)act_rows * kTileN * 2;
    L.empty = L.full + 8 * stages;
    L.afull = L.empty + 8 * stages;
    L.dfull = L.afull + 8 * stages;
    L.dempty = L.dfull + 8;
    L.drain = L.dempty + 8;
    L.tmem_slot = L.drain + 8;
    L.abort_flag = L.tmem_slot + 4;
    L.epi_decision = L.abort_flag + 4;
    L.epi_last = L.epi_decision + 4;
    L.end = L.epi_last + 4;
    L.a_col0 = (uint32_t)((act_rows + 31) & ~31);
    return L;
}

constexpr int gemm_ctas_per_sm(int act_rows) { return act_rows <= kPairMaxRows ? 2 : 1; }

// Deepest ring that fits for this activation box, with `ctas` CTAs per SM
// sharing its shared and tensor memory.
constexpr int gemm_stages(int bits, int act_rows, int ctas = 1) {
    const int smem = ctas == 1 ? kSmemLimit : kSmemPerSm / ctas - 1024;
    int s = kMaxStages;
    while (s > 2 && gemm_layout(bits, act_rows, s).end + 1024 > (uint32_t)smem) --s;
    const int by_tmem = (kTmemCols / ctas - (int)gemm_layout(bits, act_rows, 1).a_col0) / kACols;
    return s < by_tmem ? s : by_tmem;
}
static_assert(gemm_stages(4, kPairMaxRows, 2) >= 4 && gemm_stages(8, kPairMaxRows, 2) >= 4,
              "paired CTAs keep at least four stages");
constexpr int kFullTileStages = 4;
static_assert(gemm_stages(4, kTileM) == kFullTileStages && gemm_stages(8, kTileM) == kFullTileStages,
              "a full token tile keeps four stages");
static_assert(gemm_stages(4, 16) == kMaxStages - 1 || gemm_stages(4, 16) == kMaxStages,
              "short token tiles get a deep ring");

// Bounded waits that report through this file's device error word.
__device__ __forceinline__ bool gemm_wait(uint32_t bar, uint32_t parity, uint64_t limit_ns,
                                          volatile uint32_t *abort_flag) {
    return mbar_wait(bar, parity, limit_ns, abort_flag, &g_device_error_word);
}
__device__ __forceinline__ void gemm_drain(uint32_t bar, uint32_t parity) {
    mbar_drain(bar, parity, &g_device_error_word);
}

__device__ __forceinline__ void tma_store_2d(const CUtensorMap *map, uint32_t src, int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
            reinterpret_cast<uint64_t>(map)),
        "r"(src), "r"(x), "r"(y)
        : "memory");
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

__device__ __forceinline__ void tma_store_wait_read() {
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}

__device__ __forceinline__ void tma_store_wait_all() {
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

__device__ __forceinline__ void epilogue_bar_sync() {
    asm volatile("bar.sync 1, %0;" ::"n"(32 * kEpilogueWarps) : "memory");
}

// int8 codes: bf16 pair (byte 2i, byte 2i+1) of word wx (the code word XOR
// 0x80808080).  Bits 0x4B000000 | byte form the fp32 2^23 + q + 128; one
// subtraction leaves q exactly, the pair packs to bf16 exactly (|q| <= 127)
// and mul.rn.bf16x2 by (S, S) rounds S*q once, as qz_dequantize does.
__device__ __forceinline__ uint32_t dequant_pair_i8_nat(uint32_t wx, int i, uint32_t s2) {
    const float f0 = __uint_as_float(dev::prmt(wx, 0x4B000000u, (uint32_t)(2 * i) | 0x7540u));
    const float f1 = __uint_as_float(dev::prmt(wx, 0x4B000000u, (uint32_t)(2 * i + 1) | 0x7540u));
    return dev::bf16x2_mul(dev::pack_bf16x2(__fsub_rn(f0, 8388736.0f), __fsub_rn(f1, 8388736.0f)),
                           s2);
}

// Work item: one 128-row x 256-token output tile and, when the tiles are
// fewer than the SMs, one of `splits` equal K ranges of it (split-K).
struct WorkItem {
    int tile, split, n0, m0, kt0, kt1;
};
__device__ __forceinline__ WorkItem work_item(int item, int splits, int tiles_n, int KT) {
    WorkItem w;
    w.tile = item / splits;
    w.split = item - w.tile * splits;
    w.n0 = (w.tile % tiles_n) * kTileN;
    w.m0 = (w.tile / tiles_n) * kTileM;
    w.kt0 = (int)((int64_t)w.split * KT / splits);
    w.kt1 = (int)((int64_t)(w.split + 1) * KT / splits);
    return w;
}

// MMA N for a tile: its tokens rounded up to 16 (the kind::f16 granularity).
__device__ __forceinline__ int mma_n(int M, int m0) {
    const int mt = M - m0 < kTileM ? M - m0 : kTileM;
    return (mt + 15) & ~15;
}

// FIXED_STAGES > 0: full 256-token tiles, no split-K, a ring of that depth,
// the layout known at compile time (the large-M path); 0: layout from the
// launch's activation box and ring depth, split-K allowed.
template <int BITS, int FIXED_STAGES>
__device__ __forceinline__ GemmLayout kernel_layout(int act_rows, int stages) {
    if constexpr (FIXED_STAGES > 0) {
        constexpr GemmLayout L = gemm_layout(BITS, kTileM, FIXED_STAGES);
        return L;
    } else {
        return gemm_layout(BITS, act_rows, stages);
    }
}

template <int BITS, int FIXED_STAGES, int CTAS>
__global__ void __launch_bounds__(kThreads, CTAS)
wa16_gemm_tcgen05(const __grid_constant__ CUtensorMap act_map,
                   const __grid_constant__ CUtensorMap pack_map,
                   const __grid_constant__ CUtensorMap y_map,
                   const uint16_t *__restrict__ scales, const uint8_t *__restrict__ zeros,
                   int M, int N, int K, int group_size, uint16_t *__restrict__ y,
                   int use_tma_store, int act_rows, int stages_rt, int splits,
                   float *__restrict__ partials, uint32_t *__restrict__ counters,
                   uint64_t wait_limit) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const int stages = FIXED_STAGES > 0 ? FIXED_STAGES : stages_rt;
    if (FIXED_STAGES > 0) splits = 1;             // the host launches it only unsplit
    const GemmLayout SmemLayout = kernel_layout<BITS, FIXED_STAGES>(act_rows, stages_rt);
    constexpr int kPackBytes = kPackStageBytes<BITS>;
    const uint32_t kActStageBytes = SmemLayout.act_stage;
    volatile uint32_t *abort_flag = reinterpret_cast<volatile uint32_t *>(smem + SmemLayout.abort_flag);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + SmemLayout.tmem_slot);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int KT = K / kTileK;
    const int tiles_n = (N + kTileN - 1) / kTileN;
    const int tiles = tiles_n * ((M + kTileM - 1) / kTileM);
    const int items = tiles * splits;
    const uint32_t act_bytes = kActStageBytes;                    // one activation box

    auto full_bar = [&](int s) { return sbase + SmemLayout.full + 8 * s; };
    auto empty_bar = [&](int s) { return sbase + SmemLayout.empty + 8 * s; };
    auto afull_bar = [&](int s) { return sbase + SmemLayout.afull + 8 * s; };
    const uint32_t dfull_bar = sbase + SmemLayout.dfull;
    const uint32_t dempty_bar = sbase + SmemLayout.dempty;
    const uint32_t drain_bar = sbase + SmemLayout.drain;

    if (threadIdx.x == 0) {
        for (int s = 0; s < stages; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1 + kDequantWarps);   // MMA commit + dequant warps
            mbar_init(afull_bar(s), kDequantWarps);
        }
        mbar_init(dfull_bar, 1);
        mbar_init(dempty_bar, kEpilogueWarps);
        mbar_init(drain_bar, 1);
        *abort_flag = 0u;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&act_map)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&pack_map)) : "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(tmem_slot)),
                     "r"(kTmemCols / CTAS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const uint32_t tmem_acc = tmem_base;                     // columns [0, act_rows)
    const uint32_t tmem_a = tmem_base + SmemLayout.a_col0;   // A slots: stages x 32 columns

    if (warp == 0) {
        // ---------------- TMA producer ----------------
        if (lane == 0) {
            int issued_round[kMaxStages];
            for (int s = 0; s < kMaxStages; ++s) issued_round[s] = -1;
            int s = 0, r = 0;                         // ring slot and its round
            bool ok = true;
            for (int item = blockIdx.x; item < items && ok; item += gridDim.x) {
                const WorkItem wk = work_item(item, splits, tiles_n, KT);
                for (int kt = wk.kt0; kt < wk.kt1; ++kt, s = (s + 1 == stages ? 0 : s + 1),
                         r += (s == 0)) {
                    if (r > 0 && !gemm_wait(empty_bar(s), (r - 1) & 1, wait_limit, abort_flag)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(full_bar(s), act_bytes + kPackBytes);
                    tma_load_2d(sbase + SmemLayout.act + s * kActStageBytes, &act_map,
                                kt * kTileK, wk.m0, full_bar(s));
                    tma_load_2d(sbase + SmemLayout.pack + s * kPackBytes, &pack_map,
                                kt * (kTileK * BITS / 8), wk.n0, full_bar(s));
                    issued_round[s] = r;
                }
            }
            // every issued copy must have landed before the CTA may exit
            for (int q = 0; q < stages; ++q)
                if (issued_round[q] >= 0) gemm_drain(full_bar(q), issued_round[q] & 1);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            bool ok = true;
            int s = 0, r = 0, tcount = 0;
            for (int item = blockIdx.x; item < items && ok; item += gridDim.x, ++tcount) {
                const WorkItem wk = work_item(item, splits, tiles_n, KT);
                const uint32_t idesc = idesc_bf16(kTileN, mma_n(M, wk.m0));
                if (tcount > 0 && !gemm_wait(dempty_bar, (tcount - 1) & 1, wait_limit, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                for (int kt = wk.kt0; kt < wk.kt1;
                     ++kt, s = (s + 1 == stages ? 0 : s + 1), r += (s == 0)) {
                    ok = gemm_wait(full_bar(s), r & 1, wait_limit, abort_flag) &&
                         gemm_wait(afull_bar(s), r & 1, wait_limit, abort_flag);
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t act_addr = sbase + SmemLayout.act + s * kActStageBytes;
#pragma unroll
                    for (int j = 0; j < kTileK / 16; ++j)
                        mma_ts(tmem_acc, tmem_a + s * kACols + j * 8,
                               smem_desc_sw128(act_addr + j * 32), idesc,
                               (kt > wk.kt0 || j > 0) ? 1u : 0u);
                    mma_commit(empty_bar(s));
                }
                if (ok) mma_commit(dfull_bar);
            }
            // every issued MMA must finish before tensor memory is released
            mma_commit(drain_bar);
            gemm_drain(drain_bar, 0);
        }
        __syncwarp();
    } else if (warp < kFirstEpilogueWarp) {
        // ---------------- dequantize (warps 2..9) ----------------
        const int quarter = warp & 3;                 // tensor-memory lane quarter
        const int khalf = (warp - 2) / 4;             // which 32 of the 64 k of a stage
        const int row_local = quarter * 32 + lane;
        const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
        int s = 0, r = 0;                             // ring slot and its round
        bool ok = true;
        for (int item = blockIdx.x; item < items && ok; item += gridDim.x) {
            const WorkItem wk = work_item(item, splits, tiles_n, KT);
            const int n = wk.n0 + row_local;
            // Rows beyond N: the codes are TMA fill (zero) and the scale is
            // taken as 0, so their A entries are +-0 and their outputs are
            // never stored.
            const bool valid = n < N;
            if constexpr (BITS == 4) {
                const int gpr = K / group_size;
                const int spg = group_size / kTileK;      // stages per group
                const uint16_t *srow = scales + (int64_t)(valid ? n : 0) * gpr;
                const uint8_t *zrow = zeros + (int64_t)(valid ? n : 0) * gpr;
                const int g0 = wk.kt0 / spg;              // group of the first stage
                int kt = wk.kt0;
                // One stage: convert the codes of slot s with scale bits sb and zero zb.
                auto stage = [&](uint32_t sb, uint32_t zb) -> bool {
                    // warp-uniform: the tcgen05.st below needs every lane
                    if (!__all_sync(0xFFFFFFFFu,
                                    gemm_wait(full_bar(s), r & 1, wait_limit, abort_flag)))
                        return false;
                    const uint4 p = *reinterpret_cast<const uint4 *>(
                        smem + SmemLayout.pack + s * kPackBytes + row_local * (kTileK / 2) +
                        khalf * 16);
                    __syncwarp();
                    if (lane == 0) mbar_arrive(empty_bar(s));   // code stage consumed
                    const uint32_t s2 = sb * 0x00010001u;
                    const uint32_t z2 = (0x4300u + zb) * 0x00010001u;
                    const uint32_t words[4] = {p.x, p.y, p.z, p.w};
                    uint32_t a[16];
#pragma unroll
                    for (int wi = 0; wi < 4; ++wi) {
                        const uint32_t w = words[wi], w4 = w >> 4;
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            a[wi * 4 + i] = dequant_pair_nat(w, w4, i, s2, z2);
                    }
                    tmem_st_x16(tmem_a + lane_base + s * kACols + khalf * 16, a);
                    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(afull_bar(s));
                    ++kt;
                    s = s + 1 == stages ? 0 : s + 1;
                    r += (s == 0);
                    return true;
                };
                const bool quads = (gpr & 3) == 0 && (reinterpret_cast<uintptr_t>(scales) & 7) == 0 &&
                                   (reinterpret_cast<uintptr_t>(zeros) & 3) == 0;
                if (quads) {
                    // Scales and zeros of four consecutive groups come in one 8-byte
                    // and one 4-byte load.  Two register sets alternate over the
                    // quads, and a set is reloaded only after its quad is done, so a
                    // load is issued four groups before its first use and no
                    // register holding a load in flight is ever copied.
                    const uint2 *squad = reinterpret_cast<const uint2 *>(srow);
                    const uint32_t *zquad = reinterpret_cast<const uint32_t *>(zrow);
                    const int nq = gpr >> 2;
                    int qa = g0 >> 2, gi = g0 & 3, st = wk.kt0 - g0 * spg;
                    int qb = qa + 1;
                    uint2 sA = (valid && qa < nq) ? __ldg(&squad[qa]) : make_uint2(0u, 0u);
                    uint32_t zA = (valid && qa < nq) ? __ldg(&zquad[qa]) : 0u;
                    uint2 sB = (valid && qb < nq) ? __ldg(&squad[qb]) : make_uint2(0u, 0u);
                    uint32_t zB = (valid && qb < nq) ? __ldg(&zquad[qb]) : 0u;
                    // the stages of groups gi..3 of one quad
                    auto run_quad = [&](uint2 sw, uint32_t zw) {
                        for (; gi < 4 && kt < wk.kt1 && ok; ++gi, st = 0) {
                            const uint32_t sb = ((gi < 2 ? sw.x : sw.y) >> (16 * (gi & 1))) & 0xFFFFu;
                            const uint32_t zb = (zw >> (8 * gi)) & 0xFFu;
                            for (; st < spg && kt < wk.kt1; ++st)
                                if (!stage(sb, zb)) {
                                    ok = false;
                                    break;
                                }
                        }
                        gi = 0;
                    };
                    while (true) {
                        run_quad(sA, zA);
                        if (kt >= wk.kt1 || !ok) break;
                        qa += 2;
                        sA = (valid && qa < nq) ? __ldg(&squad[qa]) : make_uint2(0u, 0u);
                        zA = (valid && qa < nq) ? __ldg(&zquad[qa]) : 0u;
                        run_quad(sB, zB);
                        if (kt >= wk.kt1 || !ok) break;
                        qb += 2;
                        sB = (valid && qb < nq) ? __ldg(&squad[qb]) : make_uint2(0u, 0u);
                        zB = (valid && qb < nq) ? __ldg(&zquad[qb]) : 0u;
                    }
                } else {
                    // Scales and zeros of the next kMetaFifo groups wait in a
                    // register FIFO (a group spans spg stages); no per-stage
                    // index arithmetic is needed.
                    uint32_t sq[kMetaFifo], zq[kMetaFifo];
#pragma unroll
                    for (int q = 0; q < kMetaFifo; ++q) {
                        sq[q] = (valid && g0 + q < gpr) ? __ldg(&srow[g0 + q]) : 0u;
                        zq[q] = (valid && g0 + q < gpr) ? __ldg(&zrow[g0 + q]) : 0u;
                    }
                    int stage_in_group = wk.kt0 - g0 * spg, next_group = g0 + kMetaFifo;
                    while (kt < wk.kt1) {
                        const uint32_t sb = sq[0], zb = zq[0];
                        if (++stage_in_group == spg) {       // the next stage starts a new group
                            stage_in_group = 0;
#pragma unroll
                            for (int q = 0; q < kMetaFifo - 1; ++q) {
                                sq[q] = sq[q + 1];
                                zq[q] = zq[q + 1];
                            }
                            sq[kMetaFifo - 1] =
                                (valid && next_group < gpr) ? __ldg(&srow[next_group]) : 0u;
                            zq[kMetaFifo - 1] =
                                (valid && next_group < gpr) ? __ldg(&zrow[next_group]) : 0u;
                            ++next_group;
                        }
                        if (!stage(sb, zb)) {
                            ok = false;
                            break;
                        }
                    }
                }
            } else {
                // one scale per weight row for the whole K
                const uint32_t s2 = valid ? (uint32_t)__ldg(&scales[n]) * 0x00010001u : 0u;
                for (int kt = wk.kt0; kt < wk.kt1;
                     ++kt, s = (s + 1 == stages ? 0 : s + 1), r += (s == 0)) {
                    if (!__all_sync(0xFFFFFFFFu,
                                    gemm_wait(full_bar(s), r & 1, wait_limit, abort_flag))) {
                        ok = false;
                        break;
                    }
                    const uint8_t *src =
                        smem + SmemLayout.pack + s * kPackBytes + row_local * kTileK + khalf * 32;
                    const uint4 p0 = *reinterpret_cast<const uint4 *>(src);
                    const uint4 p1 = *reinterpret_cast<const uint4 *>(src + 16);
                    __syncwarp();
                    if (lane == 0) mbar_arrive(empty_bar(s));   // code stage consumed
                    const uint32_t words[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
                    uint32_t a[16];
#pragma unroll
                    for (int wi = 0; wi < 8; ++wi) {
                        const uint32_t wx = words[wi] ^ 0x80808080u;
#pragma unroll
                        for (int i = 0; i < 2; ++i)
                            a[wi * 2 + i] = dequant_pair_i8_nat(wx, i, s2);
                    }
                    tmem_st_x16(tmem_a + lane_base + s * kACols + khalf * 16, a);
                    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(afull_bar(s));
                }
            }
        }
        __syncwarp();
    } else {
        // ---------------- epilogue (warps 10..13) ----------------
        const int quarter = warp & 3;
        const int row_local = quarter * 32 + lane;
        const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
        const bool storer = warp == kFirstEpilogueWarp && lane == 0;
        uint16_t *staging = reinterpret_cast<uint16_t *>(smem + SmemLayout.staging);
        volatile uint32_t *epi_decision =
            reinterpret_cast<volatile uint32_t *>(smem + SmemLayout.epi_decision);
        volatile uint32_t *epi_last = reinterpret_cast<volatile uint32_t *>(smem + SmemLayout.epi_last);
        int tcount = 0;
        for (int item = blockIdx.x; item < items; item += gridDim.x, ++tcount) {
            const WorkItem wk = work_item(item, splits, tiles_n, KT);
            const int n0 = wk.n0, m0 = wk.m0;
            const int chunks = mma_n(M, m0) / 16;     // accumulator columns the MMAs wrote
            // One decision for the four epilogue warps (they meet at named
            // barriers below): the storer publishes the abort flag after every
            // warp has finished its bounded wait.
            __all_sync(0xFFFFFFFFu, gemm_wait(dfull_bar, tcount & 1, wait_limit, abort_flag));
            epilogue_bar_sync();
            if (storer) {
                // the previous tile's store must have finished reading the staging tile
                if (use_tma_store) tma_store_wait_read();
                *epi_decision = *abort_flag;
            }
            epilogue_bar_sync();
            if (*epi_decision) break;
            tc_fence_after();
            const int n = n0 + row_local;
            if (FIXED_STAGES == 0 && splits > 1) {
                // split-K: this split's fp32 partial goes to partials[split][m][n]
                float *part = partials + (int64_t)wk.split * M * N;
#pragma unroll 1
                for (int c = 0; c < chunks; ++c) {
                    uint32_t v[16];
                    tmem_ld_x16(tmem_acc + lane_base + c * 16, v);
                    if (n < N) {
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            const int m = m0 + c * 16 + j;
                            if (m < M) part[(int64_t)m * N + n] = __uint_as_float(v[j]);
                        }
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(dempty_bar);
                __threadfence();
                epilogue_bar_sync();
                if (storer) *epi_last = atomicAdd(&counters[wk.tile], 1u) == (uint32_t)(splits - 1);
                epilogue_bar_sync();
                if (*epi_last) {
                    // The last split of the tile adds the partials in split
                    // order.  With N % 4 == 0 thread t takes rows n0 + 4(t%32)
                    // .. +3 (float4) and tokens m0 + t/32, +4, ...; otherwise
                    // one row per thread.
                    __threadfence();
                    const int m_end = M < m0 + kTileM ? M : m0 + kTileM;
                    const int t = (int)threadIdx.x - 32 * kFirstEpilogueWarp;
                    if ((N & 3) == 0) {
                        const int nq = n0 + 4 * (t & 31);
                        if (nq < N) {
                            for (int mb = m0 + (t >> 5); mb < m_end; mb += 16) {
                                float4 acc[4];
#pragma unroll
                                for (int j = 0; j < 4; ++j) acc[j] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 2
                                for (int sp = 0; sp < splits; ++sp) {
                                    float4 v[4];
#pragma unroll
                                    for (int j = 0; j < 4; ++j) {
                                        const int m = mb + 4 * j;
                                        v[j] = m < m_end ? __ldcg(reinterpret_cast<const float4 *>(
                                                               &partials[((int64_t)sp * M + m) * N + nq]))
                                                         : make_float4(0.f, 0.f, 0.f, 0.f);
                                    }
#pragma unroll
                                    for (int j = 0; j < 4; ++j) {
                                        acc[j].x += v[j].x;
                                        acc[j].y += v[j].y;
                                        acc[j].z += v[j].z;
                                        acc[j].w += v[j].w;
                                    }
                                }
#pragma unroll
                                for (int j = 0; j < 4; ++j) {
                                    const int m = mb + 4 * j;
                                    if (m < m_end) {
                                        uint2 o;
                                        o.x = dev::f32_to_bf16_rne(acc[j].x) | (dev::f32_to_bf16_rne(acc[j].y) << 16);
                                        o.y = dev::f32_to_bf16_rne(acc[j].z) | (dev::f32_to_bf16_rne(acc[j].w) << 16);
                                        *reinterpret_cast<uint2 *>(&y[(int64_t)m * N + nq]) = o;
                                    }
                                }
                            }
                        }
                    } else if (n < N) {
                        for (int mb = m0; mb < m_end; mb += 8) {
                            float acc[8];
#pragma unroll
                            for (int j = 0; j < 8; ++j) acc[j] = 0.0f;
#pragma unroll 2
                            for (int sp = 0; sp < splits; ++sp) {
                                float v[8];
#pragma unroll
                                for (int j = 0; j < 8; ++j)
                                    v[j] = mb + j < m_end
                                               ? __ldcg(&partials[((int64_t)sp * M + mb + j) * N + n])
                                               : 0.0f;
#pragma unroll
                                for (int j = 0; j < 8; ++j) acc[j] += v[j];
                            }
#pragma unroll
                            for (int j = 0; j < 8; ++j)
                                if (mb + j < m_end)
                                    y[(int64_t)(mb + j) * N + n] = (uint16_t)dev::f32_to_bf16_rne(acc[j]);
                        }
                    }
                    if (storer) counters[wk.tile] = 0u;
                }
                continue;
            }
#pragma unroll 1
            for (int c = 0; c < chunks; ++c) {
                uint32_t v[16];
                tmem_ld_x16(tmem_acc + lane_base + c * 16, v);
                if (use_tma_store) {
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        staging[(c * 16 + j) * kTileN + row_local] =
                            (uint16_t)dev::f32_to_bf16_rne(__uint_as_float(v[j]));
                } else if (n < N) {
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const int m = m0 + c * 16 + j;
                        if (m < M)
                            y[(int64_t)m * N + n] =
                                (uint16_t)dev::f32_to_bf16_rne(__uint_as_float(v[j]));
                    }
                }
            }
            // accumulator read: the next tile's MMAs may start
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(dempty_bar);
            if (use_tma_store) {
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                epilogue_bar_sync();
                if (storer) tma_store_2d(&y_map, sbase + SmemLayout.staging, n0, m0);
            }
        }
        if (storer) tma_store_wait_all();
        __syncwarp();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                     "r"(kTmemCols / CTAS)
                     : "memory");
    }
}

}  // namespace

// Split-K: when the 128 x 256 output tiles are fewer than the SMs, each
// tile's K range is divided among up to kMaxSplits CTAs (at least 4 stages
// each); their fp32 partials meet in the workspace.
// Tokens per activation box: a whole tile, or all of M rounded up to 16.
int gemm_act_rows(int64_t M) { return M >= kTileM ? kTileM : (int)((M + 15) & ~int64_t(15)); }

// `sms`: the SMs the grid is sized for (fewer SMs give fewer or equal splits,
// so a workspace sized for kSmCount serves every device).
int gemm_splits(int64_t M, int64_t N, int64_t K, int sms) {
    const int64_t tiles = ceil_div(N, kTileN) * ceil_div(M, kTileM);
    const int64_t slots = (int64_t)sms * gemm_ctas_per_sm(gemm_act_rows(M));
    if (tiles >= slots) return 1;
    int64_t s = slots / tiles;
    if (s > kMaxSplits) s = kMaxSplits;
    if (s > K / kTileK / 4) s = K / kTileK / 4;
    return s < 1 ? 1 : (int)s;
}

// fp32 partials [splits][M][N], then one uint32 arrival counter per tile
size_t gemm_partial_bytes(int64_t M, int64_t N, int64_t K, int sms) {
    const int s = gemm_splits(M, N, K, sms);
    if (s == 1) return 0;
    return (((size_t)s * M * N * sizeof(float)) + 255) & ~(size_t)255;
}

size_t gemm_workspace_bytes_for(int64_t M, int64_t N, int64_t K, int sms) {
    if (gemm_splits(M, N, K, sms) == 1) return 0;
    const int64_t tiles = ceil_div(N, kTileN) * ceil_div(M, kTileM);
    return gemm_partial_bytes(M, N, K, sms) +
           (size_t)ceil_div(tiles, 64) * 64 * sizeof(uint32_t);
}

size_t gemm_workspace_bytes(int64_t M, int64_t N, int64_t K) {
    return gemm_workspace_bytes_for(M, N, K, kSmCount);
}

unsigned int *device_error_word() {
    static void *addr[kMaxDevices] = {};
    static DeviceOnce once;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return nullptr;
    }
    const cudaError_t e = once.run(dev, [dev] {
        return cudaGetSymbolAddress(&addr[dev], g_device_error_word);
    });
    return e == cudaSuccess ? static_cast<unsigned int *>(addr[dev]) : nullptr;
}

namespace {

template <int BITS>
qz_status launch_gemm(const void *a, const void *codes, const void *scales, const void *zeros,
                      int64_t M, int64_t N, int64_t K, int64_t group_size, void *y,
                      void *workspace, cudaStream_t st) {
    constexpr int kRowBytesPerK = BITS;   // code bytes of a row per 8 k
    const int act_rows = gemm_act_rows(M);
    const int ctas = gemm_ctas_per_sm(act_rows);
    const int sms = device_sm_count();
    const int splits = gemm_splits(M, N, K, sms);
    float *partials = nullptr;
    uint32_t *counters = nullptr;
    if (splits > 1) {
        partials = static_cast<float *>(workspace);
        counters = reinterpret_cast<uint32_t *>(static_cast<char *>(workspace) +
                                                gemm_partial_bytes(M, N, K, sms));
    }
    CUtensorMap act_map, pack_map, y_map;
    if (!make_map_2d(&act_map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a, (uint64_t)K, (uint64_t)M,
                     (uint64_t)K * 2, kTileK, act_rows, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map_2d(&pack_map, CU_TENSOR_MAP_DATA_TYPE_UINT8, codes,
                     (uint64_t)K * kRowBytesPerK / 8, (uint64_t)N,
                     (uint64_t)K * kRowBytesPerK / 8, kTileK * kRowBytesPerK / 8, kTileN,
                     CU_TENSOR_MAP_SWIZZLE_NONE))
        return QZ_ERR_CUDA;
    // bf16 output rows must be 16-byte multiples for a TMA store
    const int use_tma_store = (N % 8 == 0) ? 1 : 0;
    if (use_tma_store) {
        if (!make_map_2d(&y_map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, y, (uint64_t)N, (uint64_t)M,
                         (uint64_t)N * 2, kTileN, act_rows, CU_TENSOR_MAP_SWIZZLE_NONE))
            return QZ_ERR_CUDA;
    } else {
        y_map = act_map;   // unused
    }
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return QZ_ERR_CUDA;
    }
    static DeviceOnce attr_once;
    const cudaError_t attr_err = attr_once.run(dev, [] {
        cudaError_t e = cudaFuncSetAttribute(wa16_gemm_tcgen05<BITS, kFullTileStages, 1>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             kSmemLimit);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(wa16_gemm_tcgen05<BITS, 0, 1>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(wa16_gemm_tcgen05<BITS, 0, 2>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit);
        // two CTAs per SM need the whole unified memory as shared memory
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(wa16_gemm_tcgen05<BITS, 0, 2>,
                                     cudaFuncAttributePreferredSharedMemoryCarveout, 100);
        return e;
    });
    if (attr_err != cudaSuccess) return QZ_ERR_CUDA;
    const int stages = gemm_stages(BITS, act_rows, ctas);
    const uint32_t smem_bytes = gemm_layout(BITS, act_rows, stages).end + 1024;
    const int64_t items = ceil_div(N, kTileN) * ceil_div(M, kTileM) * splits;
    const int grid = (int)std::min<int64_t>(items, (int64_t)sms * ctas);
    auto kernel = act_rows == kTileM && splits == 1 ? wa16_gemm_tcgen05<BITS, kFullTileStages, 1>
                  : ctas == 2                      ? wa16_gemm_tcgen05<BITS, 0, 2>
                                                   : wa16_gemm_tcgen05<BITS, 0, 1>;
    kernel<<<grid, kThreads, smem_bytes, st>>>(
        act_map, pack_map, y_map, static_cast<const uint16_t *>(scales),
        static_cast<const uint8_t *>(zeros), (int)M, (int)N, (int)K, (int)group_size,
        static_cast<uint16_t *>(y), use_tma_store, act_rows, stages, splits, partials, counters,
        device_wait_limit());
    return launch_status();
}

}  // namespace

qz_status launch_w4a16_gemm(const void *a, const void *codes, const void *scales,
                            const void *zeros, int64_t M, int64_t N, int64_t K,
                            int64_t group_size, void *y, void *workspace, cudaStream_t st) {
    return launch_gemm<4>(a, codes, scales, zeros, M, N, K, group_size, y, workspace, st);
}

qz_status launch_w8a16_gemm(const void *a, const void *codes, const void *scales, int64_t M,
                            int64_t N, int64_t K, void *y, void *workspace, cudaStream_t st) {
    return launch_gemm<8>(a, codes, scales, nullptr, M, N, K, K, y, workspace, st);
}

}  // namespace qz

extern "C" QZ_API qz_status qz_device_status(void) {
    if (cudaDeviceSynchronize() != cudaSuccess) return QZ_ERR_CUDA;
    unsigned int word = 0;
    if (cudaMemcpyFromSymbol(&word, qz::g_device_error_word, sizeof word) != cudaSuccess)
        return QZ_ERR_CUDA;
    if (word == 0) return QZ_OK;
    const unsigned int zero = 0;
    if (cudaMemcpyToSymbol(qz::g_device_error_word, &zero, sizeof zero) != cudaSuccess)
        return QZ_ERR_CUDA;
    return QZ_ERR_DEVICE_TIMEOUT;
}
