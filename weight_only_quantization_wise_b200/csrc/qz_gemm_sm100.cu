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
// Persistent kernel: each CTA loops over work items, each a K range of one
// tile of 128 weight rows x 256 tokens: whole tiles for the full waves, and
// the K steps of the last, partial wave spread evenly over the CTAs, whose
// fp32 partials meet in the workspace (GemmSched).  The roles:
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

#include <algorithm>
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
    uint32_t act, pack, staging, full, empty, afull, dfull, dempty, drain, fixbar, tmem_slot,
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
    L.fixbar = L.drain + 8;
    L.tmem_slot = L.fixbar + 8;
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
static_assert(kTileK == 64, "the MMA issuer writes out the four 16-wide K steps of a stage");

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

__device__ __forceinline__ void bulk_load(uint32_t dst, const void *src, uint32_t bytes,
                                          uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
            "r"(dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}

__device__ __forceinline__ void epilogue_bar_sync() {
    asm volatile("bar.sync 1, %0;" ::"n"(32 * kEpilogueWarps) : "memory");
}

// int8 codes: bf16 pair (byte 2i, byte 2i+1) of word wx (the code word XOR
// 0x80808080): one packed subtraction gives the pair of q exactly
// (dev::i8_codes_bf16x2) and mul.rn.bf16x2 by (S, S) rounds S*q once, as
// qz_dequantize does.
__device__ __forceinline__ uint32_t dequant_pair_i8_nat(uint32_t wx, int i, uint32_t s2) {
    return dev::bf16x2_mul(dev::i8_codes_bf16x2(dev::prmt(wx, 0x4B000000u, (uint32_t)(2 * i) | 0x7540u),
                                                dev::prmt(wx, 0x4B000000u, (uint32_t)(2 * i + 1) | 0x7540u)),
                           s2);
}

// Work item: a K range [kt0, kt1) of one output tile (128 weight rows x up
// to 256 tokens).  nseg == 1: the whole tile, written directly.  nseg > 1:
// one of the nseg CTAs that share the tile; its fp32 partial goes to
// workspace slot `slot`, the tile's slots are slot0 .. slot0 + nseg - 1 in K
// order, and the last of them to arrive at counter `ctr` adds them.
struct WorkItem {
    int n0, m0, kt0, kt1, nseg, slot, slot0, ctr;
};

// Schedule of one launch (host-made, passed by value).  Tiles [0, dp_tiles)
// are whole work items, tile c + i * grid on CTA c.  The K steps of tiles
// [dp_tiles, tiles) -- the last, partial wave, or all tiles when they are
// fewer than the CTAs -- are laid end to end, sk_steps = (tiles - dp_tiles)
// * KT of them, and CTA c < sk_ctas takes steps [b_c, b_{c+1}) with b_c =
// floor(c * sk_steps / sk_ctas) (at least kMinSegSteps each): every CTA then
// carries the same work, up to one step.  A CTA's range cut at tile
// boundaries gives its segments; segment (CTA c, tail tile t) takes slot
// c + t, which grows with the segment's first step, so the slots are unique,
// each tile's slots are consecutive, and all are below sk_ctas + tail tiles
// - 1.
// A CTA runs its whole tiles first and its segments last.  Every CTA ends
// its range at about the same time, so the segment that ends a range
// usually finds the tile's other segments done and adds them at once from
// its own accumulator, after its main loop, when the CTA's whole ring and
// staging memory are free to receive them; additions that overlapped other
// CTAs' main loops (loads competing with the dequantizing warps') slowed
// those to half speed.
struct GemmSched {
    int tiles_n;        // tiles along N
    int KT;             // 64-wide K steps per tile
    int tiles;
    int dp_tiles;
    int sk_ctas;
    int64_t sk_steps;
};

#ifndef QZ_SLOT_SKEW
#define QZ_SLOT_SKEW 1
#endif
#ifndef QZ_LAND_STAGE
#define QZ_LAND_STAGE 1
#endif
// Partial slots are act_rows x 128 fp32 each, placed 1 KB further apart than
// that, so that CTAs writing or reading the same offset of their slots at
// the same time do not all meet in the same memory channels.
constexpr int kSlotSkewFloats = QZ_SLOT_SKEW ? 256 : 0;
__host__ __device__ constexpr int64_t slot_stride(int act_rows) {
    return (int64_t)act_rows * kTileN + kSlotSkewFloats;
}
constexpr int kMaxSegsPerTile = 6;   // tail CTAs per tail tile, on average, at most
constexpr int kMinSegSteps = 4;      // K steps of a tail CTA's range, at least
// Sharing the last wave must save each CTA at least this many K steps: the
// partial writes, the additions and the slower segments cost 15-25 us, about
// 48 steps of a full tile (measured: 2048 x 8192 x 8192 gains 3%, 256 and 128
// tokens over 8192 x 8192 gain 8-9%; savings of 17-35 steps lost 3-20%).
constexpr int kMinGainSteps = 48;

// The tail CTA whose range holds step p.
__host__ __device__ __forceinline__ int sched_cta_of(const GemmSched &S, int64_t p) {
    return (int)(((p + 1) * S.sk_ctas - 1) / S.sk_steps);
}
__host__ __device__ __forceinline__ int64_t sched_bound(const GemmSched &S, int c) {
    return (int64_t)c * S.sk_steps / S.sk_ctas;
}
__host__ __device__ __forceinline__ int sched_segments(const GemmSched &S, int c) {
    if (c >= S.sk_ctas) return 0;
    const int64_t b0 = sched_bound(S, c), b1 = sched_bound(S, c + 1);
    return (int)((b1 - 1) / S.KT - b0 / S.KT + 1);
}
__host__ __device__ __forceinline__ int sched_count(const GemmSched &S, int c, int grid) {
    const int whole = c < S.dp_tiles ? (S.dp_tiles - 1 - c) / grid + 1 : 0;
    return whole + sched_segments(S, c);
}
__host__ __device__ __forceinline__ WorkItem sched_item(const GemmSched &S, int c, int grid, int i) {
    WorkItem w;
    const int whole = c < S.dp_tiles ? (S.dp_tiles - 1 - c) / grid + 1 : 0;
    int tile;
    if (i >= whole) {
        const int64_t b0 = sched_bound(S, c), b1 = sched_bound(S, c + 1);
        const int t = (int)(b0 / S.KT) + (i - whole);       // tail tile
        const int64_t t0 = (int64_t)t * S.KT;
        w.kt0 = (int)((b0 > t0 ? b0 : t0) - t0);
        w.kt1 = (int)((b1 < t0 + S.KT ? b1 : t0 + S.KT) - t0);
        const int cf = sched_cta_of(S, t0), cl = sched_cta_of(S, t0 + S.KT - 1);
        w.nseg = cl - cf + 1;
        w.slot = c + t;
        w.slot0 = cf + t;
        w.ctr = t;
        tile = S.dp_tiles + t;
    } else {
        tile = c + i * grid;
        w.kt0 = 0;
        w.kt1 = S.KT;
        w.nseg = 1;
        w.slot = w.slot0 = w.ctr = 0;
    }
    w.n0 = (tile % S.tiles_n) * kTileN;
    w.m0 = (tile / S.tiles_n) * kTileM;
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
                   int use_tma_store, int act_rows, int stages_rt, const GemmSched sched,
                   float *__restrict__ partials, uint32_t *__restrict__ counters,
                   uint64_t wait_limit) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const int stages = FIXED_STAGES > 0 ? FIXED_STAGES : stages_rt;
    const GemmLayout SmemLayout = kernel_layout<BITS, FIXED_STAGES>(act_rows, stages_rt);
    constexpr int kPackBytes = kPackStageBytes<BITS>;
    const uint32_t kActStageBytes = SmemLayout.act_stage;
    volatile uint32_t *abort_flag = reinterpret_cast<volatile uint32_t *>(smem + SmemLayout.abort_flag);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + SmemLayout.tmem_slot);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int items = sched_count(sched, blockIdx.x, gridDim.x);
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
        mbar_init(sbase + SmemLayout.fixbar, 1);
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
            for (int item = 0; item < items && ok; ++item) {
                const WorkItem wk = sched_item(sched, blockIdx.x, gridDim.x, item);
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
            for (int item = 0; item < items && ok; ++item, ++tcount) {
                const WorkItem wk = sched_item(sched, blockIdx.x, gridDim.x, item);
                const uint32_t idesc = idesc_bf16(kTileN, mma_n(M, wk.m0));
                if (tcount > 0 && !gemm_wait(dempty_bar, (tcount - 1) & 1, wait_limit, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                // This one thread's instruction stream is the pace of the
                // whole pipeline (its barriers are found ready): one probe of
                // both barriers before the bounded waits, one shared-memory
                // descriptor per stage advanced by 32 bytes (2 in its
                // 16-byte address field) per 16-wide K step.
                for (int kt = wk.kt0; kt < wk.kt1;
                     ++kt, s = (s + 1 == stages ? 0 : s + 1), r += (s == 0)) {
                    if (!(mbar_try_wait(full_bar(s), r & 1) && mbar_try_wait(afull_bar(s), r & 1))) {
                        ok = gemm_wait(full_bar(s), r & 1, wait_limit, abort_flag) &&
                             gemm_wait(afull_bar(s), r & 1, wait_limit, abort_flag);
                        if (!ok) break;
                    }
                    tc_fence_after();
                    const uint64_t bdesc = smem_desc_sw128(sbase + SmemLayout.act + s * kActStageBytes);
                    const uint32_t acol = tmem_a + s * kACols;
                    mma_ts(tmem_acc, acol, bdesc, idesc, kt > wk.kt0 ? 1u : 0u);
                    mma_ts(tmem_acc, acol + 8, bdesc + 2, idesc, 1u);
                    mma_ts(tmem_acc, acol + 16, bdesc + 4, idesc, 1u);
                    mma_ts(tmem_acc, acol + 24, bdesc + 6, idesc, 1u);
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
        for (int item = 0; item < items && ok; ++item) {
            const WorkItem wk = sched_item(sched, blockIdx.x, gridDim.x, item);
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
                    // The codes were consumed by the conversion above, so
                    // their loads have returned; the stage's refill also
                    // waits for this stage's MMA, which follows afull, so
                    // releasing it here costs nothing.
                    if (lane == 0) {
                        mbar_arrive(empty_bar(s));
                        mbar_arrive(afull_bar(s));
                    }
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
                    if (lane == 0) {                  // codes consumed; A slot written
                        mbar_arrive(empty_bar(s));
                        mbar_arrive(afull_bar(s));
                    }
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
        uint32_t fix_phase = 0;      // parity of the addition barrier's next phase
        for (int item = 0; item < items; ++item, ++tcount) {
            const WorkItem wk = sched_item(sched, blockIdx.x, gridDim.x, item);
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
            if (wk.nseg > 1) {
                // A shared tile.  Its partials live in slots laid out [token -
                // m0][row - n0] (act_rows x 128 fp32); the last of the nseg
                // segments to arrive adds them in slot (K) order.
                // (paired CTAs, with short token tiles and few registers, add
                // from memory)
                const bool final_item = CTAS == 1 && item + 1 == items;
                bool own_tmem = false;        // the sum takes this segment from tensor memory
                if (final_item) {
                    // if every other segment has arrived, add straight from
                    // the accumulator without writing this one out
                    if (storer)
                        *epi_last = *reinterpret_cast<volatile uint32_t *>(&counters[wk.ctr]) ==
                                    (uint32_t)(wk.nseg - 1);
                    epilogue_bar_sync();
                    own_tmem = *epi_last;
                }
                if (!own_tmem) {
                    float *part = partials + wk.slot * slot_stride(act_rows);
#pragma unroll 1
                    for (int c = 0; c < chunks; ++c) {
                        uint32_t v[16];
                        tmem_ld_x16(tmem_acc + lane_base + c * 16, v);
#pragma unroll
                        for (int j = 0; j < 16; ++j)
                            __stcg(&part[(c * 16 + j) * kTileN + row_local], __uint_as_float(v[j]));
                    }
                    __threadfence();
                    epilogue_bar_sync();
                    if (storer)
                        *epi_last = atomicAdd(&counters[wk.ctr], 1u) == (uint32_t)(wk.nseg - 1);
                    epilogue_bar_sync();
                    const bool last = *epi_last;
                    own_tmem = last && final_item;
                    if (!own_tmem) {
                        // the accumulator is free for the next item's MMAs
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(dempty_bar);
                    }
                    if (!last) continue;
                }
                __threadfence();
                const int mt = (M < m0 + kTileM ? M : m0 + kTileM) - m0;
                const int nread = wk.nseg - (own_tmem ? 1 : 0);
                // tokens per round when the other slots land in the ring and
                // staging memory (free: this CTA's main loop is over)
                const bool stage_y = QZ_LAND_STAGE && use_tma_store;
                const uint32_t land_bytes = stage_y ? SmemLayout.staging : SmemLayout.full;
                const int tr = own_tmem ? (int)(land_bytes / ((uint32_t)nread * kTileN * 4)) & ~15 : 0;
                if (CTAS == 1 && own_tmem && tr >= 16) {
                    const int own_sg = wk.slot - wk.slot0;
                    const float *land = reinterpret_cast<const float *>(smem);
                    const uint32_t bar = sbase + SmemLayout.fixbar;
                    const int toks = chunks * 16;
                    for (int r0 = 0; r0 < toks; r0 += tr) {
                        const int rt = toks - r0 < tr ? toks - r0 : tr;
                        if (storer) {
                            // the slots were written through the generic proxy;
                            // the landing zone was last used by it as well
                            asm volatile("fence.proxy.async;" ::: "memory");
                            mbar_arrive_expect_tx(bar, (uint32_t)(nread * rt * kTileN * 4));
                            for (int sg = 0, k = 0; sg < wk.nseg; ++sg) {
                                if (sg == own_sg) continue;
                                bulk_load(sbase + (uint32_t)(k++ * tr * kTileN * 4),
                                          partials + (wk.slot0 + sg) * slot_stride(act_rows) + r0 * kTileN,
                                          (uint32_t)(rt * kTileN * 4), bar);
                            }
                        }
                        gemm_wait(bar, fix_phase & 1u, wait_limit, abort_flag);
                        fix_phase ^= 1u;
#pragma unroll 1
                        for (int c = r0 / 16; c < (r0 + rt) / 16; ++c) {
                            uint32_t own[16];
                            tmem_ld_x16(tmem_acc + lane_base + c * 16, own);
                            // 16 tokens of this thread's row, the slots added in
                            // order, each slot's 16 values loaded together
                            const float *lc = land + (c * 16 - r0) * kTileN + row_local;
                            float acc[16];
#pragma unroll 1
                            for (int sg = 0, k = 0; sg < wk.nseg; ++sg) {
                                float v[16];
                                if (sg == own_sg) {
#pragma unroll
                                    for (int j = 0; j < 16; ++j) v[j] = __uint_as_float(own[j]);
                                } else {
                                    const float *lk = lc + k++ * tr * kTileN;
#pragma unroll
                                    for (int j = 0; j < 16; ++j) v[j] = lk[j * kTileN];
                                }
#pragma unroll
                                for (int j = 0; j < 16; ++j) acc[j] = sg == 0 ? v[j] : acc[j] + v[j];
                            }
#pragma unroll
                            for (int j = 0; j < 16; ++j) {
                                if (stage_y)
                                    staging[(c * 16 + j) * kTileN + row_local] =
                                        (uint16_t)dev::f32_to_bf16_rne(acc[j]);
                                else if (n < N && c * 16 + j < mt)
                                    y[(int64_t)(m0 + c * 16 + j) * N + n] =
                                        (uint16_t)dev::f32_to_bf16_rne(acc[j]);
                            }
                        }
                        // every thread is done with this round's landing zone
                        epilogue_bar_sync();
                    }
                    // after an abort the copies may still be on their way
                    if (storer && *abort_flag) gemm_drain(bar, (fix_phase & 1u) ^ 1u);
                    if (stage_y) {
                        // one store of the whole tile, as for an unshared one
                        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                        epilogue_bar_sync();
                        if (storer) tma_store_2d(&y_map, sbase + SmemLayout.staging, n0, m0);
                    }
                } else {
                    // From memory (the rare shared tile whose last segment is
                    // not this CTA's last item, or slots too large to land):
                    // thread t adds rows n0 + 4(t%32) .. +3 (float4) of tokens
                    // m0 + t/32, +4, +8, ..., this segment's slot included.
                    if (own_tmem) {
                        // this segment's slot was written unless the check found
                        // every other segment done: write it now
                        float *part = partials + wk.slot * slot_stride(act_rows);
#pragma unroll 1
                        for (int c = 0; c < chunks; ++c) {
                            uint32_t v[16];
                            tmem_ld_x16(tmem_acc + lane_base + c * 16, v);
#pragma unroll
                            for (int j = 0; j < 16; ++j)
                                __stcg(&part[(c * 16 + j) * kTileN + row_local], __uint_as_float(v[j]));
                        }
                        __threadfence();
                        epilogue_bar_sync();
                    }
                    const int t = (int)threadIdx.x - 32 * kFirstEpilogueWarp;
                    const int nl = 4 * (t & 31), nq = n0 + nl;
                    const float *base = partials + wk.slot0 * slot_stride(act_rows) + nl;
                    const int64_t slot_floats = slot_stride(act_rows);
                    for (int mb = t >> 5; mb < mt; mb += 16) {
                        float4 acc[4];
#pragma unroll
                        for (int j = 0; j < 4; ++j) acc[j] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 2
                        for (int sg = 0; sg < wk.nseg; ++sg) {
                            float4 v[4];
#pragma unroll
                            for (int j = 0; j < 4; ++j)
                                v[j] = mb + 4 * j < mt
                                           ? __ldcg(reinterpret_cast<const float4 *>(
                                                 base + sg * slot_floats + (mb + 4 * j) * kTileN))
                                           : make_float4(0.f, 0.f, 0.f, 0.f);
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
                            const int m = m0 + mb + 4 * j;
                            if (mb + 4 * j >= mt) continue;
                            uint16_t *yr = y + (int64_t)m * N;
                            if ((N & 3) == 0) {
                                if (nq < N) {
                                    uint2 o;
                                    o.x = dev::f32_to_bf16_rne(acc[j].x) | (dev::f32_to_bf16_rne(acc[j].y) << 16);
                                    o.y = dev::f32_to_bf16_rne(acc[j].z) | (dev::f32_to_bf16_rne(acc[j].w) << 16);
                                    *reinterpret_cast<uint2 *>(yr + nq) = o;
                                }
                            } else {
                                const float e[4] = {acc[j].x, acc[j].y, acc[j].z, acc[j].w};
#pragma unroll
                                for (int q = 0; q < 4; ++q)
                                    if (nq + q < N) yr[nq + q] = (uint16_t)dev::f32_to_bf16_rne(e[q]);
                            }
                        }
                    }
                }
                if (own_tmem) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(dempty_bar);
                }
                if (storer) counters[wk.ctr] = 0u;
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

// Tokens per activation box: a whole tile, or all of M rounded up to 16.
int gemm_act_rows(int64_t M) { return M >= kTileM ? kTileM : (int)((M + 15) & ~int64_t(15)); }

namespace {

// The schedule for a grid of `sms` SMs (see GemmSched).  The tiles of the
// last partial wave (all tiles, when they are fewer than the CTAs) share
// their K steps evenly over up to every CTA, at least kMinSegSteps steps
// each and at most kMaxSegsPerTile CTAs per tile on average, when that
// shortens each CTA's work by at least kMinGainSteps K steps ((grid - tail
// tiles) * KT / grid); otherwise every tile is a whole work item.
GemmSched gemm_schedule(int64_t M, int64_t N, int64_t K, int sms) {
    GemmSched S{};
    S.tiles_n = (int)ceil_div(N, kTileN);
    S.KT = (int)(K / kTileK);
    S.tiles = S.tiles_n * (int)ceil_div(M, kTileM);
    const int grid = sms * gemm_ctas_per_sm(gemm_act_rows(M));
    const int tail = S.tiles >= grid ? S.tiles % grid : S.tiles;
    if ((S.tiles >= grid && tail == 0) ||
        (int64_t)(grid - tail) * S.KT < (int64_t)kMinGainSteps * grid) {
        S.dp_tiles = S.tiles;
        return S;
    }
    S.dp_tiles = S.tiles - tail;
    S.sk_steps = (int64_t)tail * S.KT;
    int64_t p = std::min<int64_t>({(int64_t)grid, (int64_t)kMaxSegsPerTile * tail,
                                   S.sk_steps / kMinSegSteps});
    S.sk_ctas = (int)std::max<int64_t>(p, 1);
    return S;
}

// CTAs to launch: every slot when the tiles fill a wave; otherwise one per
// tile, or one per tail range when the tiles' K steps are shared.
int gemm_grid(const GemmSched &S, int sms, int ctas) {
    const int grid = sms * ctas;
    if (S.tiles >= grid) return grid;
    return S.sk_ctas > 0 ? S.sk_ctas : S.tiles;
}

// Workspace of a schedule: fp32 partial slots (sk_ctas + tail tiles - 1 of
// act_rows x 128), then one uint32 arrival counter per tail tile.
size_t sched_partial_bytes(const GemmSched &S, int64_t M) {
    const int64_t slots = S.sk_ctas + (S.tiles - S.dp_tiles) - 1;
    return ((size_t)slots * slot_stride(gemm_act_rows(M)) * sizeof(float) + 255) & ~(size_t)255;
}

}  // namespace

size_t gemm_workspace_bytes_for(int64_t M, int64_t N, int64_t K, int sms) {
    const GemmSched S = gemm_schedule(M, N, K, sms);
    if (S.sk_ctas == 0) return 0;
    return sched_partial_bytes(S, M) +
           (size_t)ceil_div(S.tiles - S.dp_tiles, 64) * 64 * sizeof(uint32_t);
}

// The largest workspace over every SM count up to kSmCount (the schedule
// depends on the grid in no monotone way).
size_t gemm_workspace_bytes(int64_t M, int64_t N, int64_t K) {
    size_t most = 0;
    for (int sms = 1; sms <= kSmCount; ++sms)
        most = std::max(most, gemm_workspace_bytes_for(M, N, K, sms));
    return most;
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
    const GemmSched sched = gemm_schedule(M, N, K, sms);
    float *partials = nullptr;
    uint32_t *counters = nullptr;
    if (sched.sk_ctas > 0) {
        partials = static_cast<float *>(workspace);
        counters = reinterpret_cast<uint32_t *>(static_cast<char *>(workspace) +
                                                sched_partial_bytes(sched, M));
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
    const int grid = gemm_grid(sched, sms, ctas);
    auto kernel = act_rows == kTileM ? wa16_gemm_tcgen05<BITS, kFullTileStages, 1>
                  : ctas == 2                      ? wa16_gemm_tcgen05<BITS, 0, 2>
                                                   : wa16_gemm_tcgen05<BITS, 0, 1>;
    kernel<<<grid, kThreads, smem_bytes, st>>>(
        act_map, pack_map, y_map, static_cast<const uint16_t *>(scales),
        static_cast<const uint8_t *>(zeros), (int)M, (int)N, (int)K, (int)group_size,
        static_cast<uint16_t *>(y), use_tma_store, act_rows, stages, sched, partials, counters,
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
