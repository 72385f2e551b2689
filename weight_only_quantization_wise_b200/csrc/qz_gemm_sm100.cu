// qz_gemm_sm100.cu -- W4A16 prefill GEMM on the sm_100a (tcgen05) tensor cores,
// and the device error word used by bounded device-side waits.
//
// Quantization concepts guide, "Quantize weights or activations": weight-only
// methods dequantize the weights to the compute dtype before each matmul;
// prefill and large batches are compute-bound, so this path must keep the
// tensor cores busy.  The GPTQ explainer: the dequantization happens inside
// the matmul kernel, with no separate conversion pass.
//
// y (M x N) = a (M x K) * w_hat^T with w_hat = bf16_rne(S * (q - Z)).
//
// Persistent kernel: each CTA loops over tiles of 128 weight rows x 256
// tokens (tile t = blockIdx.x + i * gridDim.x).  The roles:
//   warp 0       TMA producer: per 64-wide K step, the activation tile
//                (256 tokens x 64 bf16, 128-byte swizzle) and the packed codes
//                (128 rows x 32 bytes) into a STAGES-deep shared-memory ring.
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

constexpr int kStages = 4;
constexpr int kTileN = 128;               // weight rows per tile (MMA M)
constexpr int kTileM = 256;               // tokens per tile (MMA N)
constexpr int kTileK = 64;                // K per stage
constexpr int kActStageBytes = kTileM * kTileK * 2;      // 32 KB
constexpr int kPackStageBytes = kTileN * kTileK / 2;     // 4 KB
constexpr int kStagingBytes = kTileM * kTileN * 2;       // 64 KB bf16 output tile
constexpr int kAccCols = kTileM;                         // fp32 accumulator columns
constexpr int kACols = kTileK / 2;                       // A columns per stage (bf16 pairs)
constexpr int kTmemCols = 512;
constexpr int kDequantWarps = 8;
constexpr int kMetaFifo = 2;              // groups of scales/zeros loaded ahead
constexpr int kEpilogueWarps = 4;
constexpr int kFirstEpilogueWarp = 2 + kDequantWarps;
constexpr int kThreads = 32 * (2 + kDequantWarps + kEpilogueWarps);
constexpr int kSmemBytes =
    kStages * (kActStageBytes + kPackStageBytes) + kStagingBytes + 1024 + 256;

// instruction descriptor: MMA M = 128 weight rows, N = 256 tokens
constexpr uint32_t kIdesc = idesc_bf16(kTileN, kTileM);

struct SmemLayout {
    // offsets from the 1024-aligned base
    static constexpr uint32_t act = 0;
    static constexpr uint32_t pack = act + kStages * kActStageBytes;
    static constexpr uint32_t staging = pack + kStages * kPackStageBytes;
    static constexpr uint32_t bars = staging + kStagingBytes;
    // barriers: full[S], empty[S], afull[S], dfull, dempty, drain
    static constexpr uint32_t full = bars;
    static constexpr uint32_t empty = full + 8 * kStages;
    static constexpr uint32_t afull = empty + 8 * kStages;
    static constexpr uint32_t dfull = afull + 8 * kStages;
    static constexpr uint32_t dempty = dfull + 8;
    static constexpr uint32_t drain = dempty + 8;
    static constexpr uint32_t tmem_slot = drain + 8;
    static constexpr uint32_t abort_flag = tmem_slot + 4;
    static constexpr uint32_t epi_decision = abort_flag + 4;
    static constexpr uint32_t end = epi_decision + 4;
};
static_assert(SmemLayout::end + 1024 <= kSmemBytes, "shared memory layout");
static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");

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

__global__ void __launch_bounds__(kThreads, 1)
w4a16_gemm_tcgen05(const __grid_constant__ CUtensorMap act_map,
                   const __grid_constant__ CUtensorMap pack_map,
                   const __grid_constant__ CUtensorMap y_map,
                   const uint16_t *__restrict__ scales, const uint8_t *__restrict__ zeros,
                   int M, int N, int K, int group_size, uint16_t *__restrict__ y,
                   int use_tma_store, uint64_t wait_limit) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    volatile uint32_t *abort_flag = reinterpret_cast<volatile uint32_t *>(smem + SmemLayout::abort_flag);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + SmemLayout::tmem_slot);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int KT = K / kTileK;
    const int tiles_n = (N + kTileN - 1) / kTileN;
    const int tiles = tiles_n * ((M + kTileM - 1) / kTileM);

    auto full_bar = [&](int s) { return sbase + SmemLayout::full + 8 * s; };
    auto empty_bar = [&](int s) { return sbase + SmemLayout::empty + 8 * s; };
    auto afull_bar = [&](int s) { return sbase + SmemLayout::afull + 8 * s; };
    const uint32_t dfull_bar = sbase + SmemLayout::dfull;
    const uint32_t dempty_bar = sbase + SmemLayout::dempty;
    const uint32_t drain_bar = sbase + SmemLayout::drain;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
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
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const uint32_t tmem_acc = tmem_base;                // columns [0, 256)
    const uint32_t tmem_a = tmem_base + kAccCols;       // A slots: kStages x 32 columns

    if (warp == 0) {
        // ---------------- TMA producer ----------------
        if (lane == 0) {
            int issued_round[kStages];
            for (int s = 0; s < kStages; ++s) issued_round[s] = -1;
            int it = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x) {
                const int n0 = (tile % tiles_n) * kTileN, m0 = (tile / tiles_n) * kTileM;
                for (int kt = 0; kt < KT; ++kt, ++it) {
                    const int s = it % kStages, r = it / kStages;
                    if (r > 0 && !gemm_wait(empty_bar(s), (r - 1) & 1, wait_limit, abort_flag)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(full_bar(s), kActStageBytes + kPackStageBytes);
                    tma_load_2d(sbase + SmemLayout::act + s * kActStageBytes, &act_map,
                                kt * kTileK, m0, full_bar(s));
                    tma_load_2d(sbase + SmemLayout::pack + s * kPackStageBytes, &pack_map,
                                kt * (kTileK / 2), n0, full_bar(s));
                    issued_round[s] = r;
                }
            }
            // every issued copy must have landed before the CTA may exit
            for (int s = 0; s < kStages; ++s)
                if (issued_round[s] >= 0) gemm_drain(full_bar(s), issued_round[s] & 1);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            bool ok = true;
            int it = 0, tcount = 0;
            for (int tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x, ++tcount) {
                if (tcount > 0 && !gemm_wait(dempty_bar, (tcount - 1) & 1, wait_limit, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                for (int kt = 0; kt < KT; ++kt, ++it) {
                    const int s = it % kStages, r = it / kStages;
                    ok = gemm_wait(full_bar(s), r & 1, wait_limit, abort_flag) &&
                         gemm_wait(afull_bar(s), r & 1, wait_limit, abort_flag);
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t act_addr = sbase + SmemLayout::act + s * kActStageBytes;
#pragma unroll
                    for (int j = 0; j < kTileK / 16; ++j)
                        mma_ts(tmem_acc, tmem_a + s * kACols + j * 8,
                               smem_desc_sw128(act_addr + j * 32), kIdesc, (kt > 0 || j > 0) ? 1u : 0u);
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
        const int gpr = K / group_size;
        const int spg = group_size / kTileK;          // stages per group
        int it = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x) {
            const int n = (tile % tiles_n) * kTileN + row_local;
            const bool valid = n < N;
            const uint16_t *srow = scales + (int64_t)(valid ? n : 0) * gpr;
            const uint8_t *zrow = zeros + (int64_t)(valid ? n : 0) * gpr;
            // Scales and zeros of the next kMetaFifo groups wait in a register
            // FIFO (a group spans spg stages), so their loads are issued up to
            // kMetaFifo groups before use and no per-stage index arithmetic is
            // needed.
            uint32_t sq[kMetaFifo], zq[kMetaFifo];
#pragma unroll
            for (int q = 0; q < kMetaFifo; ++q) {
                sq[q] = (valid && q < gpr) ? __ldg(&srow[q]) : 0u;
                zq[q] = (valid && q < gpr) ? __ldg(&zrow[q]) : 0u;
            }
            int stage_in_group = 0, next_group = kMetaFifo;
            for (int kt = 0; kt < KT; ++kt, ++it) {
                const int s = it % kStages, r = it / kStages;
                const uint32_t sb = sq[0], zb = zq[0];
                if (++stage_in_group == spg) {               // the next stage starts a new group
                    stage_in_group = 0;
#pragma unroll
                    for (int q = 0; q < kMetaFifo - 1; ++q) {
                        sq[q] = sq[q + 1];
                        zq[q] = zq[q + 1];
                    }
                    sq[kMetaFifo - 1] = (valid && next_group < gpr) ? __ldg(&srow[next_group]) : 0u;
                    zq[kMetaFifo - 1] = (valid && next_group < gpr) ? __ldg(&zrow[next_group]) : 0u;
                    ++next_group;
                }
                // warp-uniform: the tcgen05.st below needs every lane
                if (!__all_sync(0xFFFFFFFFu, gemm_wait(full_bar(s), r & 1, wait_limit, abort_flag))) {
                    ok = false;
                    break;
                }
                const uint4 p = *reinterpret_cast<const uint4 *>(
                    smem + SmemLayout::pack + s * kPackStageBytes + row_local * (kTileK / 2) +
                    khalf * 16);
                __syncwarp();
                if (lane == 0) mbar_arrive(empty_bar(s));     // packed stage consumed
                const uint32_t s2 = sb * 0x00010001u;
                const uint32_t z2 = (0x4300u + zb) * 0x00010001u;
                const uint32_t words[4] = {p.x, p.y, p.z, p.w};
                uint32_t a[16];
#pragma unroll
                for (int wi = 0; wi < 4; ++wi) {
                    const uint32_t w = words[wi], w4 = w >> 4;
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        a[wi * 4 + i] = valid ? dequant_pair_nat(w, w4, i, s2, z2) : 0u;
                }
                tmem_st_x16(tmem_a + lane_base + s * kACols + khalf * 16, a);
                asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(afull_bar(s));
            }
        }
        __syncwarp();
    } else {
        // ---------------- epilogue (warps 10..13) ----------------
        const int quarter = warp & 3;
        const int row_local = quarter * 32 + lane;
        const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
        const bool storer = warp == kFirstEpilogueWarp && lane == 0;
        uint16_t *staging = reinterpret_cast<uint16_t *>(smem + SmemLayout::staging);
        volatile uint32_t *epi_decision =
            reinterpret_cast<volatile uint32_t *>(smem + SmemLayout::epi_decision);
        int tcount = 0;
        for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x, ++tcount) {
            const int n0 = (tile % tiles_n) * kTileN, m0 = (tile / tiles_n) * kTileM;
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
#pragma unroll 1
            for (int c = 0; c < kTileM / 16; ++c) {
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
                if (storer) tma_store_2d(&y_map, sbase + SmemLayout::staging, n0, m0);
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
                     "r"(kTmemCols)
                     : "memory");
    }
}

}  // namespace

size_t gemm_workspace_bytes(int64_t, int64_t, int64_t) { return 0; }

unsigned int *device_error_word() {
    static unsigned int *addr[64] = {};
    static std::once_flag once[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::call_once(once[dev], [dev] {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_device_error_word) == cudaSuccess)
            addr[dev] = static_cast<unsigned int *>(p);
    });
    return addr[dev];
}

qz_status launch_w4a16_gemm(const void *a, const void *codes, const void *scales,
                            const void *zeros, int64_t M, int64_t N, int64_t K,
                            int64_t group_size, void *y, void *, cudaStream_t st) {
    CUtensorMap act_map, pack_map, y_map;
    if (!make_map_2d(&act_map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a, (uint64_t)K, (uint64_t)M,
                     (uint64_t)K * 2, kTileK, kTileM, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map_2d(&pack_map, CU_TENSOR_MAP_DATA_TYPE_UINT8, codes, (uint64_t)K / 2,
                     (uint64_t)N, (uint64_t)K / 2, kTileK / 2, kTileN,
                     CU_TENSOR_MAP_SWIZZLE_NONE))
        return QZ_ERR_CUDA;
    // bf16 output rows must be 16-byte multiples for a TMA store
    const int use_tma_store = (N % 8 == 0) ? 1 : 0;
    if (use_tma_store) {
        if (!make_map_2d(&y_map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, y, (uint64_t)N, (uint64_t)M,
                         (uint64_t)N * 2, kTileN, kTileM, CU_TENSOR_MAP_SWIZZLE_NONE))
            return QZ_ERR_CUDA;
    } else {
        y_map = act_map;   // unused
    }
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return QZ_ERR_CUDA;
    static std::once_flag attr_once[64];
    if (dev >= 0 && dev < 64)
        std::call_once(attr_once[dev], [] {
            cudaFuncSetAttribute(w4a16_gemm_tcgen05, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kSmemBytes);
        });
    const int64_t tiles = ceil_div(N, kTileN) * ceil_div(M, kTileM);
    const int grid = (int)std::min<int64_t>(tiles, kSmCount);
    w4a16_gemm_tcgen05<<<grid, kThreads, kSmemBytes, st>>>(
        act_map, pack_map, y_map, static_cast<const uint16_t *>(scales),
        static_cast<const uint8_t *>(zeros), (int)M, (int)N, (int)K, (int)group_size,
        static_cast<uint16_t *>(y), use_tma_store, device_wait_limit());
    return launch_status();
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
