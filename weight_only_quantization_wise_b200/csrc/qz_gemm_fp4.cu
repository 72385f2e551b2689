// qz_gemm_fp4.cu -- W4A4 prefill GEMM: FP4 (E2M1) weights and activations
// with block scales, on the sm_100a block-scaled tensor-core MMA.
//
// Quantization concepts guide, "Quantize weights or activations": for
// compute-bound prefill, quantizing the activations as well lets the matmul
// itself run on low-precision tensor cores (NVFP4 W4A4), while decode keeps
// 16-bit activations (W4A16).  Section "FP4 with block scales": every block
// of 16 (NVFP4, E4M3 scale, plus one fp32 scale per tensor) or 32 (MXFP4,
// power-of-two E8M0 scale) values carries its own scale.
//
// y (M x N) = a_hat (M x K) * w_hat^T, with a_hat the activations quantized
// on the fly exactly as qz_fp4_quantize does and w_hat the FP4 weights; the
// tensor core applies the block scales inside the MMA, the epilogue applies
// the two NVFP4 tensor scales and rounds to bf16.
//
// Persistent kernel, one CTA per SM, tiles of 128 tokens x 256 weight rows
// (tile t = blockIdx.x + i * gridDim.x, token blocks fastest so that the CTAs
// running together share weight tiles in L2).  The roles:
//   warp 0      TMA producer: per 256-wide K stage, the activation codes (128
//               tokens x 128 bytes) and the weight codes (256 rows x 128
//               bytes), both with the 128-byte swizzle, and the stage's block
//               scales of both operands (bulk copies of 512-byte scale atoms)
//               into a 4-deep ring.
//   warp 1      allocates tensor memory; one lane copies each stage's scales
//               into tensor memory (tcgen05.cp) and issues the block-scaled
//               MMAs: M = 128 tokens, N = 256 weight rows, K = 64 per MMA,
//               fp32 accumulators in tensor memory columns 0..255.
//   warps 2..5  epilogue: tcgen05.ld of a token row's 256 accumulators,
//               times the tensor scales, bf16 rounding, 16-byte stores.
//
// Scale layout read by the MMA (the "MMA scale layout" of include/qz.h):
// for every 128 rows and 4 consecutive scales of a row ("atom", 512 bytes),
// scale j of row r sits at byte (r % 32) * 16 + ((r % 128) / 32) * 4 + j % 4;
// atom (r / 128, j / 4) starts at ((r / 128) * (scales per row / 4) + j / 4)
// * 512.  tcgen05.cp (32x128b, replicated to the four lane quarters) moves
// one atom into four tensor-memory columns: the layout the MMA reads.
//
// Every mbarrier wait is bounded; on expiry the CTA records the fault in the
// device error word and an abort flag, drains what it issued, frees tensor
// memory and exits.
#include <cuda.h>
#include <cuda_runtime.h>

#include "qz_sm100.cuh"

namespace qz {
namespace {

using namespace sm100;

constexpr int kTok = 128;              // tokens per tile (MMA M)
constexpr int kRows = 256;             // weight rows per tile (MMA N)
constexpr int kStageK = 256;           // K per stage: one 128-byte swizzle row of codes
constexpr int kRowBytes = kStageK / 2; // code bytes of one row per stage
constexpr int kMmaK = 64;              // K per MMA
constexpr int kSteps = kStageK / kMmaK;
constexpr int kStages = 4;
constexpr int kAtomBytes = 512;        // 128 rows x 4 scales
constexpr int kEpilogueWarps = 4;
constexpr int kThreads = 32 * (2 + kEpilogueWarps);
constexpr int kTmemCols = 512;
constexpr int kAccCols = kRows;        // fp32 accumulators: one column per weight row
constexpr int kSmemLimit = 227 * 1024;

template <int KIND>
struct Fp4Cfg {
    static constexpr int kBlock = KIND == 0 ? 32 : 16;
    static constexpr int kAtoms = kStageK / kBlock / 4;      // scale atoms per row block and stage
    static constexpr int kStepsPerAtom = kSteps / kAtoms;    // MMAs served by one atom
    static constexpr uint32_t kSfaBytes = kAtoms * kAtomBytes;
    static constexpr uint32_t kSfbBytes = 2 * kAtoms * kAtomBytes;   // two 128-row blocks
    static constexpr uint32_t kActBytes = kTok * kRowBytes;          // 16 KB
    static constexpr uint32_t kWgtBytes = kRows * kRowBytes;         // 32 KB
    // byte offsets from the 1024-aligned base
    static constexpr uint32_t kAct = 0;
    static constexpr uint32_t kWgt = kAct + kStages * kActBytes;
    static constexpr uint32_t kSfa = kWgt + kStages * kWgtBytes;
    static constexpr uint32_t kSfb = kSfa + kStages * kSfaBytes;
    static constexpr uint32_t kFull = kSfb + kStages * kSfbBytes;
    static constexpr uint32_t kEmpty = kFull + 8 * kStages;
    static constexpr uint32_t kDfull = kEmpty + 8 * kStages;
    static constexpr uint32_t kDempty = kDfull + 8;
    static constexpr uint32_t kDrain = kDempty + 8;
    static constexpr uint32_t kTmemSlot = kDrain + 8;
    static constexpr uint32_t kAbort = kTmemSlot + 4;
    static constexpr uint32_t kEnd = kAbort + 4;
    // tensor-memory columns of the scales: per stage and atom, 4 for the
    // activations and 4 for each of the two 128-row halves of the weights
    static constexpr int kSfCols = 12;
    static_assert(kAccCols + kStages * kAtoms * kSfCols <= kTmemCols, "tensor memory");
    static_assert(kEnd + 1024 <= (uint32_t)kSmemLimit, "shared memory");
};

// Instruction descriptor of the block-scaled kinds: A and B E2M1 (format 1)
// at bits 7 and 10, both K-major, N >> 3 at bit 17, the scale format at bit
// 23 (0 = E4M3, 1 = E8M0), M >> 4 at bit 24, the scale-factor byte of A at
// bit 29 and of B at bit 4.
constexpr uint32_t idesc_fp4(int kind, int m, int n) {
    return (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) |
           ((kind == 0 ? 1u : 0u) << 23) | ((uint32_t)(m >> 4) << 24);
}

// Shared-memory descriptor of a 512-byte scale atom as tcgen05.cp reads it:
// 32 rows of 16 bytes, no swizzle, 8-row groups 128 bytes apart.
__device__ __forceinline__ uint64_t smem_desc_atom(uint32_t addr) {
    uint64_t d = 0;
    d |= (uint64_t)((addr >> 4) & 0x3FFFu);
    d |= (uint64_t)1u << 16;                 // leading byte offset (one 16-byte column)
    d |= (uint64_t)(128u >> 4) << 32;        // stride byte offset
    d |= (uint64_t)1u << 46;                 // version
    return d;                                // layout type 0: no swizzle
}

__device__ __forceinline__ void tc_cp_atom(uint32_t taddr, uint64_t sdesc) {
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc)
                 : "memory");
}

template <int KIND>
__device__ __forceinline__ void mma_fp4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                        uint32_t idesc, uint32_t sfa, uint32_t sfb,
                                        uint32_t accumulate) {
    if constexpr (KIND == 1) {
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "setp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.scale_vec::4X "
            "[%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d_tmem),
            "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
            : "memory");
    } else {
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "setp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.scale_vec::2X "
            "[%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d_tmem),
            "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
            : "memory");
    }
}

// 1D bulk copy global -> shared, completion counted on `bar`.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void *src, uint32_t bytes,
                                          uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
            "r"(dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}

__device__ __forceinline__ void tmem_ld_x16_nowait(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {"
        "%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
}

__device__ __forceinline__ float nv_tensor_scale(float amax) {
    return amax > 0.0f ? __fdiv_rn(amax, 2688.0f) : 1.0f;
}

struct Fp4GemmArgs {
    const uint8_t *a_sf;        // activation scales, MMA layout
    const uint8_t *w_sf;        // weight scales, MMA layout
    const unsigned *a_amax;     // NVFP4: max |a| (fp32 bits), written by the quantize pass
    const float *w_tensor_scale;// NVFP4: the weights' tensor scale
    uint16_t *y;
    int M, N, K;
    int vec_store;              // N % 8 == 0 and y 16-byte aligned
    unsigned *err_word;
    uint64_t wait_limit;
};

template <int KIND>
__global__ void __launch_bounds__(kThreads, 1)
w4a4_gemm_tcgen05(const __grid_constant__ CUtensorMap act_map,
                  const __grid_constant__ CUtensorMap wgt_map, const Fp4GemmArgs p) {
    using C = Fp4Cfg<KIND>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    volatile uint32_t *abort_flag = reinterpret_cast<volatile uint32_t *>(smem + C::kAbort);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::kTmemSlot);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int KT = p.K / kStageK;
    const int atoms_k = p.K / C::kBlock / 4;          // scale atoms per 128-row block
    const int tiles_m = (p.M + kTok - 1) / kTok;
    const int tiles = tiles_m * ((p.N + kRows - 1) / kRows);

    auto full_bar = [&](int s) { return sbase + C::kFull + 8 * s; };
    auto empty_bar = [&](int s) { return sbase + C::kEmpty + 8 * s; };
    const uint32_t dfull_bar = sbase + C::kDfull;
    const uint32_t dempty_bar = sbase + C::kDempty;
    const uint32_t drain_bar = sbase + C::kDrain;
    auto wait = [&](uint32_t bar, uint32_t parity) {
        return mbar_wait(bar, parity, p.wait_limit, abort_flag, p.err_word);
    };

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
        }
        mbar_init(dfull_bar, 1);
        mbar_init(dempty_bar, kEpilogueWarps);
        mbar_init(drain_bar, 1);
        *abort_flag = 0u;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&act_map)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&wgt_map)) : "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(tmem_slot)),
                     "n"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        // ---------------- TMA producer ----------------
        if (lane == 0) {
            int issued_round[kStages];
            for (int s = 0; s < kStages; ++s) issued_round[s] = -1;
            int s = 0, r = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
                const int m0 = (t % tiles_m) * kTok, n0 = (t / tiles_m) * kRows;
                const bool second_half = n0 + kRows / 2 < p.N;   // weight rows n0+128.. exist
                const uint8_t *sfa = p.a_sf + ((int64_t)(m0 / 128) * atoms_k) * kAtomBytes;
                const uint8_t *sfb = p.w_sf + ((int64_t)(n0 / 128) * atoms_k) * kAtomBytes;
                const uint32_t tx = C::kActBytes + C::kWgtBytes + C::kSfaBytes +
                                    (second_half ? 2u : 1u) * (C::kSfbBytes / 2);
                for (int kt = 0; kt < KT; ++kt, s = (s + 1 == kStages ? 0 : s + 1), r += (s == 0)) {
                    if (r > 0 && !wait(empty_bar(s), (r - 1) & 1)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(full_bar(s), tx);
                    tma_load_2d(sbase + C::kAct + s * C::kActBytes, &act_map, kt * kRowBytes, m0,
                                full_bar(s));
                    tma_load_2d(sbase + C::kWgt + s * C::kWgtBytes, &wgt_map, kt * kRowBytes, n0,
                                full_bar(s));
                    const int64_t a0 = (int64_t)kt * C::kAtoms * kAtomBytes;
                    bulk_load(sbase + C::kSfa + s * C::kSfaBytes, sfa + a0, C::kSfaBytes, full_bar(s));
                    bulk_load(sbase + C::kSfb + s * C::kSfbBytes, sfb + a0, C::kSfbBytes / 2,
                              full_bar(s));
                    if (second_half)
                        bulk_load(sbase + C::kSfb + s * C::kSfbBytes + C::kSfbBytes / 2,
                                  sfb + (int64_t)atoms_k * kAtomBytes + a0, C::kSfbBytes / 2,
                                  full_bar(s));
                    issued_round[s] = r;
                }
            }
            for (int q = 0; q < kStages; ++q)
                if (issued_round[q] >= 0) mbar_drain(full_bar(q), issued_round[q] & 1, p.err_word);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------- scale copies and MMA issue ----------------
        if (lane == 0) {
            bool ok = true;
            int s = 0, r = 0, tcount = 0;
            const uint32_t sf_tmem = tmem_base + kAccCols;
            for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x, ++tcount) {
                if (tcount > 0 && !wait(dempty_bar, (tcount - 1) & 1)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                for (int kt = 0; kt < KT; ++kt, s = (s + 1 == kStages ? 0 : s + 1), r += (s == 0)) {
                    if (!wait(full_bar(s), r & 1)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t act = sbase + C::kAct + s * C::kActBytes;
                    const uint32_t wgt = sbase + C::kWgt + s * C::kWgtBytes;
                    const uint32_t sfa_s = sbase + C::kSfa + s * C::kSfaBytes;
                    const uint32_t sfb_s = sbase + C::kSfb + s * C::kSfbBytes;
                    // the stage's scales first, then its MMAs back to back: an
                    // MMA waits for the copies before it, so copies interleaved
                    // with the MMAs would stall every MMA
#pragma unroll
                    for (int a = 0; a < C::kAtoms; ++a) {
                        const uint32_t col = sf_tmem + (uint32_t)((s * C::kAtoms + a) * C::kSfCols);
                        tc_cp_atom(col, smem_desc_atom(sfa_s + a * kAtomBytes));
                        tc_cp_atom(col + 4, smem_desc_atom(sfb_s + a * kAtomBytes));
                        tc_cp_atom(col + 8, smem_desc_atom(sfb_s + (C::kAtoms + a) * kAtomBytes));
                    }
#pragma unroll
                    for (int a = 0; a < C::kAtoms; ++a) {
                        const uint32_t col = sf_tmem + (uint32_t)((s * C::kAtoms + a) * C::kSfCols);
#pragma unroll
                        for (int st = 0; st < C::kStepsPerAtom; ++st) {
                            const int ks = a * C::kStepsPerAtom + st;
                            // MXFP4: an atom holds the scales of two MMAs, bytes
                            // 0-1 and 2-3 of each column
                            const uint32_t sf_id = KIND == 0 ? (uint32_t)(2 * st) : 0u;
                            const uint32_t idesc =
                                idesc_fp4(KIND, kTok, kRows) | (sf_id << 29) | (sf_id << 4);
                            mma_fp4<KIND>(tmem_base, smem_desc_sw128(act + ks * 32),
                                          smem_desc_sw128(wgt + ks * 32), idesc, col | (sf_id << 30),
                                          (col + 4) | (sf_id << 30),
                                          (kt > 0 || ks > 0) ? 1u : 0u);
                        }
                    }
                    mma_commit(empty_bar(s));
                }
                if (ok) mma_commit(dfull_bar);
            }
            mma_commit(drain_bar);
            mbar_drain(drain_bar, 0, p.err_word);
        }
        __syncwarp();
    } else {
        // ---------------- epilogue (warps 2..5) ----------------
        const int quarter = warp & 3;
        const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
        float out_scale = 1.0f;
        if (KIND == 1)
            out_scale = __fmul_rn(nv_tensor_scale(__uint_as_float(*p.a_amax)), *p.w_tensor_scale);
        int tcount = 0;
        for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++tcount) {
            const int m0 = (t % tiles_m) * kTok, n0 = (t / tiles_m) * kRows;
            if (!__all_sync(0xFFFFFFFFu, wait(dfull_bar, tcount & 1))) break;
            tc_fence_after();
            const int m = m0 + quarter * 32 + lane;
            uint16_t *yrow = p.y + (int64_t)m * p.N;
#pragma unroll 1
            for (int c4 = 0; c4 < kAccCols / 64; ++c4) {
                uint32_t v[4][16];
#pragma unroll
                for (int q = 0; q < 4; ++q) tmem_ld_x16_nowait(tmem_base + lane_base + c4 * 64 + q * 16, v[q]);
                asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
                if (m < p.M) {
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const int n = n0 + c4 * 64 + q * 16;
                        uint32_t o[8];
#pragma unroll
                        for (int j = 0; j < 8; ++j)
                            o[j] = dev::pack_bf16x2(__fmul_rn(__uint_as_float(v[q][2 * j]), out_scale),
                                                    __fmul_rn(__uint_as_float(v[q][2 * j + 1]), out_scale));
                        if (p.vec_store && n + 16 <= p.N) {
                            uint4 *dst = reinterpret_cast<uint4 *>(yrow + n);
                            dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
                            dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
                        } else {
#pragma unroll
                            for (int j = 0; j < 16; ++j)
                                if (n + j < p.N)
                                    yrow[n + j] = (uint16_t)(o[j / 2] >> (16 * (j & 1)));
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(dempty_bar);
        }
        __syncwarp();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                     "n"(kTmemCols)
                     : "memory");
    }
}

}  // namespace

// Scale atoms of a matrix of `rows` rows in the MMA scale layout.
size_t fp4_mma_scale_bytes(int64_t rows, int64_t K, int kind) {
    const int64_t blk = kind == 0 ? 32 : 16;
    return (size_t)ceil_div(rows, 128) * (size_t)(K / blk / 4) * kAtomBytes;
}

// Workspace of qz_fp4a4_gemm: the activation codes, their scales in the MMA
// layout (sized for NVFP4, the larger), and one word for max |a|.
size_t fp4a4_codes_bytes(int64_t M, int64_t K) { return ((size_t)M * (K / 2) + 255) & ~(size_t)255; }
size_t fp4a4_scales_bytes(int64_t M, int64_t K) {
    return (fp4_mma_scale_bytes(M, K, 1) + 255) & ~(size_t)255;
}
size_t fp4a4_workspace_bytes(int64_t M, int64_t K) {
    return fp4a4_codes_bytes(M, K) + fp4a4_scales_bytes(M, K) + 256;
}

qz_status launch_fp4_quantize_mma(const void *a, int64_t M, int64_t K, int kind, void *codes,
                                  void *scales_mma, void *amax_word, cudaStream_t st);

qz_status launch_fp4a4_gemm(const void *a, const void *w_codes, const void *w_scales_mma,
                            const void *w_tensor_scale, int64_t M, int64_t N, int64_t K, int kind,
                            void *y, void *workspace, cudaStream_t st) {
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    uint8_t *a_codes = ws;
    uint8_t *a_sf = ws + fp4a4_codes_bytes(M, K);
    unsigned *a_amax = reinterpret_cast<unsigned *>(a_sf + fp4a4_scales_bytes(M, K));
    qz_status q = launch_fp4_quantize_mma(a, M, K, kind, a_codes, a_sf, a_amax, st);
    if (q != QZ_OK) return q;

    CUtensorMap act_map, wgt_map;
    if (!make_map_2d_cached(&act_map, CU_TENSOR_MAP_DATA_TYPE_UINT8, a_codes, (uint64_t)K / 2,
                            (uint64_t)M, (uint64_t)K / 2, kRowBytes, kTok,
                            CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map_2d_cached(&wgt_map, CU_TENSOR_MAP_DATA_TYPE_UINT8, w_codes, (uint64_t)K / 2,
                            (uint64_t)N, (uint64_t)K / 2, kRowBytes, kRows,
                            CU_TENSOR_MAP_SWIZZLE_128B))
        return QZ_ERR_CUDA;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return QZ_ERR_CUDA;
    }
    static DeviceOnce attr_once;
    const cudaError_t attr_err = attr_once.run(dev, [] {
        cudaError_t e = cudaFuncSetAttribute(w4a4_gemm_tcgen05<0>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(w4a4_gemm_tcgen05<1>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit);
        return e;
    });
    if (attr_err != cudaSuccess) return QZ_ERR_CUDA;
    unsigned *err = device_error_word();
    if (!err) return QZ_ERR_CUDA;

    Fp4GemmArgs args;
    args.a_sf = a_sf;
    args.w_sf = static_cast<const uint8_t *>(w_scales_mma);
    args.a_amax = a_amax;
    args.w_tensor_scale = static_cast<const float *>(w_tensor_scale);
    args.y = static_cast<uint16_t *>(y);
    args.M = (int)M;
    args.N = (int)N;
    args.K = (int)K;
    args.vec_store = (N % 8 == 0 && (reinterpret_cast<uintptr_t>(y) & 15) == 0) ? 1 : 0;
    args.err_word = err;
    args.wait_limit = device_wait_limit();
    const int64_t tiles = ceil_div(M, kTok) * ceil_div(N, kRows);
    const int grid = (int)(tiles < device_sm_count() ? tiles : device_sm_count());
    if (kind == 0) {
        w4a4_gemm_tcgen05<0><<<grid, kThreads, Fp4Cfg<0>::kEnd + 1024, st>>>(act_map, wgt_map, args);
    } else {
        w4a4_gemm_tcgen05<1><<<grid, kThreads, Fp4Cfg<1>::kEnd + 1024, st>>>(act_map, wgt_map, args);
    }
    return launch_status();
}

}  // namespace qz
