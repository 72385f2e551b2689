// qz_gemv_sm100.cu -- W4A16 decode GEMV on the sm_100a (tcgen05) tensor cores.
//
// Quantization concepts guide, "Quantize weights or activations": decoding
// one token at a time is bound by reading the weights, so 4-bit weights move a
// quarter of the bytes -- provided the kernel dequantizes inside the matmul
// (GPTQ explainer) and keeps up with HBM.  y (M x N) = a (M x K) * w_hat^T,
// M <= 16, w_hat = bf16_rne(S * (q - Z)) per element exactly as
// qz_dequantize forms it.
//
// On this part the mma.sync formulation of the GEMV runs out of issue slots
// before HBM does: every lane rebuilds MMA register operands (activation
// permutes, per-lane addressing) on top of the dequantization.  Here each
// dequantizing thread owns one weight row and writes its bf16 pairs straight
// into tensor memory as the A operand; one thread issues the MMAs with the
// activations read from shared memory by descriptor, so the per-weight work
// is the dequantization itself.
//
// Units of work: (128-row task, 128-wide K block).  The units are split into
// equal contiguous ranges, one per CTA, two CTAs per SM (stream-K), so every
// SM streams the same number of bytes.  Roles of the 6 warps of a CTA:
//   warp 0      TMA producer: per unit, the packed codes of 128 rows x 128 k
//               (64 bytes per row, 64-byte swizzle) and the activations of 16
//               token rows x 128 k (two 128-byte-swizzled boxes; rows >= M
//               read as zero) into a kStages-deep shared-memory ring.
//   warp 1      allocates 256 tensor-memory columns; one lane issues
//               tcgen05.mma M = 128, N = 16, K = 16 (8 per unit).  With
//               N = 16 an MMA is short, so consecutive K steps rotate over
//               four 16-column fp32 accumulators instead of chaining on one;
//               the epilogue adds the four in a fixed order.
//   warps 2..5  thread = weight row (its warp's tensor-memory lane quarter):
//               per unit, reads its 64 bytes of codes, dequantizes them into
//               64 natural-order bf16 pairs (byte permute + LOP3 + packed
//               bf16 subtract and multiply, bit-identical to qz_dequantize)
//               and stores them with tcgen05.st into one of kAStages A slots.
//               The scale and zero words of its row travel through a
//               per-thread cp.async ring kSzDepth units ahead.  At the end of
//               each task range they read the accumulator (tcgen05.ld) and
//               write y directly, or -- when other CTAs hold other K ranges of
//               the task -- write an fp32 partial slot; the last CTA of the
//               task (atomic counter) adds the slots in order and resets the
//               counter, so the result is deterministic.
// Every mbarrier wait is bounded (caller-set limit); on expiry every role
// stops, in-flight copies and MMAs are drained, tensor memory is released
// and the device error word reports the timeout.
#include <cuda.h>
#include <cuda_runtime.h>

#include "qz_sm100.cuh"

namespace qz {
namespace {

using namespace sm100;

constexpr int kRows = 128;                 // weight rows per task (MMA M)
constexpr int kTok = 16;                   // token columns (MMA N)
constexpr int kBlockK = 128;               // K per unit
constexpr int kStages = 6;                 // shared-memory ring
constexpr int kAStages = 3;                // tensor-memory A ring
constexpr int kSzDepth = 8;                // per-thread scale/zero ring
constexpr int kDequantWarps = 4;
constexpr int kThreads = 32 * (2 + kDequantWarps);
constexpr int kCodeBytes = kRows * kBlockK / 2;            // 8 KB
constexpr int kActBox = kTok * 64 * 2;                     // 2 KB: 16 rows x 64 bf16
constexpr int kActBytes = 2 * kActBox;                     // 4 KB
constexpr int kStageBytes = kCodeBytes + kActBytes;        // 12 KB
constexpr int kACols = kBlockK / 2;                        // 64 columns per A slot
constexpr int kAccCol = kAStages * kACols;                 // 192
constexpr int kAccs = 4;                                   // independent accumulators
constexpr int kTmemCols = 256;
constexpr uint32_t kIdesc = idesc_bf16(kRows, kTok);

struct Layout {
    static constexpr uint32_t ring = 0;                                  // 1024-aligned stages
    static constexpr uint32_t sz = ring + kStages * kStageBytes;         // [depth][2][128] words
    static constexpr uint32_t sz_bytes = kSzDepth * 2 * kRows * 4;
    static constexpr uint32_t bars = sz + sz_bytes;
    static constexpr uint32_t cfull = bars;
    static constexpr uint32_t cempty = cfull + 8 * kStages;
    static constexpr uint32_t afull = cempty + 8 * kStages;
    static constexpr uint32_t aempty = afull + 8 * kAStages;
    static constexpr uint32_t dfull = aempty + 8 * kAStages;
    static constexpr uint32_t dempty = dfull + 8;
    static constexpr uint32_t drain = dempty + 8;
    static constexpr uint32_t tmem_slot = drain + 8;
    static constexpr uint32_t abort_flag = tmem_slot + 4;
    static constexpr uint32_t flag = abort_flag + 4;                     // epilogue broadcast
    static constexpr uint32_t end = flag + 4;
};
constexpr int kSmemBytes = Layout::end + 1024;             // + alignment slack
static_assert(kSmemBytes * 2 <= 227 * 1024, "two CTAs per SM");
static_assert(kAccCol + kAccs * kTok <= kTmemCols, "tensor-memory columns");

struct TcArgs {
    const uint16_t *scales;
    const uint8_t *zeros;
    int M, N, K, group_size;
    int bpg_shift;          // log2(group_size / 128)
    int64_t units;          // tasks * kblocks
    int ctas;               // launched CTAs
    int kblocks, slots;
    uint16_t *y;
    float *partials;
    uint32_t *counters;
    uint64_t wait_limit;
    unsigned int *err;
};

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
__device__ __forceinline__ void epi_bar() {
    asm volatile("bar.sync 1, %0;" ::"n"(32 * kDequantWarps) : "memory");
}

// Position of a unit: 128-row task and 128-wide K block.
struct Cursor {
    int task, kb;
    __device__ __forceinline__ void next(int KB) {
        if (++kb == KB) { kb = 0; ++task; }
    }
};

// First CTA whose unit range [c*U/C, (c+1)*U/C) contains unit u.
__device__ __forceinline__ int64_t cta_of_unit(int64_t u, int64_t U, int64_t C) {
    return ((u + 1) * C - 1) / U;
}

__global__ void __launch_bounds__(kThreads, 2)
w4a16_gemv_tcgen05(const __grid_constant__ CUtensorMap code_map,
                   const __grid_constant__ CUtensorMap act_map, const TcArgs p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    volatile uint32_t *abort_flag = reinterpret_cast<volatile uint32_t *>(smem + Layout::abort_flag);
    volatile uint32_t *flag = reinterpret_cast<volatile uint32_t *>(smem + Layout::flag);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + Layout::tmem_slot);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t U = p.units;
    const int64_t u0 = (int64_t)blockIdx.x * U / p.ctas;
    const int64_t u1 = (int64_t)(blockIdx.x + 1) * U / p.ctas;
    const int nunits = (int)(u1 - u0);
    const int KB = p.kblocks;

    auto cfull = [&](int s) { return sbase + Layout::cfull + 8 * s; };
    auto cempty = [&](int s) { return sbase + Layout::cempty + 8 * s; };
    auto afull = [&](int s) { return sbase + Layout::afull + 8 * s; };
    auto aempty = [&](int s) { return sbase + Layout::aempty + 8 * s; };
    const uint32_t dfull = sbase + Layout::dfull, dempty = sbase + Layout::dempty;
    const uint32_t drain = sbase + Layout::drain;
    auto wait = [&](uint32_t bar, uint32_t parity) {
        return mbar_wait(bar, parity, p.wait_limit, abort_flag, p.err);
    };
    // (task, kb) of this CTA's first unit; every role then steps through its
    // units with a Cursor (no division per unit).
    const int task0 = (int)(u0 / KB), kb0 = (int)(u0 - (int64_t)task0 * KB);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(cfull(s), 1);
            mbar_init(cempty(s), kDequantWarps + 1);     // dequant warps + MMA commit
        }
        for (int s = 0; s < kAStages; ++s) {
            mbar_init(afull(s), kDequantWarps);
            mbar_init(aempty(s), 1);
        }
        mbar_init(dfull, 1);
        mbar_init(dempty, kDequantWarps);
        mbar_init(drain, 1);
        *abort_flag = 0u;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&code_map)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&act_map)) : "memory");
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
    const uint32_t tmem_acc = tmem_base + kAccCol;      // kAccs x 16 columns

    if (warp == 0) {
        // ---------------- TMA producer ----------------
        if (lane == 0) {
            int issued_round[kStages];
            for (int s = 0; s < kStages; ++s) issued_round[s] = -1;
            Cursor cur{task0, kb0};
            for (int it = 0, s = 0, r = 0; it < nunits; ++it, cur.next(KB)) {
                if (r > 0 && !wait(cempty(s), (r - 1) & 1)) break;
                const uint32_t st = sbase + Layout::ring + s * kStageBytes;
                mbar_arrive_expect_tx(cfull(s), kStageBytes);
                tma_load_2d(st, &code_map, cur.kb * (kBlockK / 2), cur.task * kRows, cfull(s));
                tma_load_2d(st + kCodeBytes, &act_map, cur.kb * kBlockK, 0, cfull(s));
                tma_load_2d(st + kCodeBytes + kActBox, &act_map, cur.kb * kBlockK + 64, 0, cfull(s));
                issued_round[s] = r;
                if (++s == kStages) { s = 0; ++r; }
            }
            // every issued copy must have landed before the CTA may exit
            for (int s = 0; s < kStages; ++s)
                if (issued_round[s] >= 0) mbar_drain(cfull(s), issued_round[s] & 1, p.err);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            int seg = 0;
            bool ok = true;
            bool seg_start = true;
            int kb = kb0;
            for (int it = 0, s = 0, r = 0, sa = 0, ra = 0; it < nunits && ok; ++it) {
                if (seg_start && seg > 0 && !wait(dempty, (seg - 1) & 1)) break;
                ok = wait(cfull(s), r & 1) && wait(afull(sa), ra & 1);
                if (!ok) break;
                tc_fence_after();
                const uint32_t act = sbase + Layout::ring + s * kStageBytes + kCodeBytes;
#pragma unroll
                for (int kk = 0; kk < kBlockK / 16; ++kk)
                    mma_ts(tmem_acc + (kk % kAccs) * kTok, tmem_base + sa * kACols + kk * 8,
                           smem_desc_sw128(act + (kk >> 2) * kActBox + (kk & 3) * 32), kIdesc,
                           (!seg_start || kk >= kAccs) ? 1u : 0u);
                mma_commit(cempty(s));
                mma_commit(aempty(sa));
                seg_start = it == nunits - 1 || kb == KB - 1;      // last unit of a task range
                if (seg_start) {
                    mma_commit(dfull);
                    ++seg;
                }
                if (++kb == KB) kb = 0;
                if (++s == kStages) { s = 0; ++r; }
                if (++sa == kAStages) { sa = 0; ++ra; }
            }
            // every issued MMA must finish before tensor memory is released
            mma_commit(drain);
            mbar_drain(drain, 0, p.err);
        }
        __syncwarp();
    } else {
        // ---------------- dequantize + epilogue (warps 2..5) ----------------
        const int quarter = warp & 3;                 // tensor-memory lane quarter
        const int row_local = quarter * 32 + lane;
        const int tid = row_local;                    // 0..127
        const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
        const int64_t gpr = p.K / p.group_size;
        const uint32_t *scale_words = reinterpret_cast<const uint32_t *>(p.scales);
        const uint32_t *zero_words = reinterpret_cast<const uint32_t *>(p.zeros);
        const uint32_t sz_base = sbase + Layout::sz;
        // 64-byte swizzle: 16-byte chunk c of row r sits at chunk c ^ ((r >> 1) & 3)
        const int swz = (row_local >> 1) & 3;

        // Scale/zero entry of this thread's row for a unit: row_entry + (kb >> shift),
        // where row_entry = n * gpr changes only with the task.
        struct RowCursor {
            Cursor c;
            int64_t row_entry;
            bool valid;
            __device__ __forceinline__ void set_row(int row_local, int N, int64_t gpr) {
                const int64_t n = (int64_t)c.task * kRows + row_local;
                valid = n < N;
                row_entry = valid ? n * gpr : 0;
            }
            __device__ __forceinline__ void next(int KB, int row_local, int N, int64_t gpr) {
                if (++c.kb == KB) {
                    c.kb = 0;
                    ++c.task;
                    set_row(row_local, N, gpr);
                }
            }
        };
        const uint32_t sz_thread = sz_base + (uint32_t)tid * 4u;
        auto issue_sz = [&](const RowCursor &rc, int slot) {
            if (rc.valid) {
                const int64_t e = rc.row_entry + (rc.c.kb >> p.bpg_shift);
                cp_async4(sz_thread + (uint32_t)(slot * 2 * kRows) * 4u, scale_words + (e >> 1));
                cp_async4(sz_thread + (uint32_t)((slot * 2 + 1) * kRows) * 4u, zero_words + (e >> 2));
            }
        };
        RowCursor ahead{{task0, kb0}, 0, false};       // unit it + kSzDepth - 1
        ahead.set_row(row_local, p.N, gpr);
#pragma unroll 1
        for (int q = 0; q < kSzDepth - 1; ++q) {
            if (q < nunits) issue_sz(ahead, q);
            cp_async_commit();
            ahead.next(KB, row_local, p.N, gpr);
        }
        // swizzled byte offsets of this row's four 16-byte code chunks
        uint32_t chunk_off[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) chunk_off[j] = (uint32_t)(row_local * 64 + 16 * (j ^ swz));

        int seg = 0;
        bool seg_whole_start = kb0 == 0;             // the current task range starts at kb 0
        RowCursor cur{{task0, kb0}, 0, false};
        cur.set_row(row_local, p.N, gpr);
        for (int it = 0, s = 0, r = 0, sa = 0, ra = 0, slot = 0; it < nunits;
             ++it, cur.next(KB, row_local, p.N, gpr)) {
            // scale and zero of this unit (own copies)
            cp_async_wait<kSzDepth - 2>();
            const int64_t e = cur.row_entry + (cur.c.kb >> p.bpg_shift);
            const uint32_t sw = *reinterpret_cast<const uint32_t *>(
                smem + Layout::sz + ((slot * 2 + 0) * kRows + tid) * 4);
            const uint32_t zw = *reinterpret_cast<const uint32_t *>(
                smem + Layout::sz + ((slot * 2 + 1) * kRows + tid) * 4);
            // unit it + kSzDepth - 1 goes to slot (it - 1) mod kSzDepth, read one unit ago
            if (it + kSzDepth - 1 < nunits) issue_sz(ahead, slot == 0 ? kSzDepth - 1 : slot - 1);
            cp_async_commit();
            ahead.next(KB, row_local, p.N, gpr);
            const int cs = s, cr = r, csa = sa, cra = ra;
            if (++s == kStages) { s = 0; ++r; }
            if (++sa == kAStages) { sa = 0; ++ra; }
            if (++slot == kSzDepth) slot = 0;
            const uint32_t os = (uint32_t)(e & 1) * 2u, oz = (uint32_t)(e & 3);
            const uint32_t s2 = dev::prmt(sw, 0u, os * 0x0101u + (os + 1u) * 0x1010u);   // (S, S)
            const uint32_t z2 = dev::prmt(zw, 0x43434343u, oz * 0x0101u + 0x4040u);      // bf16(128+Z) x2

            // Waits are decided per warp (tcgen05.st needs every lane).  A warp
            // whose wait fails skips the unit's work but keeps iterating to the
            // end of the task range, where the four warps meet and stop
            // together (the abort flag is set by then).
            bool good = __all_sync(0xFFFFFFFFu, wait(cfull(cs), cr & 1));
            if (good) {
                const uint8_t *stage = smem + Layout::ring + cs * kStageBytes;
                uint4 c[4];
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    c[j] = *reinterpret_cast<const uint4 *>(stage + chunk_off[j]);
                __syncwarp();
                if (lane == 0) mbar_arrive(cempty(cs));             // codes consumed
                good = cra == 0 || __all_sync(0xFFFFFFFFu, wait(aempty(csa), (cra - 1) & 1));
                if (good) {
                    // chunk q = k 32q..32q+31 = A columns 16q..16q+15 (natural order)
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const uint32_t words[4] = {c[q].x, c[q].y, c[q].z, c[q].w};
                        uint32_t a[16];
#pragma unroll
                        for (int wi = 0; wi < 4; ++wi) {
                            const uint32_t w = words[wi], w4 = w >> 4;
#pragma unroll
                            for (int i = 0; i < 4; ++i)
                                a[wi * 4 + i] = dequant_pair_nat(w, w4, i, s2, z2);
                        }
                        tmem_st_x16(tmem_base + lane_base + csa * kACols + q * 16, a);
                    }
                    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(afull(csa));
                }
            }

            if (!(it == nunits - 1 || cur.c.kb == KB - 1)) continue;
            // ---------------- epilogue of the task range ending at unit it ----------------
            const int task = cur.c.task;
            const bool whole = seg_whole_start && cur.c.kb == KB - 1;
            seg_whole_start = true;                          // the next range starts at kb 0
            __all_sync(0xFFFFFFFFu, wait(dfull, seg & 1));
            epi_bar();
            if (warp == 2 && lane == 0) *flag = *abort_flag;
            epi_bar();
            if (*flag) break;                                   // the four warps together
            tc_fence_after();
            float v[16];
            {
                uint32_t r0[16], r1[16];
                tmem_ld_x16(tmem_acc + lane_base, r0);
                tmem_ld_x16(tmem_acc + lane_base + kTok, r1);
#pragma unroll
                for (int t = 0; t < 16; ++t) v[t] = __uint_as_float(r0[t]) + __uint_as_float(r1[t]);
                tmem_ld_x16(tmem_acc + lane_base + 2 * kTok, r0);
                tmem_ld_x16(tmem_acc + lane_base + 3 * kTok, r1);
#pragma unroll
                for (int t = 0; t < 16; ++t) v[t] += __uint_as_float(r0[t]) + __uint_as_float(r1[t]);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(dempty);                  // accumulator free again
            const int64_t n = (int64_t)task * kRows + row_local;
            if (whole) {
                if (n < p.N)
                    for (int t = 0; t < p.M; ++t)
                        p.y[(int64_t)t * p.N + n] = (uint16_t)dev::f32_to_bf16_rne(v[t]);
            } else {
                const int64_t first = cta_of_unit((int64_t)task * KB, U, p.ctas);
                const int64_t last = cta_of_unit((int64_t)task * KB + KB - 1, U, p.ctas);
                const int contributors = (int)(last - first + 1);
                const int64_t slot_elems = (int64_t)p.M * kRows;
                float *base = p.partials + (int64_t)task * p.slots * slot_elems;
                float *mine = base + (blockIdx.x - first) * slot_elems;
                for (int t = 0; t < p.M; ++t) __stcg(&mine[t * kRows + row_local], v[t]);
                __threadfence();
                epi_bar();
                if (warp == 2 && lane == 0) *flag = atomicAdd(&p.counters[task], 1u);
                epi_bar();
                const bool last_one = *flag == (uint32_t)(contributors - 1);
                if (last_one) {
                    __threadfence();
                    // add the slots in slot order, all tokens' loads of two slots together
                    float sum[kTok];
#pragma unroll
                    for (int t = 0; t < kTok; ++t) sum[t] = 0.0f;
                    for (int c = 0; c < contributors; c += 2) {
                        float x0[kTok], x1[kTok];
                        const float *s0 = base + (int64_t)c * slot_elems + row_local;
                        const bool two = c + 1 < contributors;
#pragma unroll
                        for (int t = 0; t < kTok; ++t) {
                            x0[t] = t < p.M ? __ldcg(s0 + t * kRows) : 0.0f;
                            x1[t] = (t < p.M && two) ? __ldcg(s0 + slot_elems + t * kRows) : 0.0f;
                        }
#pragma unroll
                        for (int t = 0; t < kTok; ++t) {
                            sum[t] += x0[t];
                            if (two) sum[t] += x1[t];
                        }
                    }
                    if (n < p.N) {
#pragma unroll
                        for (int t = 0; t < kTok; ++t)
                            if (t < p.M)
                                p.y[(int64_t)t * p.N + n] = (uint16_t)dev::f32_to_bf16_rne(sum[t]);
                    }
                    epi_bar();
                    if (warp == 2 && lane == 0) p.counters[task] = 0u;
                }
                epi_bar();                                   // *flag is reused
            }
            ++seg;
        }
        cp_async_wait<0>();
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

bool tc_gemv_eligible(const void *a, const void *codes, const void *scales, const void *zeros,
                      int64_t M, int64_t N, int64_t K, int64_t group_size) {
    const int64_t bpg = group_size / kBlockK;     // units per group: a power of two
    return M >= 1 && M <= kTok && K % kBlockK == 0 && group_size % kBlockK == 0 &&
           K % group_size == 0 && (bpg & (bpg - 1)) == 0 && aligned(a, 16) && aligned(codes, 16) && aligned(scales, 4) &&
           aligned(zeros, 4) && (N * (K / group_size)) % 4 == 0;
}

TcGemvPlan tc_gemv_plan(int64_t M, int64_t N, int64_t K) {
    TcGemvPlan p{};
    p.tasks = ceil_div(N, kRows);
    p.kblocks = K / kBlockK;
    const int64_t units = p.tasks * p.kblocks;
    p.ctas = units < 2 * kSmCount ? units : 2 * kSmCount;
    const int64_t per_cta = units / p.ctas;
    p.slots = ceil_div(p.kblocks, per_cta) + 1;
    if (p.slots > p.kblocks) p.slots = p.kblocks;
    p.partial_bytes = (size_t)p.tasks * p.slots * (size_t)M * kRows * sizeof(float);
    p.partial_bytes = (p.partial_bytes + 255) & ~(size_t)255;
    return p;
}

qz_status launch_w4a16_gemv_tc(const void *a, const void *codes, const void *scales,
                               const void *zeros, int64_t M, int64_t N, int64_t K,
                               int64_t group_size, void *y, float *partials, uint32_t *counters,
                               cudaStream_t st) {
    CUtensorMap code_map, act_map;
    if (!make_map_2d(&code_map, CU_TENSOR_MAP_DATA_TYPE_UINT8, codes, (uint64_t)K / 2,
                     (uint64_t)N, (uint64_t)K / 2, kBlockK / 2, kRows, CU_TENSOR_MAP_SWIZZLE_64B) ||
        !make_map_2d(&act_map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a, (uint64_t)K, (uint64_t)M,
                     (uint64_t)K * 2, 64, kTok, CU_TENSOR_MAP_SWIZZLE_128B))
        return QZ_ERR_CUDA;
    unsigned int *err = device_error_word();
    if (!err) return QZ_ERR_CUDA;
    const TcGemvPlan plan = tc_gemv_plan(M, N, K);
    TcArgs args;
    args.scales = static_cast<const uint16_t *>(scales);
    args.zeros = static_cast<const uint8_t *>(zeros);
    args.M = (int)M; args.N = (int)N; args.K = (int)K; args.group_size = (int)group_size;
    {
        const int64_t bpg = group_size / kBlockK;
        int sh = 0;
        while ((int64_t(1) << sh) < bpg) ++sh;
        args.bpg_shift = sh;
    }
    args.units = plan.tasks * plan.kblocks;
    args.ctas = (int)plan.ctas;
    args.kblocks = (int)plan.kblocks;
    args.slots = (int)plan.slots;
    args.y = static_cast<uint16_t *>(y);
    args.partials = partials;
    args.counters = counters;
    args.wait_limit = device_wait_limit();
    args.err = err;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return QZ_ERR_CUDA;
    static std::once_flag attr_once[64];
    if (dev >= 0 && dev < 64)
        std::call_once(attr_once[dev], [] {
            cudaFuncSetAttribute(w4a16_gemv_tcgen05, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kSmemBytes);
        });
    w4a16_gemv_tcgen05<<<(unsigned)plan.ctas, kThreads, kSmemBytes, st>>>(code_map, act_map, args);
    return launch_status();
}

}  // namespace qz
