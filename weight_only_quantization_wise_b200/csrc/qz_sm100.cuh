// qz_sm100.cuh -- sm_100a building blocks shared by the tcgen05 kernels:
// mbarriers with bounded waits, TMA 2D loads, tcgen05 MMA / TMEM access,
// shared-memory matrix descriptors, and host-side tensor-map encoding.
// Internal; not installed.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "qz_internal.cuh"

namespace qz {
namespace sm100 {

#ifdef __CUDACC__
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

// try_wait that lets the hardware suspend the thread for up to `hint_ns`
// while the phase is incomplete (fewer polling instructions).
__device__ __forceinline__ bool mbar_try_wait_hint(uint32_t bar, uint32_t parity, uint32_t hint_ns) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(hint_ns)
        : "memory");
    return ok != 0;
}

// Bounded wait: true when the phase completed, false when `limit_ns` of wall
// time ran out (then the CTA-local abort flag and the device error word are
// set) or another thread of the CTA aborted; the caller unwinds either way.
// Each poll may suspend the thread for up to a microsecond, so checking the
// clock and the abort flag after every poll costs little.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, uint64_t limit_ns,
                                          volatile uint32_t *abort_flag, unsigned int *err_word) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    for (;;) {
        if (mbar_try_wait_hint(bar, parity, 1000u)) return true;
        if (*abort_flag) return false;
        if (global_ns() - t0 > limit_ns) break;
    }
    *abort_flag = 1u;
    atomicOr(err_word, 1u);
    return false;
}

// Wait used while unwinding: copies and MMAs already issued complete on their
// own, so this bound (2 s) is independent of the caller's limit.
constexpr uint64_t kDrainLimitNs = 2000000000ull;
__device__ __forceinline__ void mbar_drain(uint32_t bar, uint32_t parity, unsigned int *err_word) {
    volatile uint32_t never = 0;
    mbar_wait(bar, parity, kDrainLimitNs, &never, err_word);
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, int x, int y,
                                            uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
        : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups
// 1024 bytes apart (stride byte offset), leading byte offset unused (1),
// descriptor version 1.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr) {
    uint64_t d = 0;
    d |= (uint64_t)((addr >> 4) & 0x3FFFu);
    d |= (uint64_t)1u << 16;                 // leading byte offset (16 B units)
    d |= (uint64_t)(1024u >> 4) << 32;       // stride byte offset
    d |= (uint64_t)1u << 46;                 // version
    d |= (uint64_t)2u << 61;                 // 128-byte swizzle
    return d;
}

// Instruction descriptor, kind::f16: D f32, A bf16, B bf16, both K-major,
// N >> 3 at bit 17, M >> 4 at bit 24.
constexpr uint32_t idesc_bf16(int m, int n) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) |
           ((uint32_t)(m >> 4) << 24);
}

// D (tensor memory) (+)= A (tensor memory) * B (shared memory descriptor).
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void mma_commit(uint32_t bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
        : "memory");
}

__device__ __forceinline__ void tmem_st_x16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {"
        "%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15])
        : "memory");
}

__device__ __forceinline__ void tmem_ld_x16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {"
        "%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Natural-order bf16 pair (k = 2i, 2i+1) of a packed code word: byte i of
// `w` holds q_{2i} in its low nibble, byte i of `w >> 4` holds q_{2i+1}.
// z2 holds bf16(128 + Z) twice; the result is bf16_rne(S * (q - Z)).
__device__ __forceinline__ uint32_t dequant_pair_nat(uint32_t w, uint32_t w4, int i,
                                                     uint32_t s2, uint32_t z2) {
    const uint32_t sel = (uint32_t)i | ((uint32_t)(4 + i) << 8);
    const uint32_t t = dev::prmt(w, w4, sel);
    const uint32_t x = dev::and_or<0x000F000Fu>(t, 0x43004300u);  // bf16(128 + q)
    return dev::bf16x2_mul(dev::bf16x2_sub(x, z2), s2);
}
#endif  // __CUDACC__

// ---------------------------------------------------------------------------
// Host: tensor maps through the driver entry point (no link-time libcuda).
// ---------------------------------------------------------------------------
using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion,
                                   CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// 2D tensor map over a row-major array: `inner` elements per row, `outer`
// rows `row_bytes` apart; box of box_inner x box_outer; out-of-range
// elements of a box read as zero.
inline bool make_map_2d(CUtensorMap *map, CUtensorMapDataType dt, const void *base, uint64_t inner,
                        uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
                        CUtensorMapSwizzle swz) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {row_bytes};
    const cuuint32_t box[2] = {box_inner, box_outer};
    const cuuint32_t elem[2] = {1, 1};
    return fn(map, dt, 2, const_cast<void *>(base), dims, strides, box, elem,
              CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// make_map_2d through a small process-wide cache: a map depends only on its
// arguments, so a cached copy for the same arguments is always valid (also
// when the memory behind `base` was freed and allocated again).  Saves the
// host time of encoding the maps of every launch in decode loops.
inline bool make_map_2d_cached(CUtensorMap *map, CUtensorMapDataType dt, const void *base,
                               uint64_t inner, uint64_t outer, uint64_t row_bytes,
                               uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swz) {
    struct Entry {
        const void *base;
        uint64_t inner, outer, row_bytes;
        uint32_t box_inner, box_outer;
        int dt, swz;
        bool used;
        CUtensorMap map;
    };
    constexpr int kEntries = 64;
    static Entry table[kEntries];
    static int next = 0;
    static std::mutex mu;
    {
        std::lock_guard<std::mutex> lock(mu);
        for (const Entry &e : table)
            if (e.used && e.base == base && e.inner == inner && e.outer == outer &&
                e.row_bytes == row_bytes && e.box_inner == box_inner && e.box_outer == box_outer &&
                e.dt == (int)dt && e.swz == (int)swz) {
                *map = e.map;
                return true;
            }
    }
    if (!make_map_2d(map, dt, base, inner, outer, row_bytes, box_inner, box_outer, swz))
        return false;
    std::lock_guard<std::mutex> lock(mu);
    Entry &e = table[next];
    next = (next + 1) % kEntries;
    e = Entry{base, inner, outer, row_bytes, box_inner, box_outer, (int)dt, (int)swz, true, *map};
    return true;
}

}  // namespace sm100
}  // namespace qz
