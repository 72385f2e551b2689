// qz_internal.cuh -- internal helpers shared by the libqz CUDA sources.
// Not installed; the public interface is include/qz.h.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <mutex>

#include "qz.h"

namespace qz {

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------

// SMs of a B200.  Workspace sizes (qz_workspace_bytes, a pure function of
// the shapes) are computed for this count; grids are sized for the device's
// own count capped at it (device_sm_count), and every split-K plan made for
// fewer SMs needs no more workspace than the plan for kSmCount.
constexpr int kSmCount = 148;
constexpr int kMaxDevices = 64;

// A set-up step that must succeed once per device (a symbol address, a
// kernel attribute).  run() calls `setup` (which returns a cudaError_t) until
// it has succeeded once for the device; a failure is not remembered, so the
// next call retries (and the failed call's CUDA error is cleared, so it does
// not surface in a later launch check).  Thread-safe.
class DeviceOnce {
  public:
    template <typename F>
    cudaError_t run(int dev, F &&setup) {
        if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
        if (done_[dev].load(std::memory_order_acquire)) return cudaSuccess;
        std::lock_guard<std::mutex> lock(mu_);
        if (done_[dev].load(std::memory_order_relaxed)) return cudaSuccess;
        const cudaError_t e = setup();
        if (e == cudaSuccess) done_[dev].store(true, std::memory_order_release);
        else cudaGetLastError();
        return e;
    }

  private:
    std::mutex mu_;
    std::atomic<bool> done_[kMaxDevices] = {};
};

// SMs the grids of the current device are sized for: its multiprocessor
// count, capped at kSmCount (read once per device; kSmCount if the query
// fails).
int device_sm_count();

inline bool aligned(const void *p, size_t a) {
    return (reinterpret_cast<uintptr_t>(p) % a) == 0;
}

inline qz_status launch_status() {
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? QZ_OK : QZ_ERR_CUDA;
}

inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Code range of a format (see qz.h).
inline void code_range(int bits, int symmetric, int *qmin, int *qmax) {
    if (symmetric) {
        *qmax = (1 << (bits - 1)) - 1;
        *qmin = -*qmax;
    } else if (bits == 4) {
        *qmin = 0;
        *qmax = 15;
    } else {
        *qmin = -128;
        *qmax = 127;
    }
}

// ---------------------------------------------------------------------------
// Launchers (defined in the .cu files; arguments already validated)
// ---------------------------------------------------------------------------

qz_status launch_quantize_pack(const void *w, int64_t N, int64_t K, int bits,
                               int symmetric, int64_t group_size, void *codes,
                               void *scales, void *zeros, void *workspace,
                               cudaStream_t stream);
size_t quantize_workspace_bytes(int64_t group_size);

qz_status launch_dequantize(const void *codes, const void *scales, const void *zeros,
                            int64_t N, int64_t K, int bits, int symmetric,
                            int64_t group_size, void *w_hat, cudaStream_t stream);

// GEMV work plan (stream-K): the (128-row task x 128-wide K block) units
// are split into equal contiguous ranges, one per launched CTA; each of a
// CTA's four consumer warps owns 32 rows of every unit (a subtask), and a
// subtask whose units span several CTAs is reduced through per-subtask
// partial slots.
struct GemvPlan {
    int unit_k;           // K per unit: 128, or 256 (int4 two-half units)
    int64_t tasks;        // 128-row tasks
    int64_t kblocks;      // units per task (K / unit_k)
    int64_t ctas;         // launched CTAs (each owns at least one unit)
    int64_t slots;        // partial slots per subtask (max contributors)
    size_t partial_bytes; // fp32 partials [tasks * 4][slots][M][32]
    size_t counter_bytes; // uint32 arrival counter per 32-row subtask
    size_t total_bytes;
};
// Workspace: fp32 partials at offset 0, then one uint32 counter per subtask.
// `sms`: the SMs the grid is sized for (device_sm_count() at launch).
GemvPlan gemv_plan(int64_t M, int64_t N, int64_t K, int bits, int sms, int unit_k = 128);
// K per unit the int4 GEMV takes for these arguments (128 or 256); without
// pointers, for 16-byte aligned scale and zero arrays.
int gemv_unit_k(int bits, int64_t M, int64_t N, int64_t K, int64_t group_size,
                const void *scales, const void *zeros);
int gemv_fp4_unit_k(int64_t M, int64_t K, const void *scales);
inline int gemv_unit_k(int bits, int64_t M, int64_t N, int64_t K, int64_t group_size) {
    static const uint4 aligned_probe[1] = {};
    return gemv_unit_k(bits, M, N, K, group_size, aligned_probe, aligned_probe);
}
// Workspace bytes that serve the plan of every SM count up to kSmCount.
size_t gemv_workspace_bound(int64_t M, int64_t N, int64_t K, int bits, int max_unit_k = 128);

// `overlap`: qz_set_launch_overlap mode for this launch.
qz_status launch_w4a16_gemv(const void *a, const void *codes, const void *scales,
                            const void *zeros, int64_t M, int64_t N, int64_t K,
                            int64_t group_size, void *y, void *workspace,
                            const GemvPlan &plan, int overlap, cudaStream_t stream);
qz_status launch_w8a16_gemv(const void *a, const void *codes, const void *scales,
                            int64_t M, int64_t N, int64_t K, void *y, void *workspace,
                            const GemvPlan &plan, int overlap, cudaStream_t stream);

// FP4 with block scales (qz_fp4.cu, qz_gemv.cu, qz_gemm_fp4.cu); kind 0 =
// MXFP4, 1 = NVFP4.
int fp4_block_size(int kind);
qz_status launch_fp4_quantize(const void *w, int64_t N, int64_t K, int kind, void *codes,
                              void *scales, void *tensor_scale, cudaStream_t stream);
qz_status launch_fp4_dequantize(const void *codes, const void *scales, const void *tensor_scale,
                                int64_t N, int64_t K, int kind, void *w_hat, cudaStream_t stream);
qz_status launch_fp4a16_gemv(const void *a, const void *codes, const void *scales,
                             const void *tensor_scale, int64_t M, int64_t N, int64_t K, int kind,
                             void *y, void *workspace, const GemvPlan &plan, int overlap,
                             cudaStream_t stream);

// W4A4 GEMM: the MMA scale layout (atoms of 128 rows x 4 scales), the
// in-call activation quantization and the block-scaled tcgen05 GEMM.
size_t fp4_mma_scale_bytes(int64_t rows, int64_t K, int kind);
size_t fp4a4_workspace_bytes(int64_t M, int64_t K);
qz_status launch_fp4_scales_to_mma(const void *scales, int64_t rows, int64_t K, int kind,
                                   void *scales_mma, cudaStream_t stream);
qz_status launch_fp4a4_gemm(const void *a, const void *w_codes, const void *w_scales_mma,
                            const void *w_tensor_scale, int64_t M, int64_t N, int64_t K, int kind,
                            void *y, void *workspace, cudaStream_t stream);

// Split-K workspace of the GEMM whose grid is sized for `sms` SMs; the
// kSmCount figure (gemm_workspace_bytes) bounds every smaller count.
size_t gemm_workspace_bytes_for(int64_t M, int64_t N, int64_t K, int sms);
size_t gemm_workspace_bytes(int64_t M, int64_t N, int64_t K);
qz_status launch_w4a16_gemm(const void *a, const void *codes, const void *scales,
                            const void *zeros, int64_t M, int64_t N, int64_t K,
                            int64_t group_size, void *y, void *workspace,
                            cudaStream_t stream);
qz_status launch_w8a16_gemm(const void *a, const void *codes, const void *scales, int64_t M,
                            int64_t N, int64_t K, void *y, void *workspace, cudaStream_t stream);

// GPTQ (qz_gptq.cu): fp64 workspace of the damped Hessian factor, its
// inverse, the working weights and one block of scaled errors.
size_t gptq_workspace_bytes(int64_t N, int64_t K);
qz_status launch_gptq(const void *w, const void *x, int64_t N, int64_t K, int64_t n_samples,
                      int bits, int symmetric, int64_t group_size, double damp, void *codes,
                      void *scales, void *zeros, void *workspace, cudaStream_t stream);

uint64_t device_wait_limit();
// qz_set_launch_overlap mode (0 or 1) for the decode GEMV launches.
int32_t launch_overlap();
// Device address of the word that bounded device-side waits set on expiry
// (read and cleared by qz_device_status); null if it cannot be resolved.
unsigned int *device_error_word();

}  // namespace qz

// ---------------------------------------------------------------------------
// Device side
// ---------------------------------------------------------------------------
#ifdef __CUDACC__
namespace qz {
namespace dev {

// bf16 (as 16 raw bits) widened to fp32: exact.
__device__ __forceinline__ float bf16_lo(uint32_t pair) { return __uint_as_float(pair << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t pair) { return __uint_as_float(pair & 0xFFFF0000u); }

// fp32 -> bf16 bits, round to nearest even (hardware conversion).
__device__ __forceinline__ uint32_t f32_to_bf16_rne(float x) {
    uint16_t r;
    asm("cvt.rn.bf16.f32 %0, %1;" : "=h"(r) : "f"(x));
    return r;
}

// Exact int8 code pair to bf16x2 (q_lo, q_hi): the code bytes u = b ^ 0x80
// sit in bits 0..7 of the fp32 2^23 (mlo, mhi: 2^23 + q + 128), and one
// sub.rn.f32x2 of 2^23 + 128 leaves both q exactly; the pack is exact
// (|q| <= 128).  A bf16 multiply by (S, S) then rounds S*q once.  (One fma
// per value forming S*q directly would overflow its intermediate 2^15 S for
// scales above 2^113, which finite bf16 weights can reach.)
__device__ __forceinline__ uint32_t i8_codes_bf16x2(uint32_t mlo, uint32_t mhi) {
    uint32_t lo, hi;
    asm("{\n\t.reg .b64 mm, kk, qq;\n\t"
        "mov.b64 mm, {%2, %3};\n\t"
        "mov.b64 kk, {%4, %4};\n\t"
        "sub.rn.f32x2 qq, mm, kk;\n\t"
        "mov.b64 {%0, %1}, qq;\n\t}"
        : "=r"(lo), "=r"(hi)
        : "r"(mlo), "r"(mhi), "r"(0x4B000080u));       // 2^23 + 128
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(__uint_as_float(hi)), "f"(__uint_as_float(lo)));
    return r;
}

// Two fp32 -> packed bf16x2 (lo in bits 0..15), round to nearest even.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// fp32 scale -> bf16 bits rounded toward +inf (S >= 0).
__device__ __forceinline__ uint32_t bf16_round_up_bits(float s) {
    uint32_t b = __float_as_uint(s);
    uint32_t kept = b & 0xFFFF0000u;
    if (b & 0x0000FFFFu) kept += 0x00010000u;
    return kept >> 16;
}

// Packed bf16x2 arithmetic, one IEEE rounding to nearest even per lane.
__device__ __forceinline__ uint32_t bf16x2_sub(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}
__device__ __forceinline__ uint32_t bf16x2_add(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("add.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}
__device__ __forceinline__ uint32_t bf16x2_mul(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

// Streaming 16-byte global load that does not allocate in L1.
__device__ __forceinline__ uint4 ld_stream_v4(const void *p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// Warp-level tensor-core MMA: D(16x8 f32) += A(16x16 bf16, row) * B(16x8 bf16, col).
__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], uint32_t a0, uint32_t a1,
                                               uint32_t a2, uint32_t a3, uint32_t b0,
                                               uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// (a & MASK) | c as one LOP3 with the mask as its immediate; written out
// because the plain expression with two constants compiles to two
// instructions.
template <uint32_t MASK>
__device__ __forceinline__ uint32_t and_or(uint32_t a, uint32_t c) {
    uint32_t r;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(a), "n"(MASK), "r"(c));
    return r;
}

// Byte permute.
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
    return r;
}

}  // namespace dev
}  // namespace qz
#endif
