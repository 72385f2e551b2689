// qz_gemv_noalloc.cu -- qz_w4a16_gemv_noalloc: the W4A16 decode GEMV for
// callers that cannot allocate device memory.
//
// Some callers have no way to call cudaMalloc on their path: a plugin running
// inside a host application that owns all device memory and exposes no
// allocator, or latency-critical code where an allocation (which may
// synchronize the device and takes unbounded time) is not acceptable.  Such a
// caller cannot provide the split-K workspace that qz_w4a16_gemv needs.  This
// entry point runs the same kernel with its scratch in a fixed-size array
// that is part of the library image itself.
//
// The array is a file-scope __device__ variable: every GPU that loads this
// library holds kScratchBytes for it until the process exits.  In host code
// its name is only a host-side stand-in, so the device address is looked up
// once per device (cudaGetSymbolAddress, with that device current) and passed
// to the kernel.  All calls share the array: calls whose work overlaps on the
// GPU race on it and must not be issued concurrently.
#include <cuda_runtime.h>

#include "qz_internal.cuh"

namespace qz {
namespace {

constexpr size_t kScratchBytes = QZ_GEMV_NOALLOC_SCRATCH_BYTES;

static __device__ __align__(256) unsigned char g_gemv_scratch[kScratchBytes];

DeviceOnce g_scratch_once;
void *g_scratch_ptr[kMaxDevices];

// Device address of the scratch array on the current device, looked up with
// that device current on the first call that succeeds for it (a failed
// look-up is retried by the next call).
qz_status scratch_address(void **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return QZ_ERR_CUDA;
    }
    if (dev < 0 || dev >= kMaxDevices) return QZ_ERR_UNSUPPORTED;
    const cudaError_t e = g_scratch_once.run(dev, [dev] {
        return cudaGetSymbolAddress(&g_scratch_ptr[dev], g_gemv_scratch);
    });
    if (e != cudaSuccess || g_scratch_ptr[dev] == nullptr) return QZ_ERR_CUDA;
    *out = g_scratch_ptr[dev];
    return QZ_OK;
}

bool is_aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

}  // namespace
}  // namespace qz

extern "C" QZ_API qz_status qz_w4a16_gemv_noalloc(const void *a, const void *codes,
                                                  const void *scales, const void *zeros,
                                                  int64_t M, int64_t N, int64_t K,
                                                  int64_t group_size, void *y, void *stream) {
    constexpr int64_t kMaxDim = (int64_t(1) << 31) - 1;
    if (M < 1 || N < 1 || K < 1 || N > kMaxDim || K > kMaxDim) return QZ_ERR_INVALID_ARG;
    if (M > 16 || K % 128 != 0) return QZ_ERR_UNSUPPORTED;
    if (N * K > (int64_t(1) << 40)) return QZ_ERR_INVALID_ARG;
    if (group_size <= 0 || K % group_size != 0) return QZ_ERR_INVALID_ARG;
    if (group_size % 32 != 0) return QZ_ERR_UNSUPPORTED;
    if (!a || !codes || !scales || !zeros || !y) return QZ_ERR_INVALID_ARG;
    if (!qz::is_aligned(a, 16) || !qz::is_aligned(codes, 16) || !qz::is_aligned(scales, 2) ||
        !qz::is_aligned(y, 2))
        return QZ_ERR_ALIGNMENT;
    const qz::GemvPlan plan = qz::gemv_plan(M, N, K, 4, qz::device_sm_count(),
                                            qz::gemv_unit_k(4, M, N, K, group_size, scales, zeros));
    if (plan.total_bytes > qz::kScratchBytes) return QZ_ERR_WORKSPACE;   // beyond the built-in maximum
    void *scratch = nullptr;
    if (plan.total_bytes > 0) {
        const qz_status s = qz::scratch_address(&scratch);
        if (s != QZ_OK) return s;
        // the split-K counters must start at zero; the partials are fully
        // overwritten before they are read
        if (cudaMemsetAsync(static_cast<char *>(scratch) + plan.partial_bytes, 0,
                            plan.counter_bytes, static_cast<cudaStream_t>(stream)) != cudaSuccess)
            return QZ_ERR_CUDA;
    }
    // plain stream order: the counter reset above is not a kernel, so a
    // programmatic dependency on it would not be ordered
    return qz::launch_w4a16_gemv(a, codes, scales, zeros, M, N, K, group_size, y, scratch, plan,
                                 0, static_cast<cudaStream_t>(stream));
}
