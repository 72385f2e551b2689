// qz_api.cu -- the exported C ABI (include/qz.h): argument validation and
// dispatch to the kernels.  Every check runs on the host before any launch.
#include <cuda_runtime.h>

#include <atomic>

#include "qz_internal.cuh"

namespace qz {

static std::atomic<uint64_t> g_wait_limit{0};
constexpr uint64_t kDefaultWaitLimit = 2000000000ull;   // 2 s in nanoseconds

static std::atomic<int32_t> g_launch_overlap{0};

int32_t launch_overlap() { return g_launch_overlap.load(std::memory_order_relaxed); }

uint64_t device_wait_limit() {
    const uint64_t v = g_wait_limit.load(std::memory_order_relaxed);
    return v ? v : kDefaultWaitLimit;
}

int device_sm_count() {
    static DeviceOnce once;
    static int count[kMaxDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return kSmCount;
    }
    const cudaError_t e = once.run(dev, [dev] {
        int n = 0;
        const cudaError_t r = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        if (r == cudaSuccess) count[dev] = n < 1 ? 1 : (n > kSmCount ? kSmCount : n);
        return r;
    });
    return e == cudaSuccess ? count[dev] : kSmCount;
}

namespace {

constexpr int64_t kMaxDim = (int64_t(1) << 31) - 1;
constexpr int64_t kMaxElems = int64_t(1) << 40;

bool format_ok(int32_t bits, int32_t symmetric) {
    return (bits == 4 || bits == 8) && (symmetric == 0 || symmetric == 1);
}

// Shape/format checks shared by quantize_pack and dequantize.
qz_status check_matrix_format(int64_t N, int64_t K, int32_t bits, int32_t symmetric,
                              int64_t g) {
    if (!format_ok(bits, symmetric)) return QZ_ERR_UNSUPPORTED;
    if (N < 1 || K < 1 || N > kMaxDim || K > kMaxDim || N * K > kMaxElems)
        return QZ_ERR_INVALID_ARG;
    if (g < 0) return QZ_ERR_INVALID_ARG;
    if (g > 0 && K % g != 0) return QZ_ERR_INVALID_ARG;
    if (K % 8 != 0) return QZ_ERR_UNSUPPORTED;
    if (g > 0 && g % 8 != 0) return QZ_ERR_UNSUPPORTED;
    return QZ_OK;
}

// The integer decode GEMVs take up to 64 tokens; the FP4A16 GEMV up to 16.
constexpr int64_t kGemvMaxM = 64;
constexpr int64_t kFp4GemvMaxM = 16;
// The GEMM entry points hand M <= 32 to the decode kernel: measured on
// 8192 x 8192, it takes 29.0 us (int4) and 31.1 us (int8) at M = 32 against
// the tcgen05 GEMM's 30.3 and 33.0 us, and loses from M = 64 on.
constexpr int64_t kGemmToGemvMaxM = 32;

qz_status check_gemv_shape(int64_t M, int64_t N, int64_t K, int64_t max_m = kGemvMaxM) {
    if (M < 1 || N < 1 || K < 1 || N > kMaxDim || K > kMaxDim) return QZ_ERR_INVALID_ARG;
    if (M > max_m) return QZ_ERR_UNSUPPORTED;
    if (K % 128 != 0) return QZ_ERR_UNSUPPORTED;
    if ((int64_t)N * K > kMaxElems) return QZ_ERR_INVALID_ARG;
    return QZ_OK;
}

qz_status check_workspace(size_t need, const void *ws, size_t ws_bytes) {
    if (need == 0) return QZ_OK;
    if (ws == nullptr || ws_bytes < need) return QZ_ERR_WORKSPACE;
    if (!aligned(ws, 256)) return QZ_ERR_ALIGNMENT;
    return QZ_OK;
}

cudaStream_t as_stream(void *s) { return static_cast<cudaStream_t>(s); }

// W4A4 GEMM shapes: whole 256-wide K stages (one 128-byte row of codes per
// stage, 4 or 2 whole scale atoms).
qz_status check_fp4a4(int64_t M, int64_t N, int64_t K, int32_t kind) {
    if (kind != QZ_FP4_MX && kind != QZ_FP4_NV) return QZ_ERR_UNSUPPORTED;
    if (M < 1 || N < 1 || K < 1 || M > kMaxDim || N > kMaxDim || K > kMaxDim ||
        M * K > kMaxElems || N * K > kMaxElems || M * N > kMaxElems)
        return QZ_ERR_INVALID_ARG;
    if (K % 256 != 0) return QZ_ERR_UNSUPPORTED;
    return QZ_OK;
}

}  // namespace
}  // namespace qz

using namespace qz;

extern "C" {

QZ_API const char *qz_status_string(int status) {
    switch (status) {
    case QZ_OK: return "ok";
    case QZ_ERR_INVALID_ARG: return "invalid argument (null pointer, size or shape)";
    case QZ_ERR_ALIGNMENT: return "pointer not aligned as required";
    case QZ_ERR_UNSUPPORTED: return "format or shape not supported by the kernels";
    case QZ_ERR_WORKSPACE: return "workspace missing or too small";
    case QZ_ERR_CUDA: return "CUDA call or kernel launch failed";
    case QZ_ERR_DEVICE_TIMEOUT: return "a bounded device-side wait ran out";
    default: return "unknown status";
    }
}

QZ_API int qz_version(void) { return 101; }

QZ_API qz_status qz_packed_bytes(int64_t N, int64_t K, int32_t bits, int32_t symmetric,
                                 int64_t group_size, size_t *codes_bytes,
                                 size_t *scales_bytes, size_t *zeros_bytes) {
    if (!codes_bytes || !scales_bytes || !zeros_bytes) return QZ_ERR_INVALID_ARG;
    if (!format_ok(bits, symmetric)) return QZ_ERR_UNSUPPORTED;
    if (N < 1 || K < 1 || group_size < 0) return QZ_ERR_INVALID_ARG;
    if (group_size > 0 && K % group_size != 0) return QZ_ERR_INVALID_ARG;
    if (bits == 4 && K % 2 != 0) return QZ_ERR_INVALID_ARG;
    const int64_t groups = group_size == 0 ? 1 : N * (K / group_size);
    *codes_bytes = (size_t)(bits == 4 ? N * (K / 2) : N * K);
    *scales_bytes = (size_t)groups * 2;
    *zeros_bytes = symmetric ? 0 : (size_t)groups;
    return QZ_OK;
}

QZ_API qz_status qz_workspace_bytes(int32_t op, int64_t M, int64_t N, int64_t K,
                                    int64_t group_size, size_t *bytes) {
    if (!bytes) return QZ_ERR_INVALID_ARG;
    switch (op) {
    case QZ_OP_QUANTIZE_PACK:
        if (group_size < 0) return QZ_ERR_INVALID_ARG;
        *bytes = quantize_workspace_bytes(group_size);
        return QZ_OK;
    case QZ_OP_DEQUANTIZE:
        *bytes = 0;
        return QZ_OK;
    case QZ_OP_W4A16_GEMV:
    case QZ_OP_W8A16_GEMV: {
        const qz_status s = check_gemv_shape(M, N, K);
        if (s != QZ_OK) return s;
        *bytes = op == QZ_OP_W4A16_GEMV
                     ? gemv_workspace_bound(M, N, K, 4, gemv_unit_k(4, M, N, K, group_size))
                     : gemv_workspace_bound(M, N, K, 8);
        return QZ_OK;
    }
    case QZ_OP_W4A16_GEMM:
    case QZ_OP_W8A16_GEMM:
        if (M < 1 || N < 1 || K < 1) return QZ_ERR_INVALID_ARG;
        *bytes = M <= kGemmToGemvMaxM && K % 128 == 0
                     ? (op == QZ_OP_W4A16_GEMM
                            ? gemv_workspace_bound(M, N, K, 4, gemv_unit_k(4, M, N, K, group_size))
                            : gemv_workspace_bound(M, N, K, 8))
                     : gemm_workspace_bytes(M, N, K);
        return QZ_OK;
    case QZ_OP_FP4A16_GEMV: {
        const qz_status s = check_gemv_shape(M, N, K, kFp4GemvMaxM);
        if (s != QZ_OK) return s;
        // 256-wide units when K % 512 == 0 (and the block scales are
        // 16-byte aligned; 128-wide otherwise): the bound covers both
        *bytes = gemv_workspace_bound(M, N, K, 4, K % 512 == 0 ? 256 : 128);
        return QZ_OK;
    }
    case QZ_OP_GPTQ:
        if (N < 1 || K < 1 || N > kMaxDim || K > kMaxDim) return QZ_ERR_INVALID_ARG;
        *bytes = gptq_workspace_bytes(N, K);
        return QZ_OK;
    case QZ_OP_FP4A4_GEMM: {
        const qz_status s = check_fp4a4(M, N, K, QZ_FP4_NV);
        if (s != QZ_OK) return s;
        *bytes = fp4a4_workspace_bytes(M, K);
        return QZ_OK;
    }
    default:
        return QZ_ERR_INVALID_ARG;
    }
}

QZ_API qz_status qz_workspace_bytes_for_sms(int32_t op, int64_t M, int64_t N, int64_t K,
                                            int64_t group_size, int32_t sms, size_t *bytes) {
    if (!bytes || sms < 1 || sms > kSmCount) return QZ_ERR_INVALID_ARG;
    switch (op) {
    case QZ_OP_W4A16_GEMV:
    case QZ_OP_W8A16_GEMV: {
        const qz_status s = check_gemv_shape(M, N, K);
        if (s != QZ_OK) return s;
        *bytes = op == QZ_OP_W4A16_GEMV
                     ? gemv_plan(M, N, K, 4, sms, gemv_unit_k(4, M, N, K, group_size)).total_bytes
                     : gemv_plan(M, N, K, 8, sms).total_bytes;
        return QZ_OK;
    }
    case QZ_OP_W4A16_GEMM:
    case QZ_OP_W8A16_GEMM:
        if (M < 1 || N < 1 || K < 1) return QZ_ERR_INVALID_ARG;
        *bytes = M <= kGemmToGemvMaxM && K % 128 == 0
                     ? (op == QZ_OP_W4A16_GEMM
                            ? gemv_plan(M, N, K, 4, sms, gemv_unit_k(4, M, N, K, group_size))
                            : gemv_plan(M, N, K, 8, sms)).total_bytes
                     : gemm_workspace_bytes_for(M, N, K, sms);
        return QZ_OK;
    case QZ_OP_FP4A16_GEMV: {
        const qz_status s = check_gemv_shape(M, N, K, kFp4GemvMaxM);
        if (s != QZ_OK) return s;
        *bytes = gemv_plan(M, N, K, 4, sms, K % 512 == 0 ? 256 : 128).total_bytes;
        return QZ_OK;
    }
    default:
        return qz_workspace_bytes(op, M, N, K, group_size, bytes);
    }
}

QZ_API qz_status qz_quantize_pack(const void *w, int64_t N, int64_t K, int32_t bits,
                                  int32_t symmetric, int64_t group_size, void *codes,
                                  void *scales, void *zeros, void *workspace,
                                  size_t workspace_bytes, void *stream) {
    qz_status s = check_matrix_format(N, K, bits, symmetric, group_size);
    if (s != QZ_OK) return s;
    if (!w || !codes || !scales) return QZ_ERR_INVALID_ARG;
    if (symmetric ? (zeros != nullptr) : (zeros == nullptr)) return QZ_ERR_INVALID_ARG;
    if (!aligned(w, 16) || !aligned(codes, 16) || !aligned(scales, 2)) return QZ_ERR_ALIGNMENT;
    s = check_workspace(quantize_workspace_bytes(group_size), workspace, workspace_bytes);
    if (s != QZ_OK) return s;
    return launch_quantize_pack(w, N, K, bits, symmetric, group_size, codes, scales, zeros,
                                workspace, as_stream(stream));
}

QZ_API qz_status qz_dequantize(const void *codes, const void *scales, const void *zeros,
                               int64_t N, int64_t K, int32_t bits, int32_t symmetric,
                               int64_t group_size, void *w_hat, void *stream) {
    const qz_status s = check_matrix_format(N, K, bits, symmetric, group_size);
    if (s != QZ_OK) return s;
    if (!codes || !scales || !w_hat) return QZ_ERR_INVALID_ARG;
    if (symmetric ? (zeros != nullptr) : (zeros == nullptr)) return QZ_ERR_INVALID_ARG;
    if (!aligned(codes, 16) || !aligned(w_hat, 16) || !aligned(scales, 2)) return QZ_ERR_ALIGNMENT;
    return launch_dequantize(codes, scales, zeros, N, K, bits, symmetric, group_size, w_hat,
                             as_stream(stream));
}

QZ_API qz_status qz_w4a16_gemv(const void *a, const void *codes, const void *scales,
                               const void *zeros, int64_t M, int64_t N, int64_t K,
                               int64_t group_size, void *y, void *workspace,
                               size_t workspace_bytes, void *stream) {
    qz_status s = check_gemv_shape(M, N, K);
    if (s != QZ_OK) return s;
    if (group_size < 32 || group_size % 32 != 0 || K % group_size != 0)
        return group_size <= 0 || K % group_size != 0 ? QZ_ERR_INVALID_ARG : QZ_ERR_UNSUPPORTED;
    if (!a || !codes || !scales || !zeros || !y) return QZ_ERR_INVALID_ARG;
    if (!aligned(a, 16) || !aligned(codes, 16) || !aligned(scales, 2) || !aligned(y, 2))
        return QZ_ERR_ALIGNMENT;
    const GemvPlan plan =
        gemv_plan(M, N, K, 4, device_sm_count(), gemv_unit_k(4, M, N, K, group_size, scales, zeros));
    s = check_workspace(plan.total_bytes, workspace, workspace_bytes);
    if (s != QZ_OK) return s;
    return launch_w4a16_gemv(a, codes, scales, zeros, M, N, K, group_size, y, workspace, plan,
                             launch_overlap(), as_stream(stream));
}

QZ_API qz_status qz_w8a16_gemv(const void *a, const void *codes, const void *scales,
                               int64_t M, int64_t N, int64_t K, void *y, void *workspace,
                               size_t workspace_bytes, void *stream) {
    qz_status s = check_gemv_shape(M, N, K);
    if (s != QZ_OK) return s;
    if (!a || !codes || !scales || !y) return QZ_ERR_INVALID_ARG;
    if (!aligned(a, 16) || !aligned(codes, 16) || !aligned(scales, 2) || !aligned(y, 2))
        return QZ_ERR_ALIGNMENT;
    const GemvPlan plan = gemv_plan(M, N, K, 8, device_sm_count());
    s = check_workspace(plan.total_bytes, workspace, workspace_bytes);
    if (s != QZ_OK) return s;
    return launch_w8a16_gemv(a, codes, scales, M, N, K, y, workspace, plan, launch_overlap(),
                             as_stream(stream));
}

QZ_API qz_status qz_w4a16_gemm(const void *a, const void *codes, const void *scales,
                               const void *zeros, int64_t M, int64_t N, int64_t K,
                               int64_t group_size, void *y, void *workspace,
                               size_t workspace_bytes, void *stream) {
    if (M < 1 || N < 1 || K < 1 || M > kMaxDim || N > kMaxDim || K > kMaxDim)
        return QZ_ERR_INVALID_ARG;
    if (K % 128 != 0) return QZ_ERR_UNSUPPORTED;
    if (group_size <= 0 || K % group_size != 0) return QZ_ERR_INVALID_ARG;
    if (!a || !codes || !scales || !zeros || !y) return QZ_ERR_INVALID_ARG;
    if (M <= kGemmToGemvMaxM)   // the decode kernel covers small M with the same arithmetic
        return qz_w4a16_gemv(a, codes, scales, zeros, M, N, K, group_size, y, workspace,
                             workspace_bytes, stream);
    if (group_size % 64 != 0) return QZ_ERR_UNSUPPORTED;
    if (!aligned(a, 16) || !aligned(codes, 16) || !aligned(scales, 2) || !aligned(y, 16))
        return QZ_ERR_ALIGNMENT;
    const qz_status s = check_workspace(gemm_workspace_bytes(M, N, K), workspace, workspace_bytes);
    if (s != QZ_OK) return s;
    return launch_w4a16_gemm(a, codes, scales, zeros, M, N, K, group_size, y, workspace,
                             as_stream(stream));
}

QZ_API qz_status qz_w8a16_gemm(const void *a, const void *codes, const void *scales,
                               int64_t M, int64_t N, int64_t K, void *y, void *workspace,
                               size_t workspace_bytes, void *stream) {
    if (M < 1 || N < 1 || K < 1 || M > kMaxDim || N > kMaxDim || K > kMaxDim)
        return QZ_ERR_INVALID_ARG;
    if (K % 128 != 0) return QZ_ERR_UNSUPPORTED;
    if (!a || !codes || !scales || !y) return QZ_ERR_INVALID_ARG;
    if (M <= kGemmToGemvMaxM)   // the decode kernel covers small M with the same arithmetic
        return qz_w8a16_gemv(a, codes, scales, M, N, K, y, workspace, workspace_bytes, stream);
    if (!aligned(a, 16) || !aligned(codes, 16) || !aligned(scales, 2) || !aligned(y, 16))
        return QZ_ERR_ALIGNMENT;
    const qz_status s = check_workspace(gemm_workspace_bytes(M, N, K), workspace, workspace_bytes);
    if (s != QZ_OK) return s;
    return launch_w8a16_gemm(a, codes, scales, M, N, K, y, workspace, as_stream(stream));
}

QZ_API qz_status qz_gptq_quantize(const void *w, const void *x, int64_t N, int64_t K,
                                  int64_t n_samples, int32_t bits, int32_t symmetric,
                                  int64_t group_size, double damp, void *codes, void *scales,
                                  void *zeros, void *workspace, size_t workspace_bytes,
                                  void *stream) {
    if (!format_ok(bits, symmetric)) return QZ_ERR_UNSUPPORTED;
    if (N < 1 || K < 1 || N > kMaxDim || K > kMaxDim || n_samples < 1) return QZ_ERR_INVALID_ARG;
    if (N * K > kMaxElems || n_samples * K > kMaxElems) return QZ_ERR_INVALID_ARG;
    if (!(damp >= 0.0) || !(damp < 1e300)) return QZ_ERR_INVALID_ARG;
    if (group_size <= 0 || K % group_size != 0) return QZ_ERR_INVALID_ARG;
    if (K % 8 != 0 || group_size % 32 != 0 || (group_size % 128 != 0 && 128 % group_size != 0))
        return QZ_ERR_UNSUPPORTED;
    if (!w || !x || !codes || !scales) return QZ_ERR_INVALID_ARG;
    if (symmetric ? (zeros != nullptr) : (zeros == nullptr)) return QZ_ERR_INVALID_ARG;
    if (!aligned(w, 2) || !aligned(x, 2) || !aligned(scales, 2)) return QZ_ERR_ALIGNMENT;
    const qz_status s = check_workspace(gptq_workspace_bytes(N, K), workspace, workspace_bytes);
    if (s != QZ_OK) return s;
    return launch_gptq(w, x, N, K, n_samples, bits, symmetric, group_size, damp, codes, scales,
                       zeros, workspace, as_stream(stream));
}

QZ_API qz_status qz_fp4_packed_bytes(int64_t N, int64_t K, int32_t kind, size_t *codes_bytes,
                                     size_t *scales_bytes) {
    if (!codes_bytes || !scales_bytes) return QZ_ERR_INVALID_ARG;
    if (kind != QZ_FP4_MX && kind != QZ_FP4_NV) return QZ_ERR_UNSUPPORTED;
    if (N < 1 || K < 1 || K % fp4_block_size(kind) != 0) return QZ_ERR_INVALID_ARG;
    *codes_bytes = (size_t)(N * (K / 2));
    *scales_bytes = (size_t)(N * (K / fp4_block_size(kind)));
    return QZ_OK;
}

namespace {
qz_status check_fp4(int64_t N, int64_t K, int32_t kind) {
    if (kind != QZ_FP4_MX && kind != QZ_FP4_NV) return QZ_ERR_UNSUPPORTED;
    if (N < 1 || K < 1 || N > kMaxDim || K > kMaxDim || N * K > kMaxElems)
        return QZ_ERR_INVALID_ARG;
    if (K % fp4_block_size(kind) != 0) return QZ_ERR_INVALID_ARG;
    return QZ_OK;
}
}  // namespace

QZ_API qz_status qz_fp4_quantize(const void *w, int64_t N, int64_t K, int32_t kind, void *codes,
                                 void *block_scales, void *tensor_scale, void *stream) {
    const qz_status s = check_fp4(N, K, kind);
    if (s != QZ_OK) return s;
    if (!w || !codes || !block_scales) return QZ_ERR_INVALID_ARG;
    if (kind == QZ_FP4_NV ? tensor_scale == nullptr : tensor_scale != nullptr)
        return QZ_ERR_INVALID_ARG;
    if (!aligned(w, 16) || !aligned(codes, 16) || (tensor_scale && !aligned(tensor_scale, 4)))
        return QZ_ERR_ALIGNMENT;
    return launch_fp4_quantize(w, N, K, kind, codes, block_scales, tensor_scale,
                               as_stream(stream));
}

QZ_API qz_status qz_fp4_dequantize(const void *codes, const void *block_scales,
                                   const void *tensor_scale, int64_t N, int64_t K, int32_t kind,
                                   void *w_hat, void *stream) {
    const qz_status s = check_fp4(N, K, kind);
    if (s != QZ_OK) return s;
    if (!codes || !block_scales || !w_hat) return QZ_ERR_INVALID_ARG;
    if (kind == QZ_FP4_NV ? tensor_scale == nullptr : tensor_scale != nullptr)
        return QZ_ERR_INVALID_ARG;
    if (!aligned(codes, 4) || !aligned(w_hat, 16) || (tensor_scale && !aligned(tensor_scale, 4)))
        return QZ_ERR_ALIGNMENT;
    return launch_fp4_dequantize(codes, block_scales, tensor_scale, N, K, kind, w_hat,
                                 as_stream(stream));
}

QZ_API qz_status qz_fp4a16_gemv(const void *a, const void *codes, const void *block_scales,
                                const void *tensor_scale, int64_t M, int64_t N, int64_t K,
                                int32_t kind, void *y, void *workspace, size_t workspace_bytes,
                                void *stream) {
    qz_status s = check_gemv_shape(M, N, K, kFp4GemvMaxM);
    if (s != QZ_OK) return s;
    s = check_fp4(N, K, kind);
    if (s != QZ_OK) return s;
    if (!a || !codes || !block_scales || !y) return QZ_ERR_INVALID_ARG;
    if (kind == QZ_FP4_NV ? tensor_scale == nullptr : tensor_scale != nullptr)
        return QZ_ERR_INVALID_ARG;
    if (!aligned(a, 16) || !aligned(codes, 16) || !aligned(y, 2) ||
        (tensor_scale && !aligned(tensor_scale, 4)))
        return QZ_ERR_ALIGNMENT;
    const GemvPlan plan =
        gemv_plan(M, N, K, 4, device_sm_count(), gemv_fp4_unit_k(M, K, block_scales));
    s = check_workspace(plan.total_bytes, workspace, workspace_bytes);
    if (s != QZ_OK) return s;
    return launch_fp4a16_gemv(a, codes, block_scales, tensor_scale, M, N, K, kind, y, workspace,
                              plan, launch_overlap(), as_stream(stream));
}

QZ_API void qz_set_device_wait_limit(uint64_t limit) {
    g_wait_limit.store(limit, std::memory_order_relaxed);
}

QZ_API qz_status qz_set_launch_overlap(int32_t mode) {
    if (mode < 0 || mode > 1) return QZ_ERR_INVALID_ARG;
    g_launch_overlap.store(mode, std::memory_order_relaxed);
    return QZ_OK;
}

QZ_API qz_status qz_fp4_mma_scale_bytes(int64_t rows, int64_t K, int32_t kind, size_t *bytes) {
    if (!bytes) return QZ_ERR_INVALID_ARG;
    const qz_status s = check_fp4a4(rows, 1, K, kind);
    if (s != QZ_OK) return s;
    *bytes = fp4_mma_scale_bytes(rows, K, kind);
    return QZ_OK;
}

QZ_API qz_status qz_fp4_scales_to_mma(const void *block_scales, int64_t rows, int64_t K,
                                      int32_t kind, void *scales_mma, void *stream) {
    const qz_status s = check_fp4a4(rows, 1, K, kind);
    if (s != QZ_OK) return s;
    if (!block_scales || !scales_mma) return QZ_ERR_INVALID_ARG;
    if (!aligned(block_scales, 4) || !aligned(scales_mma, 16)) return QZ_ERR_ALIGNMENT;
    return launch_fp4_scales_to_mma(block_scales, rows, K, kind, scales_mma, as_stream(stream));
}

QZ_API qz_status qz_fp4a4_gemm(const void *a, const void *codes, const void *scales_mma,
                               const void *tensor_scale, int64_t M, int64_t N, int64_t K,
                               int32_t kind, void *y, void *workspace, size_t workspace_bytes,
                               void *stream) {
    qz_status s = check_fp4a4(M, N, K, kind);
    if (s != QZ_OK) return s;
    if (!a || !codes || !scales_mma || !y) return QZ_ERR_INVALID_ARG;
    if (kind == QZ_FP4_NV ? tensor_scale == nullptr : tensor_scale != nullptr)
        return QZ_ERR_INVALID_ARG;
    if (!aligned(a, 16) || !aligned(codes, 16) || !aligned(scales_mma, 16) || !aligned(y, 2) ||
        (tensor_scale && !aligned(tensor_scale, 4)))
        return QZ_ERR_ALIGNMENT;
    s = check_workspace(fp4a4_workspace_bytes(M, K), workspace, workspace_bytes);
    if (s != QZ_OK) return s;
    return launch_fp4a4_gemm(a, codes, scales_mma, tensor_scale, M, N, K, kind, y, workspace,
                             as_stream(stream));
}

}  // extern "C"
