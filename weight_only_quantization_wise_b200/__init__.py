"""Python binding of libqz.so, the B200 weight-only quantization library.

Argument marshalling only: every function below validates Python-side types,
allocates outputs with PyTorch when the caller did not pass them, and calls
the C entry point of the same name (declared in ``include/qz.h``) on the
``stream`` argument, else the current CUDA stream; outputs and temporary
workspaces are allocated on that same stream.  All arithmetic runs in the
library's CUDA kernels; there is no CPU or PyTorch fallback.  If ``libqz.so``
is missing the import fails.
"""
import contextlib
import ctypes
import os

import torch

__all__ = [
    "QzError", "lib", "qz_version", "qz_status_string", "qz_packed_bytes",
    "qz_workspace_bytes", "qz_workspace_bytes_for_sms", "qz_quantize_pack", "qz_dequantize",
    "qz_w4a16_gemv",
    "qz_w4a16_gemm", "qz_w8a16_gemv", "qz_w8a16_gemm", "qz_set_device_wait_limit",
    "qz_set_launch_overlap", "qz_device_status", "qz_gptq_quantize", "QZ_OP_GPTQ",
    "qz_fp4_packed_bytes", "qz_fp4_quantize", "qz_fp4_dequantize", "qz_fp4a16_gemv",
    "QZ_OP_FP4A16_GEMV", "QZ_FP4_MX", "QZ_FP4_NV", "qz_fp4_mma_scale_bytes",
    "qz_fp4_scales_to_mma", "qz_fp4a4_gemm", "QZ_OP_FP4A4_GEMM",
    "Workspace", "QZ_OP_QUANTIZE_PACK", "QZ_OP_DEQUANTIZE", "QZ_OP_W4A16_GEMV",
    "QZ_OP_W4A16_GEMM", "QZ_OP_W8A16_GEMV", "QZ_OP_W8A16_GEMM", "EXPORTED_SYMBOLS",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libqz.so")

QZ_OK = 0
QZ_ERR_DEVICE_TIMEOUT = 6
(QZ_OP_QUANTIZE_PACK, QZ_OP_DEQUANTIZE, QZ_OP_W4A16_GEMV, QZ_OP_W4A16_GEMM, QZ_OP_W8A16_GEMV,
 QZ_OP_W8A16_GEMM, QZ_OP_GPTQ, QZ_OP_FP4A16_GEMV, QZ_OP_FP4A4_GEMM) = range(9)
QZ_FP4_MX, QZ_FP4_NV = 0, 1
FP4_BLOCK = {QZ_FP4_MX: 32, QZ_FP4_NV: 16}

_i32, _i64, _sz, _p = ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t, ctypes.c_void_p
_SIGS = {
    "qz_status_string": ([ctypes.c_int], ctypes.c_char_p),
    "qz_version": ([], ctypes.c_int),
    "qz_packed_bytes": ([_i64, _i64, _i32, _i32, _i64, ctypes.POINTER(_sz),
                         ctypes.POINTER(_sz), ctypes.POINTER(_sz)], ctypes.c_int),
    "qz_workspace_bytes": ([_i32, _i64, _i64, _i64, _i64, ctypes.POINTER(_sz)], ctypes.c_int),
    "qz_workspace_bytes_for_sms": ([_i32, _i64, _i64, _i64, _i64, _i32, ctypes.POINTER(_sz)],
                                   ctypes.c_int),
    "qz_quantize_pack": ([_p, _i64, _i64, _i32, _i32, _i64, _p, _p, _p, _p, _sz, _p], ctypes.c_int),
    "qz_dequantize": ([_p, _p, _p, _i64, _i64, _i32, _i32, _i64, _p, _p], ctypes.c_int),
    "qz_w4a16_gemv": ([_p, _p, _p, _p, _i64, _i64, _i64, _i64, _p, _p, _sz, _p], ctypes.c_int),
    "qz_w4a16_gemm": ([_p, _p, _p, _p, _i64, _i64, _i64, _i64, _p, _p, _sz, _p], ctypes.c_int),
    "qz_w8a16_gemv": ([_p, _p, _p, _i64, _i64, _i64, _p, _p, _sz, _p], ctypes.c_int),
    "qz_w8a16_gemm": ([_p, _p, _p, _i64, _i64, _i64, _p, _p, _sz, _p], ctypes.c_int),
    "qz_w4a16_gemv_noalloc": ([_p, _p, _p, _p, _i64, _i64, _i64, _i64, _p, _p], ctypes.c_int),
    "qz_gptq_quantize": ([_p, _p, _i64, _i64, _i64, _i32, _i32, _i64, ctypes.c_double, _p, _p, _p,
                          _p, _sz, _p], ctypes.c_int),
    "qz_fp4_packed_bytes": ([_i64, _i64, _i32, ctypes.POINTER(_sz), ctypes.POINTER(_sz)],
                            ctypes.c_int),
    "qz_fp4_quantize": ([_p, _i64, _i64, _i32, _p, _p, _p, _p], ctypes.c_int),
    "qz_fp4_dequantize": ([_p, _p, _p, _i64, _i64, _i32, _p, _p], ctypes.c_int),
    "qz_fp4a16_gemv": ([_p, _p, _p, _p, _i64, _i64, _i64, _i32, _p, _p, _sz, _p], ctypes.c_int),
    "qz_fp4_mma_scale_bytes": ([_i64, _i64, _i32, ctypes.POINTER(_sz)], ctypes.c_int),
    "qz_fp4_scales_to_mma": ([_p, _i64, _i64, _i32, _p, _p], ctypes.c_int),
    "qz_fp4a4_gemm": ([_p, _p, _p, _p, _i64, _i64, _i64, _i32, _p, _p, _sz, _p], ctypes.c_int),
    "qz_set_device_wait_limit": ([ctypes.c_uint64], None),
    "qz_set_launch_overlap": ([ctypes.c_int32], ctypes.c_int),
    "qz_device_status": ([], ctypes.c_int),
}
EXPORTED_SYMBOLS = tuple(_SIGS)

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is not built; run `python weight_only_quantization_wise_b200/build.py` "
        "(there is no fallback implementation)")

lib = ctypes.CDLL(LIB_PATH)
for _name, (_args, _res) in _SIGS.items():
    _f = getattr(lib, _name)
    _f.argtypes = _args
    _f.restype = _res


class QzError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {qz_status_string(status)} (status {status})")


def _check(status: int, where: str) -> None:
    if status != QZ_OK:
        raise QzError(status, where)


def qz_status_string(status: int) -> str:
    return lib.qz_status_string(int(status)).decode()


def qz_version() -> int:
    return int(lib.qz_version())


def qz_packed_bytes(N, K, bits=4, symmetric=False, group_size=128):
    c, s, z = _sz(), _sz(), _sz()
    _check(lib.qz_packed_bytes(N, K, bits, int(symmetric), group_size, ctypes.byref(c),
                               ctypes.byref(s), ctypes.byref(z)), "qz_packed_bytes")
    return c.value, s.value, z.value


_WS_SIZES = {}


def qz_workspace_bytes(op, M, N, K, group_size=128) -> int:
    """Workspace bytes of a call (a pure function of the arguments; cached)."""
    key = (int(op), int(M), int(N), int(K), int(group_size))
    v = _WS_SIZES.get(key)
    if v is None:
        b = _sz()
        _check(lib.qz_workspace_bytes(*key, ctypes.byref(b)), "qz_workspace_bytes")
        v = _WS_SIZES[key] = b.value
    return v


def qz_workspace_bytes_for_sms(op, M, N, K, group_size, sms) -> int:
    """Workspace bytes of a call whose grid is sized for `sms` SMs."""
    b = _sz()
    _check(lib.qz_workspace_bytes_for_sms(int(op), int(M), int(N), int(K), int(group_size),
                                          int(sms), ctypes.byref(b)), "qz_workspace_bytes_for_sms")
    return b.value


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensors must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _launch_stream(stream, device):
    """The torch stream a call runs on: `stream`, else the current stream."""
    return torch.cuda.current_stream(device) if stream is None else stream


def _on(stream):
    """Context that makes an explicitly passed stream current for the call's
    allocations (nothing to do when the call runs on the current stream)."""
    return contextlib.nullcontext() if stream is None else torch.cuda.stream(stream)


def _handle(stream):
    return ctypes.c_void_p(stream.cuda_stream)


class Workspace:
    """A zero-filled device workspace that grows on demand.

    Each call leaves the counters in its workspace at zero again (the rest is
    scratch that every call writes before it reads), so one buffer serves
    every call issued on one stream.  Calls that may run
    concurrently need separate Workspace objects.
    """

    def __init__(self, device=None):
        self.device = torch.device(device if device is not None else "cuda")
        self.buf = None

    def get(self, nbytes: int):
        if nbytes == 0:
            return None
        if self.buf is None or self.buf.numel() < nbytes:
            self.buf = torch.zeros(max(nbytes, 256), dtype=torch.uint8, device=self.device)
        return self.buf

    def get_scratch(self, nbytes: int):
        """A second buffer for calls whose workspace is plain scratch (the
        W4A4 GEMM's quantized activations): it is not zero-filled and must
        not be the one the split-K calls count on."""
        if getattr(self, "scratch", None) is None or self.scratch.numel() < nbytes:
            self.scratch = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=self.device)
        return self.scratch


def _ws_args(workspace, nbytes, device):
    """Pointer and size of the call's workspace.  Called inside
    ``torch.cuda.stream(launch stream)``: a temporary workspace is then
    allocated and zero-filled on the stream the kernel runs on, so the fill
    is ordered before the kernel and the caching allocator hands the memory
    out again only to work queued after it on that stream."""
    if nbytes == 0:
        return None, 0
    if workspace is None:
        workspace = Workspace(device).get(nbytes)
    elif isinstance(workspace, Workspace):
        workspace = workspace.get(nbytes)
    return _ptr(workspace), workspace.numel() * workspace.element_size()


def qz_quantize_pack(w, bits=4, symmetric=False, group_size=128, codes=None, scales=None,
                     zeros=None, workspace=None, stream=None):
    """Quantize an N x K bf16 matrix; returns (codes uint8, scales bf16, zeros uint8 | None)."""
    if w.dtype != torch.bfloat16 or w.dim() != 2:
        raise ValueError("w must be a 2-D bf16 tensor")
    N, K = w.shape
    qz_packed_bytes(N, K, bits, symmetric, group_size)      # validates the format
    dev = w.device
    st = _launch_stream(stream, dev)
    with _on(stream):
        if codes is None:
            codes = torch.empty((N, K // 2) if bits == 4 else (N, K), dtype=torch.uint8,
                                device=dev)
        if scales is None:
            shape = (1,) if group_size == 0 else (N, K // group_size)
            scales = torch.empty(shape, dtype=torch.bfloat16, device=dev)
        if zeros is None and not symmetric:
            shape = (1,) if group_size == 0 else (N, K // group_size)
            zeros = torch.empty(shape, dtype=torch.uint8, device=dev)
        ws_ptr, ws_bytes = _ws_args(workspace, qz_workspace_bytes(QZ_OP_QUANTIZE_PACK, 1, N, K,
                                                                  group_size), dev)
        _check(lib.qz_quantize_pack(_ptr(w), N, K, bits, int(symmetric), group_size,
                                    _ptr(codes), _ptr(scales),
                                    _ptr(zeros) if not symmetric else None, ws_ptr, ws_bytes,
                                    _handle(st)), "qz_quantize_pack")
    return codes, scales, (None if symmetric else zeros)


def qz_dequantize(codes, scales, zeros, N, K, bits=4, symmetric=False, group_size=128,
                  out=None, stream=None):
    """w_hat = bf16(S * (q - Z)) as an N x K bf16 tensor."""
    dev = codes.device
    st = _launch_stream(stream, dev)
    with _on(stream):
        if out is None:
            out = torch.empty((N, K), dtype=torch.bfloat16, device=dev)
        _check(lib.qz_dequantize(_ptr(codes), _ptr(scales), _ptr(zeros), N, K, bits,
                                 int(symmetric), group_size, _ptr(out), _handle(st)),
               "qz_dequantize")
    return out


def _matmul_out(a, N, y):
    if a.dtype != torch.bfloat16 or a.dim() != 2:
        raise ValueError("a must be a 2-D bf16 tensor")
    if y is None:
        y = torch.empty((a.shape[0], N), dtype=torch.bfloat16, device=a.device)
    return y


def qz_w4a16_gemv(a, codes, scales, zeros, N, K, group_size=128, y=None, workspace=None,
                  stream=None):
    """y = a * w_hat^T for int4 asymmetric group-wise weights, M <= 16."""
    st = _launch_stream(stream, a.device)
    M = a.shape[0]
    with _on(stream):
        y = _matmul_out(a, N, y)
        nbytes = qz_workspace_bytes(QZ_OP_W4A16_GEMV, M, N, K, group_size)
        ws_ptr, ws_bytes = _ws_args(workspace, nbytes, a.device)
        _check(lib.qz_w4a16_gemv(_ptr(a), _ptr(codes), _ptr(scales), _ptr(zeros), M, N, K,
                                 group_size, _ptr(y), ws_ptr, ws_bytes, _handle(st)),
               "qz_w4a16_gemv")
    return y


def qz_w4a16_gemm(a, codes, scales, zeros, N, K, group_size=128, y=None, workspace=None,
                  stream=None):
    """y = a * w_hat^T for int4 asymmetric group-wise weights, any M."""
    st = _launch_stream(stream, a.device)
    M = a.shape[0]
    with _on(stream):
        y = _matmul_out(a, N, y)
        nbytes = qz_workspace_bytes(QZ_OP_W4A16_GEMM, M, N, K, group_size)
        ws_ptr, ws_bytes = _ws_args(workspace, nbytes, a.device)
        _check(lib.qz_w4a16_gemm(_ptr(a), _ptr(codes), _ptr(scales), _ptr(zeros), M, N, K,
                                 group_size, _ptr(y), ws_ptr, ws_bytes, _handle(st)),
               "qz_w4a16_gemm")
    return y


def qz_w8a16_gemv(a, codes, scales, N, K, y=None, workspace=None, stream=None):
    """y = a * w_hat^T for int8 symmetric per-channel weights, M <= 16."""
    st = _launch_stream(stream, a.device)
    M = a.shape[0]
    with _on(stream):
        y = _matmul_out(a, N, y)
        nbytes = qz_workspace_bytes(QZ_OP_W8A16_GEMV, M, N, K, K)
        ws_ptr, ws_bytes = _ws_args(workspace, nbytes, a.device)
        _check(lib.qz_w8a16_gemv(_ptr(a), _ptr(codes), _ptr(scales), M, N, K, _ptr(y),
                                 ws_ptr, ws_bytes, _handle(st)), "qz_w8a16_gemv")
    return y


def qz_w8a16_gemm(a, codes, scales, N, K, y=None, workspace=None, stream=None):
    """y = a * w_hat^T for int8 symmetric per-channel weights, any M."""
    st = _launch_stream(stream, a.device)
    M = a.shape[0]
    with _on(stream):
        y = _matmul_out(a, N, y)
        nbytes = qz_workspace_bytes(QZ_OP_W8A16_GEMM, M, N, K, K)
        ws_ptr, ws_bytes = _ws_args(workspace, nbytes, a.device)
        _check(lib.qz_w8a16_gemm(_ptr(a), _ptr(codes), _ptr(scales), M, N, K, _ptr(y),
                                 ws_ptr, ws_bytes, _handle(st)), "qz_w8a16_gemm")
    return y


def qz_gptq_quantize(w, x, bits=4, symmetric=False, group_size=128, damp=0.01, codes=None,
                     scales=None, zeros=None, workspace=None, stream=None):
    """GPTQ of one layer: ``w`` (N x K bf16) with calibration samples ``x``
    (n x K bf16); returns (codes, scales, zeros | None) in the packed format
    of :func:`qz_quantize_pack`."""
    if w.dtype != torch.bfloat16 or w.dim() != 2 or x.dtype != torch.bfloat16 or x.dim() != 2:
        raise ValueError("w and x must be 2-D bf16 tensors")
    N, K = w.shape
    if x.shape[1] != K:
        raise ValueError("x must have K columns")
    qz_packed_bytes(N, K, bits, symmetric, group_size)      # validates the format
    dev = w.device
    st = _launch_stream(stream, dev)
    with _on(stream):
        if codes is None:
            codes = torch.empty((N, K // 2) if bits == 4 else (N, K), dtype=torch.uint8,
                                device=dev)
        if scales is None:
            scales = torch.empty((N, K // group_size), dtype=torch.bfloat16, device=dev)
        if zeros is None and not symmetric:
            zeros = torch.empty((N, K // group_size), dtype=torch.uint8, device=dev)
        nbytes = qz_workspace_bytes(QZ_OP_GPTQ, 1, N, K, group_size)
        if workspace is None:
            workspace = torch.empty(nbytes, dtype=torch.uint8, device=dev)
        elif isinstance(workspace, Workspace):
            workspace = workspace.get(nbytes)
        _check(lib.qz_gptq_quantize(_ptr(w), _ptr(x), N, K, x.shape[0], bits, int(symmetric),
                                    group_size, float(damp), _ptr(codes), _ptr(scales),
                                    _ptr(zeros) if not symmetric else None, _ptr(workspace),
                                    workspace.numel() * workspace.element_size(), _handle(st)),
               "qz_gptq_quantize")
    return codes, scales, (None if symmetric else zeros)


def qz_fp4_packed_bytes(N, K, kind):
    c, s = _sz(), _sz()
    _check(lib.qz_fp4_packed_bytes(N, K, kind, ctypes.byref(c), ctypes.byref(s)),
           "qz_fp4_packed_bytes")
    return c.value, s.value


def qz_fp4_quantize(w, kind, codes=None, scales=None, tensor_scale=None, stream=None):
    """FP4 with block scales: returns (codes uint8 N x K/2, block scales uint8,
    tensor scale fp32 tensor of one element (NVFP4) or None)."""
    if w.dtype != torch.bfloat16 or w.dim() != 2:
        raise ValueError("w must be a 2-D bf16 tensor")
    N, K = w.shape
    qz_fp4_packed_bytes(N, K, kind)                      # validates the shape
    dev = w.device
    st = _launch_stream(stream, dev)
    with _on(stream):
        if codes is None:
            codes = torch.empty((N, K // 2), dtype=torch.uint8, device=dev)
        if scales is None:
            scales = torch.empty((N, K // FP4_BLOCK[kind]), dtype=torch.uint8, device=dev)
        if tensor_scale is None and kind == QZ_FP4_NV:
            tensor_scale = torch.empty(1, dtype=torch.float32, device=dev)
        _check(lib.qz_fp4_quantize(_ptr(w), N, K, kind, _ptr(codes), _ptr(scales),
                                   _ptr(tensor_scale) if kind == QZ_FP4_NV else None,
                                   _handle(st)), "qz_fp4_quantize")
    return codes, scales, (tensor_scale if kind == QZ_FP4_NV else None)


def qz_fp4_dequantize(codes, scales, tensor_scale, N, K, kind, out=None, stream=None):
    """The dequantized FP4 weights as an N x K bf16 tensor."""
    dev = codes.device
    st = _launch_stream(stream, dev)
    with _on(stream):
        if out is None:
            out = torch.empty((N, K), dtype=torch.bfloat16, device=dev)
        _check(lib.qz_fp4_dequantize(_ptr(codes), _ptr(scales), _ptr(tensor_scale), N, K, kind,
                                     _ptr(out), _handle(st)), "qz_fp4_dequantize")
    return out


def qz_fp4a16_gemv(a, codes, scales, tensor_scale, N, K, kind, y=None, workspace=None,
                   stream=None):
    """y = a * w_hat^T for FP4 weights with block scales, M <= 16."""
    st = _launch_stream(stream, a.device)
    M = a.shape[0]
    with _on(stream):
        y = _matmul_out(a, N, y)
        nbytes = qz_workspace_bytes(QZ_OP_FP4A16_GEMV, M, N, K, 0)
        ws_ptr, ws_bytes = _ws_args(workspace, nbytes, a.device)
        _check(lib.qz_fp4a16_gemv(_ptr(a), _ptr(codes), _ptr(scales), _ptr(tensor_scale), M, N,
                                  K, kind, _ptr(y), ws_ptr, ws_bytes, _handle(st)),
               "qz_fp4a16_gemv")
    return y


def qz_fp4_mma_scale_bytes(rows, K, kind) -> int:
    out = _sz()
    _check(lib.qz_fp4_mma_scale_bytes(rows, K, kind, ctypes.byref(out)), "qz_fp4_mma_scale_bytes")
    return out.value


def qz_fp4_scales_to_mma(scales, rows, K, kind, out=None, stream=None):
    """Block scales as qz_fp4_quantize writes them -> the MMA scale layout
    (uint8 tensor of qz_fp4_mma_scale_bytes(rows, K, kind) bytes)."""
    st = _launch_stream(stream, scales.device)
    with _on(stream):
        if out is None:
            out = torch.empty(qz_fp4_mma_scale_bytes(rows, K, kind), dtype=torch.uint8,
                              device=scales.device)
        _check(lib.qz_fp4_scales_to_mma(_ptr(scales), rows, K, kind, _ptr(out), _handle(st)),
               "qz_fp4_scales_to_mma")
    return out


def qz_fp4a4_gemm(a, codes, scales_mma, tensor_scale, N, K, kind, y=None, workspace=None,
                  stream=None):
    """W4A4: y = a_hat * w_hat^T with the activations quantized to the same FP4
    kind inside the call.  `workspace`: a uint8 tensor, a Workspace (its
    scratch buffer is used) or None; after the call it holds the quantized
    activations."""
    st = _launch_stream(stream, a.device)
    M = a.shape[0]
    with _on(stream):
        y = _matmul_out(a, N, y)
        nbytes = qz_workspace_bytes(QZ_OP_FP4A4_GEMM, M, N, K, 0)
        if workspace is None:
            workspace = torch.empty(nbytes, dtype=torch.uint8, device=a.device)
        elif isinstance(workspace, Workspace):
            workspace = workspace.get_scratch(nbytes)
        _check(lib.qz_fp4a4_gemm(_ptr(a), _ptr(codes), _ptr(scales_mma), _ptr(tensor_scale), M,
                                 N, K, kind, _ptr(y), _ptr(workspace),
                                 workspace.numel() * workspace.element_size(), _handle(st)),
               "qz_fp4a4_gemm")
    return y


def qz_set_device_wait_limit(limit: int) -> None:
    lib.qz_set_device_wait_limit(int(limit))


def qz_set_launch_overlap(mode: int) -> None:
    """Launch overlap of the decode GEMV with the preceding kernel (see qz.h)."""
    _check(lib.qz_set_launch_overlap(int(mode)), "qz_set_launch_overlap")


def qz_device_status() -> int:
    return int(lib.qz_device_status())
