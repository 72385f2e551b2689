"""CPU oracle for group-wise affine weight quantization (TEST INFRASTRUCTURE).

Only the test suite, ``__graft_entry__.smoke()`` and the benchmark's
``cpu_baseline`` / reference leg may import this package.  The product path
(the CUDA library and its Python binding) never does, and this package never
imports the product: the two share nothing but the seeded input generator in
``synthetic``.

The arithmetic lives in ``qz_oracle.c`` (plain scalar C, fp32 IEEE for the
quantizer, fp64 for the matmul); this module only marshals numpy arrays.
Every function cites the page passage it follows in the C source.
"""
import ctypes

import numpy as np

from . import build as _build

_lib = None

_i64 = ctypes.c_int64
_int = ctypes.c_int
_p = ctypes.c_void_p


def load(path: str):
    """Open an oracle shared library at ``path`` and declare its signatures."""
    L = ctypes.CDLL(path)
    L.qzo_bf16_to_f32.argtypes = [ctypes.c_uint16]
    L.qzo_bf16_to_f32.restype = ctypes.c_float
    L.qzo_f32_to_bf16_rne.argtypes = [ctypes.c_float]
    L.qzo_f32_to_bf16_rne.restype = ctypes.c_uint16
    L.qzo_f32_to_bf16_up.argtypes = [ctypes.c_float]
    L.qzo_f32_to_bf16_up.restype = ctypes.c_uint16
    L.qzo_code_range.argtypes = [_int, _int, ctypes.POINTER(_int), ctypes.POINTER(_int)]
    L.qzo_code_range.restype = _int
    L.qzo_quantize_pack.argtypes = [_p, _i64, _i64, _int, _int, _i64, _p, _p, _p]
    L.qzo_quantize_pack.restype = _int
    L.qzo_dequantize.argtypes = [_p, _p, _p, _i64, _i64, _int, _int, _i64, _p]
    L.qzo_dequantize.restype = _int
    L.qzo_matmul_f64.argtypes = [_p, _p, _i64, _i64, _i64, _p, _p]
    L.qzo_matmul_f64.restype = _int
    L.qzo_gptq_hessian_factor.argtypes = [_p, _i64, _i64, ctypes.c_double, _p, _p]
    L.qzo_gptq_hessian_factor.restype = _int
    L.qzo_gptq_quantize_with_factor.argtypes = [_p, _p, _i64, _i64, _i64, _int, _int, _i64,
                                                _p, _p, _p, _p]
    L.qzo_gptq_quantize_with_factor.restype = _int
    L.qzo_gptq_quantize.argtypes = [_p, _p, _i64, _i64, _i64, ctypes.c_double, _i64, _int,
                                    _int, _i64, _p, _p, _p]
    L.qzo_gptq_quantize.restype = _int
    L.qzo_e4m3_to_f64.argtypes = [ctypes.c_uint8]
    L.qzo_e4m3_to_f64.restype = ctypes.c_double
    L.qzo_e2m1_to_f64.argtypes = [ctypes.c_uint8]
    L.qzo_e2m1_to_f64.restype = ctypes.c_double
    L.qzo_fp4_quantize.argtypes = [_p, _i64, _i64, _int, _p, _p, _p]
    L.qzo_fp4_quantize.restype = _int
    L.qzo_fp4_dequantize.argtypes = [_p, _p, _p, _i64, _i64, _int, _p, _p]
    L.qzo_fp4_dequantize.restype = _int
    L.qzo_matmul_f64_exact.argtypes = [_p, _p, _i64, _i64, _i64, _p, _p]
    L.qzo_matmul_f64_exact.restype = _int
    L.qzo_matmul_f64_ab.argtypes = [_p, _p, _i64, _i64, _i64, _p, _p]
    L.qzo_matmul_f64_ab.restype = _int
    L.qzo_set_threads.argtypes = [_int]
    L.qzo_set_threads.restype = None
    L.qzo_max_threads.argtypes = []
    L.qzo_max_threads.restype = _int
    return L


def lib():
    """The oracle library, built from ``qz_oracle.c`` on first use."""
    global _lib
    if _lib is None:
        _lib = load(_build.build())
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def set_threads(n: int) -> None:
    lib().qzo_set_threads(int(n))


def max_threads() -> int:
    return int(lib().qzo_max_threads())


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to fp32 values (exact: bf16 is the top half)."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


def f32_to_bf16_rne(x: float) -> int:
    return int(lib().qzo_f32_to_bf16_rne(float(x)))


def f32_to_bf16_up(x: float) -> int:
    return int(lib().qzo_f32_to_bf16_up(float(x)))


def code_range(bits: int, symmetric: bool):
    lo, hi = _int(), _int()
    if lib().qzo_code_range(bits, int(symmetric), ctypes.byref(lo), ctypes.byref(hi)):
        raise ValueError("unsupported format")
    return lo.value, hi.value


def packed_shapes(N: int, K: int, bits: int, symmetric: bool, group_size: int):
    """Array shapes of (codes, scales, zeros); zeros is None when symmetric."""
    codes = (N, K // 2) if bits == 4 else (N, K)
    if group_size == 0:
        scales = (1,)
    else:
        scales = (N, K // group_size)
    return codes, scales, (None if symmetric else scales)


def quantize_pack(w, bits: int = 4, symmetric: bool = False, group_size: int = 128):
    """Quantize an N x K matrix.

    ``w`` is either bf16 bit patterns (uint16) or fp32 values.  Returns
    ``(codes uint8, scales bf16-bits uint16, zeros uint8 or None)``.
    """
    w = np.asarray(w)
    if w.dtype == np.uint16:
        wf = bf16_bits_to_f32(w)
    else:
        wf = np.ascontiguousarray(w, dtype=np.float32)
    if wf.ndim != 2:
        raise ValueError("w must be 2-D")
    N, K = wf.shape
    cs, ss, zs = packed_shapes(N, K, bits, symmetric, group_size)
    codes = np.zeros(cs, dtype=np.uint8)
    scales = np.zeros(ss, dtype=np.uint16)
    zeros = None if zs is None else np.zeros(zs, dtype=np.uint8)
    rc = lib().qzo_quantize_pack(_ptr(wf), N, K, bits, int(symmetric), group_size,
                                 _ptr(codes), _ptr(scales), _ptr(zeros))
    if rc != 0:
        raise ValueError("qzo_quantize_pack rejected the arguments")
    return codes, scales, zeros


def dequantize(codes, scales, zeros, N: int, K: int, bits: int = 4,
               symmetric: bool = False, group_size: int = 128) -> np.ndarray:
    """Return the bf16 bit patterns of w_hat = bf16(S * (q - Z)), N x K."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint16)
    if zeros is not None:
        zeros = np.ascontiguousarray(zeros, dtype=np.uint8)
    out = np.zeros((N, K), dtype=np.uint16)
    rc = lib().qzo_dequantize(_ptr(codes), _ptr(scales), _ptr(zeros), N, K, bits,
                              int(symmetric), group_size, _ptr(out))
    if rc != 0:
        raise ValueError("qzo_dequantize rejected the arguments")
    return out


FP4_MX, FP4_NV = 0, 1                      # MXFP4 (block 32, E8M0), NVFP4 (block 16, E4M3)
FP4_BLOCK = {FP4_MX: 32, FP4_NV: 16}


def e4m3_to_f64(b: int) -> float:
    return float(lib().qzo_e4m3_to_f64(int(b)))


def e2m1_to_f64(code: int) -> float:
    return float(lib().qzo_e2m1_to_f64(int(code)))


def fp4_quantize(w, kind: int):
    """FP4 with block scales: returns (codes uint8 N x K/2, block scales
    uint8 N x K/block, tensor scale float (NVFP4) or None)."""
    wf = _weights_f32(w)
    N, K = wf.shape
    codes = np.zeros((N, K // 2), dtype=np.uint8)
    scales = np.zeros((N, K // FP4_BLOCK[kind]), dtype=np.uint8)
    ts = np.zeros(1, dtype=np.float32)
    if lib().qzo_fp4_quantize(_ptr(wf), N, K, kind, _ptr(codes), _ptr(scales), _ptr(ts)) != 0:
        raise ValueError("qzo_fp4_quantize rejected the arguments")
    return codes, scales, (float(ts[0]) if kind == FP4_NV else None)


def fp4_dequantize(codes, scales, tensor_scale, N: int, K: int, kind: int):
    """(bf16 bits of the dequantized weights, their exact values in fp64)."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    ts = np.array([tensor_scale if tensor_scale is not None else 1.0], dtype=np.float32)
    w_hat = np.zeros((N, K), dtype=np.uint16)
    w_exact = np.zeros((N, K), dtype=np.float64)
    if lib().qzo_fp4_dequantize(_ptr(codes), _ptr(scales), _ptr(ts), N, K, kind, _ptr(w_hat),
                                _ptr(w_exact)) != 0:
        raise ValueError("qzo_fp4_dequantize rejected the arguments")
    return w_hat, w_exact


def matmul_f64_exact(a_bits, w_exact):
    """fp64 y = a @ w^T and sum_k |a w| for bf16 activations and fp64 weights."""
    a = np.ascontiguousarray(a_bits, dtype=np.uint16)
    w = np.ascontiguousarray(w_exact, dtype=np.float64)
    M, K = a.shape
    N = w.shape[0]
    y = np.zeros((M, N), dtype=np.float64)
    ya = np.zeros((M, N), dtype=np.float64)
    lib().qzo_matmul_f64_exact(_ptr(a), _ptr(w), M, N, K, _ptr(y), _ptr(ya))
    return y, ya


def matmul_f64_ab(a_exact, w_exact):
    """fp64 y = a @ w^T and sum_k |a w| for fp64 activations and weights (the
    W4A4 reference: both are exact dequantized FP4 values)."""
    a = np.ascontiguousarray(a_exact, dtype=np.float64)
    w = np.ascontiguousarray(w_exact, dtype=np.float64)
    M, K = a.shape
    N = w.shape[0]
    y = np.zeros((M, N), dtype=np.float64)
    ya = np.zeros((M, N), dtype=np.float64)
    lib().qzo_matmul_f64_ab(_ptr(a), _ptr(w), M, N, K, _ptr(y), _ptr(ya))
    return y, ya


GPTQ_BLOCK = 128      # the GPTQ explainer's lazy-batch width
GPTQ_DAMP = 0.01      # lambda = GPTQ_DAMP * mean(diag H) (a reading: the page gives no value)


def _weights_f32(w):
    w = np.asarray(w)
    if w.dtype == np.uint16:
        return bf16_bits_to_f32(w)
    return np.ascontiguousarray(w, dtype=np.float32)


def gptq_hessian_factor(x_bits, damp: float = GPTQ_DAMP):
    """H = 2 X X^T + lambda I from calibration samples (``x_bits``: bf16 bits,
    one sample per row, n x K) and U, the upper Cholesky factor of H^-1."""
    x = np.ascontiguousarray(x_bits, dtype=np.uint16)
    n, K = x.shape
    H = np.zeros((K, K), dtype=np.float64)
    U = np.zeros((K, K), dtype=np.float64)
    if lib().qzo_gptq_hessian_factor(_ptr(x), K, n, float(damp), _ptr(H), _ptr(U)) != 0:
        raise ValueError("the damped Hessian is not positive definite")
    return H, U


def gptq_quantize_with_factor(w, U, bits: int = 4, symmetric: bool = False,
                              group_size: int = 128, block: int = GPTQ_BLOCK):
    """GPTQ's column loop over the weights ``w`` (bf16 bits or fp32 values)
    with the factor ``U``; returns (codes, scales, zeros | None, compensated
    weights fp64)."""
    wf = _weights_f32(w)
    N, K = wf.shape
    Uc = np.ascontiguousarray(U, dtype=np.float64)
    if Uc.shape != (K, K):
        raise ValueError("U must be K x K")
    cs, ss, zs = packed_shapes(N, K, bits, symmetric, group_size)
    codes = np.zeros(cs, dtype=np.uint8)
    scales = np.zeros(ss, dtype=np.uint16)
    zeros = None if zs is None else np.zeros(zs, dtype=np.uint8)
    w_out = np.zeros((N, K), dtype=np.float64)
    rc = lib().qzo_gptq_quantize_with_factor(_ptr(wf), _ptr(Uc), N, K, block, bits,
                                             int(symmetric), group_size, _ptr(codes),
                                             _ptr(scales), _ptr(zeros), _ptr(w_out))
    if rc != 0:
        raise ValueError("qzo_gptq_quantize_with_factor rejected the arguments")
    return codes, scales, zeros, w_out


def gptq_quantize(w, x_bits, bits: int = 4, symmetric: bool = False, group_size: int = 128,
                  damp: float = GPTQ_DAMP, block: int = GPTQ_BLOCK):
    """GPTQ of one layer: weights ``w`` (N x K), calibration samples
    ``x_bits`` (n x K bf16 bits); returns (codes, scales, zeros | None) in
    the packed format of :func:`quantize_pack`."""
    wf = _weights_f32(w)
    N, K = wf.shape
    x = np.ascontiguousarray(x_bits, dtype=np.uint16)
    if x.shape[1] != K:
        raise ValueError("calibration samples must have K features")
    cs, ss, zs = packed_shapes(N, K, bits, symmetric, group_size)
    codes = np.zeros(cs, dtype=np.uint8)
    scales = np.zeros(ss, dtype=np.uint16)
    zeros = None if zs is None else np.zeros(zs, dtype=np.uint8)
    rc = lib().qzo_gptq_quantize(_ptr(wf), _ptr(x), N, K, x.shape[0], float(damp), block, bits,
                                 int(symmetric), group_size, _ptr(codes), _ptr(scales),
                                 _ptr(zeros))
    if rc != 0:
        raise ValueError("qzo_gptq_quantize rejected the arguments")
    return codes, scales, zeros


def matmul_f64(a_bits, w_hat_bits):
    """fp64 y = a @ w_hat^T and sum_k |a*w_hat| over bf16 bit-pattern inputs."""
    a = np.ascontiguousarray(a_bits, dtype=np.uint16)
    w = np.ascontiguousarray(w_hat_bits, dtype=np.uint16)
    M, K = a.shape
    N, K2 = w.shape
    if K != K2:
        raise ValueError("inner dimensions differ")
    y = np.zeros((M, N), dtype=np.float64)
    ya = np.zeros((M, N), dtype=np.float64)
    lib().qzo_matmul_f64(_ptr(a), _ptr(w), M, N, K, _ptr(y), _ptr(ya))
    return y, ya


# Half the spacing of the bf16 subnormals (2^-133).  Below 2^-126 a bf16
# output cannot come closer than this to an arbitrary real value, while the
# relative term 8e-3 |y| assumes bf16's normal relative precision (2^-8).
BF16_SUBNORMAL_HALF_SPACING = 2.0 ** -134


def tolerance(y_ref: np.ndarray, abs_ref: np.ndarray) -> np.ndarray:
    """Per-element bound |y - y_ref| <= 8e-3 |y_ref| + 1e-4 sum_k |a_k w_k|,
    plus half the bf16 subnormal spacing so that outputs below the smallest
    normal bf16 can meet it (negligible for every normal output)."""
    return 8e-3 * np.abs(y_ref) + 1e-4 * abs_ref + BF16_SUBNORMAL_HALF_SPACING
