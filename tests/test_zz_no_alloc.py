"""qz_w4a16_gemv_noalloc, called through the C ABI (needs a B200).

The entry point serves callers that cannot allocate device memory -- a
plugin inside an application that owns all device memory, or latency-critical
code that cannot afford cudaMalloc -- by keeping the GEMV's split-K scratch
in a fixed array inside the library.  Its results must match the regular
qz_w4a16_gemv (which takes a caller-allocated workspace) within the tolerance
the parity tests use, on consecutive calls that share that array.

This file is named so that pytest collects it last; it must also pass when it
runs alone in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import synthetic
import weight_only_quantization_wise_b200 as qz

pytestmark = pytest.mark.gpu


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def _bits(t):
    return synthetic.bf16_bits(t)


def _noalloc(a, c, s, z, N, K, g, y, stream):
    return qz.lib.qz_w4a16_gemv_noalloc(_p(a), _p(c), _p(s), _p(z), a.shape[0], N, K, g, _p(y),
                                        ctypes.c_void_p(stream.cuda_stream))


def _case(dev, M, N, K, g, seed):
    w = synthetic.weights(N, K, sigma=0.02, seed=seed)
    a = synthetic.activations(M, K, seed=seed + 1)
    c, s, z = oracle.quantize_pack(_bits(w), 4, False, g)
    w_hat = oracle.dequantize(c, s, z, N, K, 4, False, g)
    y_ref, abs_ref = oracle.matmul_f64(_bits(a), w_hat)
    to = lambda arr: torch.from_numpy(np.ascontiguousarray(arr)).to(dev)
    return (a.to(dev), to(c), synthetic.from_bf16_bits(s, dev), to(z), y_ref,
            oracle.tolerance(y_ref, abs_ref))


def test_noalloc_matches_workspace_gemv_on_consecutive_calls():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dev = torch.device("cuda:0")
    stream = torch.cuda.current_stream(dev)
    # shapes whose split-K plan uses the scratch (splits > 1), then one that
    # needs a different tile count, then the first again
    cases = [(3, 4096, 4096, 128, 21), (9, 1000, 1152, 64, 22), (3, 4096, 4096, 128, 21)]
    prepared = {}
    for M, N, K, g, seed in cases:
        assert qz.qz_workspace_bytes(qz.QZ_OP_W4A16_GEMV, M, N, K, g) > 0
        key = (M, N, K, g, seed)
        if key not in prepared:
            prepared[key] = _case(dev, M, N, K, g, seed)
        a, c, s, z, y_ref, bound = prepared[key]
        y_ws = qz.qz_w4a16_gemv(a, c, s, z, N, K, g)          # caller-allocated workspace
        y_na = torch.empty_like(y_ws)
        assert _noalloc(a, c, s, z, N, K, g, y_na, stream) == 0
        torch.cuda.synchronize()
        got = oracle.bf16_bits_to_f32(_bits(y_na)).astype(np.float64)
        ref_ws = oracle.bf16_bits_to_f32(_bits(y_ws)).astype(np.float64)
        assert (np.abs(got - ref_ws) <= bound).all(), "no-alloc differs from the workspace GEMV"
        assert (np.abs(got - y_ref) <= bound).all(), "no-alloc out of tolerance vs the oracle"


def test_noalloc_rejects_sizes_beyond_its_scratch():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    M, N, K, g = 16, 70000, 1024, 128
    need = qz.qz_workspace_bytes(qz.QZ_OP_W4A16_GEMV, M, N, K, g)
    assert need > (8 << 20)
    fake = ctypes.c_void_p(0x10000)       # rejected before any launch or lookup
    st = qz.lib.qz_w4a16_gemv_noalloc(fake, fake, fake, fake, M, N, K, g, fake, None)
    assert st == 4                        # QZ_ERR_WORKSPACE
