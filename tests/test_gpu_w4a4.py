"""W4A4 prefill GEMM (FP4 weights and activations) on the GPU vs the CPU
oracle (needs a B200).

Quantization concepts guide, "Quantize weights or activations": NVFP4 W4A4
quantizes the activations as well, so that the prefill matmul runs on 4-bit
tensor cores; section "FP4 with block scales" for the formats.  The call
quantizes the activations exactly as qz_fp4_quantize does: the codes and
block scales it leaves in the workspace are compared bit for bit with the
oracle's quantization of the same activations (the scales after undoing the
MMA scale layout).  The output is checked within |y - y_ref| <= 8e-3 |y_ref|
+ 1e-4 sum_k |a_k w_k| against the fp64 product of the oracle's exact
dequantized activations and weights (e2m1 x block scale x tensor scale):
the tensor core's products of E2M1 values and their scales are exact and its
sums are fp32, well inside that bound.
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic
import weight_only_quantization_wise_b200 as qz

pytestmark = pytest.mark.gpu

KINDS = [qz.QZ_FP4_MX, qz.QZ_FP4_NV]


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    oracle.set_threads(oracle.max_threads())
    return torch.device("cuda:0")


def u16(t):
    return synthetic.bf16_bits(t)


def u8(t):
    return t.detach().cpu().numpy().view(np.uint8)


def mma_layout_offsets(rows, per_row):
    """Byte offset of scale (r, j) in the MMA scale layout (as include/qz.h
    states it), for r < rows, j < per_row."""
    r = np.arange(rows)[:, None]
    j = np.arange(per_row)[None, :]
    return ((r // 128) * (per_row // 4) + j // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + j % 4


def from_mma_layout(buf, rows, per_row):
    return buf[mma_layout_offsets(rows, per_row)]


def oracle_quant(x_bits, kind):
    codes, scales, ts = oracle.fp4_quantize(x_bits, kind)
    rows, K = x_bits.shape
    _, exact = oracle.fp4_dequantize(codes, scales, ts, rows, K, kind)
    return codes, scales, ts, exact


def prepare_weights(w, kind, dev):
    c, s, ts = qz.qz_fp4_quantize(w.to(dev), kind)
    N, K = w.shape
    s_mma = qz.qz_fp4_scales_to_mma(s, N, K, kind)
    return c, s, ts, s_mma


def check_gemm(dev, M, N, K, kind, seed, tokens=None):
    w = synthetic.weights(N, K, sigma=0.02, seed=seed)
    a = synthetic.activations(M, K, seed=seed + 1)
    c, s, ts, s_mma = prepare_weights(w, kind, dev)
    ws = torch.empty(qz.qz_workspace_bytes(qz.QZ_OP_FP4A4_GEMM, M, N, K, 0), dtype=torch.uint8,
                     device=dev)
    y = qz.qz_fp4a4_gemm(a.to(dev), c, s_mma, ts, N, K, kind, workspace=ws)
    torch.cuda.synchronize()
    assert qz.qz_device_status() == 0
    what = f"w4a4 M={M} N={N} K={K} kind={kind}"

    # the weights as the oracle quantizes them
    wc, wsc, wts, w_exact = oracle_quant(u16(w), kind)
    assert np.array_equal(u8(c), wc) and np.array_equal(u8(s), wsc), f"{what}: weight quantize"
    # the activations the call quantized, left in the workspace
    ac, asc, ats, a_exact = oracle_quant(u16(a), kind)
    wsb = u8(ws)
    per_row = K // qz.FP4_BLOCK[kind]
    codes_bytes = M * K // 2
    sf_off = (codes_bytes + 255) // 256 * 256
    assert np.array_equal(wsb[:codes_bytes].reshape(M, K // 2), ac), f"{what}: activation codes"
    sf = wsb[sf_off:sf_off + qz.qz_fp4_mma_scale_bytes(M, K, kind)]
    assert np.array_equal(from_mma_layout(sf, M, per_row), asc), f"{what}: activation scales"
    pad_rows = -M % 128
    if pad_rows:
        padded = mma_layout_offsets(M + pad_rows, per_row)[M:]
        assert (sf[padded] == 0).all(), f"{what}: padding rows' scales"
    if kind == qz.QZ_FP4_NV:
        amax_off = sf_off + (qz.qz_fp4_mma_scale_bytes(M, K, qz.QZ_FP4_NV) + 255) // 256 * 256
        amax = wsb[amax_off:amax_off + 4].view(np.float32)[0]
        assert np.float32(amax) == np.abs(oracle.bf16_bits_to_f32(u16(a))).max(), f"{what}: amax"

    rows = np.arange(M) if tokens is None else tokens
    y_ref, abs_ref = oracle.matmul_f64_ab(a_exact[rows], w_exact)
    yv = oracle.bf16_bits_to_f32(u16(y)[rows]).astype(np.float64)
    err = np.abs(yv - y_ref)
    tol = oracle.tolerance(y_ref, abs_ref)
    if not (err <= tol).all():
        i = np.unravel_index(np.argmax(err / tol), err.shape)
        raise AssertionError(f"{what}: worst |err|/tol = {(err / tol)[i]:.3g} at {i}, "
                             f"y={yv[i]} ref={y_ref[i]}")


CASES = [  # (M, N, K)
    (128, 256, 256),      # one tile, one stage
    (1, 256, 512),        # one token
    (37, 300, 512),       # ragged tokens and weight rows (second half of the tile partly valid)
    (200, 100, 1024),     # fewer weight rows than half a tile: one scale atom row
    (256, 1000, 2048),    # several tiles in both directions, N % 8 == 0
    (129, 517, 768),      # N odd: scalar stores
    (640, 2048, 1280),    # 40 tiles of five stages each
]


@pytest.mark.parametrize("kind", KINDS)
@pytest.mark.parametrize("M,N,K", CASES)
def test_w4a4_matches_oracle(dev, M, N, K, kind):
    check_gemm(dev, M, N, K, kind, seed=M + N + K)


@pytest.mark.parametrize("kind", KINDS)
def test_w4a4_more_tiles_than_sms(dev, kind):
    """1280 tokens x 4096 weight rows: 160 tiles, so some CTAs take a second
    tile and reuse the accumulator after the epilogue has drained it."""
    check_gemm(dev, 1280, 4096, 512, kind, seed=5, tokens=np.r_[0:96, 1184:1280])


def test_w4a4_prefill_full_size_sampled(dev):
    """The prefill configuration, 2048 tokens x 8192 x 8192, NVFP4: the whole
    GEMM on the GPU, the oracle's product on 24 sampled tokens x all rows."""
    rng = np.random.default_rng(9)
    tokens = np.array(sorted(set(rng.choice(2048, 22, replace=False).tolist()) | {0, 2047}))
    check_gemm(dev, 2048, 8192, 8192, qz.QZ_FP4_NV, seed=6, tokens=tokens)


@pytest.mark.parametrize("kind", KINDS)
def test_scales_to_mma_layout(dev, kind):
    """The converted weight scales are the row-major ones moved to the MMA
    scale layout, with zero scales in the padding rows."""
    N, K = 300, 1024
    w = synthetic.weights(N, K, sigma=0.02, seed=12).to(dev)
    c, s, ts, s_mma = prepare_weights(w, kind, dev)
    torch.cuda.synchronize()
    per_row = K // qz.FP4_BLOCK[kind]
    buf = u8(s_mma)
    assert buf.size == ((N + 127) // 128) * (per_row // 4) * 512
    assert np.array_equal(from_mma_layout(buf, N, per_row), u8(s))
    padded = mma_layout_offsets((N + 127) // 128 * 128, per_row)[N:]
    assert (buf[padded] == 0).all()


def test_w4a4_repeats_bit_for_bit(dev):
    """Two calls on the same inputs give the same bits (no split-K, fixed
    MMA order)."""
    M, N, K = 300, 512, 1024
    w = synthetic.weights(N, K, sigma=0.02, seed=21).to(dev)
    a = synthetic.activations(M, K, seed=22).to(dev)
    c, s, ts, s_mma = prepare_weights(w, qz.QZ_FP4_NV, dev)
    y1 = qz.qz_fp4a4_gemm(a, c, s_mma, ts, N, K, qz.QZ_FP4_NV)
    y2 = qz.qz_fp4a4_gemm(a, c, s_mma, ts, N, K, qz.QZ_FP4_NV)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)
