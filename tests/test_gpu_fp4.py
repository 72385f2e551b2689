"""FP4 with block scales on the GPU vs the CPU oracle (needs a B200).

Quantization concepts guide, section "FP4 with block scales": E2M1 codes
(0, 0.5, 1, 1.5, 2, 3, 4, 6 and negatives) with a scale per small block,
MXFP4 (32-value blocks, power-of-two scales) and NVFP4 (16-value blocks, E4M3
scales and one fp32 tensor scale).  Codes, block scales, the tensor scale and
the dequantized bf16 weights are compared bit for bit; the FP4A16 decode GEMV
within |y - y_ref| <= 8e-3 |y_ref| + 1e-4 sum_k |a_k w_k| against the fp64
product over the exact dequantized values (e2m1 x scales), and bit for bit
with one-hot activations (one weight times 1, rounded once).
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
    return torch.device("cuda:0")


def u16(t):
    return synthetic.bf16_bits(t)


def u8(t):
    return t.detach().cpu().numpy().view(np.uint8)


def to_dev(a, dev):
    return torch.from_numpy(np.ascontiguousarray(a)).to(dev)


def gpu_quant(w_dev, kind):
    c, s, ts = qz.qz_fp4_quantize(w_dev, kind)
    torch.cuda.synchronize()
    return u8(c), u8(s), (None if ts is None else float(ts.cpu()[0]))


def assert_same(got, ref, what):
    assert np.array_equal(got[1], ref[1]), f"{what}: block scales differ"
    assert got[2] == ref[2], f"{what}: tensor scale {got[2]} vs {ref[2]}"
    if not np.array_equal(got[0], ref[0]):
        bad = np.argwhere(got[0] != ref[0])
        raise AssertionError(f"{what}: {len(bad)} code bytes differ, first {bad[:5].tolist()}")


def edge_rows(K=256):
    rng = np.random.default_rng(3)
    rows = [np.zeros(K, np.float32),                                     # all zero
            np.full(K, 6.0, np.float32),                                 # exactly the E2M1 max
            (rng.normal(0, 1, K) * 1e-38).astype(np.float32),            # bf16 subnormals
            (rng.normal(0, 1, K) * 1e30).astype(np.float32),             # huge
            -np.abs(rng.normal(0, 1, K)).astype(np.float32)]             # all negative
    r = np.zeros(K, np.float32)
    r[:8] = [6.0, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]                # half-way points
    r[32:40] = [-6.0, -0.25, -0.75, -1.25, -1.75, -2.5, -3.5, -5.0]
    rows.append(r)
    r = (rng.normal(0, 0.02, K)).astype(np.float32)
    r[::37] *= 300.0                                                     # outliers
    rows.append(r)
    return torch.from_numpy(np.stack(rows)).to(torch.bfloat16)


@pytest.mark.parametrize("kind", KINDS)
@pytest.mark.parametrize("N,K", [(64, 1024), (37, 4096), (128, 512), (3, 96)])
def test_fp4_quantize_and_dequantize_bit_exact(dev, kind, N, K):
    if K % oracle.FP4_BLOCK[kind]:
        pytest.skip("K is not a multiple of the block")
    w = synthetic.weights(N, K, sigma=0.02, seed=N + K + kind)
    ref = oracle.fp4_quantize(u16(w), kind)
    got = gpu_quant(w.to(dev), kind)
    assert_same(got, ref, f"fp4 kind={kind} {N}x{K}")
    w_hat, _ = oracle.fp4_dequantize(*ref, N, K, kind)
    ts = None if ref[2] is None else torch.tensor([ref[2]], dtype=torch.float32, device=dev)
    out = qz.qz_fp4_dequantize(to_dev(ref[0], dev), to_dev(ref[1], dev), ts, N, K, kind)
    torch.cuda.synchronize()
    assert np.array_equal(u16(out), w_hat)


@pytest.mark.parametrize("kind", KINDS)
def test_fp4_edge_rows_bit_exact(dev, kind):
    w = edge_rows()
    N, K = w.shape
    ref = oracle.fp4_quantize(u16(w), kind)
    got = gpu_quant(w.to(dev), kind)
    assert_same(got, ref, f"fp4 edge rows kind={kind}")
    w_hat, _ = oracle.fp4_dequantize(*ref, N, K, kind)
    ts = None if ref[2] is None else torch.tensor([ref[2]], dtype=torch.float32, device=dev)
    out = qz.qz_fp4_dequantize(to_dev(ref[0], dev), to_dev(ref[1], dev), ts, N, K, kind)
    torch.cuda.synchronize()
    assert np.array_equal(u16(out), w_hat)


def check_gemv(dev, kind, N, K, M, seed, rows=None):
    w = synthetic.weights(N, K, sigma=0.02, seed=seed)
    a = synthetic.activations(M, K, seed=seed + 1)
    codes, scales, ts = oracle.fp4_quantize(u16(w), kind)
    tsd = None if ts is None else torch.tensor([ts], dtype=torch.float32, device=dev)
    y = qz.qz_fp4a16_gemv(a.to(dev), to_dev(codes, dev), to_dev(scales, dev), tsd, N, K, kind)
    torch.cuda.synchronize()
    if rows is None:
        rows = np.arange(N)
    _, w_exact = oracle.fp4_dequantize(codes[rows], scales[rows], ts, len(rows), K, kind)
    y_ref, abs_ref = oracle.matmul_f64_exact(u16(a), w_exact)
    yv = oracle.bf16_bits_to_f32(u16(y)[:, rows]).astype(np.float64)
    bound = oracle.tolerance(y_ref, abs_ref)
    err = np.abs(yv - y_ref)
    assert (err <= bound).all(), f"kind={kind} {N}x{K} M={M}: max err/bound {(err / bound).max():.3f}"


@pytest.mark.parametrize("kind", KINDS)
@pytest.mark.parametrize("N,K", [(1024, 1024), (1000, 384), (4100, 1152), (17, 128), (256, 2048),
                                 (4100, 1536)])    # K % 512 == 0: units of 256 k
@pytest.mark.parametrize("M", [1, 3, 8, 16])
def test_fp4a16_gemv_tolerance(dev, kind, N, K, M):
    check_gemv(dev, kind, N, K, M, seed=N + K + M)


@pytest.mark.parametrize("kind", KINDS)
@pytest.mark.parametrize("M", [1, 16])
def test_fp4a16_gemv_70b_layer_sampled(dev, kind, M):
    rng = np.random.default_rng(9)
    rows = np.array(sorted(set(rng.choice(28672, 24, replace=False).tolist()) | {0, 28671}))
    check_gemv(dev, kind, 28672, 8192, M, seed=4, rows=rows)


@pytest.mark.parametrize("kind", KINDS)
@pytest.mark.parametrize("N,K", [(1024, 1024), (300, 384)])
def test_fp4a16_gemv_onehot_is_exact(dev, kind, N, K):
    """One-hot activations: y[m][n] is one weight times 1, rounded once to
    bf16 -- the dequantized bf16 weight."""
    w = synthetic.weights(N, K, sigma=0.02, seed=5)
    codes, scales, ts = oracle.fp4_quantize(u16(w), kind)
    w_hat, _ = oracle.fp4_dequantize(codes, scales, ts, N, K, kind)
    ks = np.random.default_rng(1).choice(K, size=16, replace=False)
    a = np.zeros((16, K), np.uint16)
    a[np.arange(16), ks] = 0x3F80
    tsd = None if ts is None else torch.tensor([ts], dtype=torch.float32, device=dev)
    y = qz.qz_fp4a16_gemv(synthetic.from_bf16_bits(a, dev), to_dev(codes, dev),
                          to_dev(scales, dev), tsd, N, K, kind)
    torch.cuda.synchronize()
    assert np.array_equal(u16(y), w_hat[:, ks].T)


def test_fp4_quantize_feeds_the_gemv(dev):
    """The GPU quantizer's output goes straight into the GEMV."""
    N, K, kind = 2048, 4096, qz.QZ_FP4_NV
    w = synthetic.weights(N, K, sigma=0.02, seed=61).to(dev)
    a = synthetic.activations(1, K, seed=62).to(dev)
    c, s, ts = qz.qz_fp4_quantize(w, kind)
    y = qz.qz_fp4a16_gemv(a, c, s, ts, N, K, kind)
    torch.cuda.synchronize()
    ref = oracle.fp4_quantize(u16(w), kind)
    assert np.array_equal(u8(c), ref[0]) and np.array_equal(u8(s), ref[1])
    _, w_exact = oracle.fp4_dequantize(*ref, N, K, kind)
    y_ref, abs_ref = oracle.matmul_f64_exact(u16(a), w_exact)
    yv = oracle.bf16_bits_to_f32(u16(y)).astype(np.float64)
    assert (np.abs(yv - y_ref) <= oracle.tolerance(y_ref, abs_ref)).all()


@pytest.mark.parametrize("kind", KINDS)
@pytest.mark.parametrize("N,K,M", [(28672, 8192, 1), (4096, 4096, 1), (8192, 8192, 16),
                                   (4096, 11008, 1)])
def test_fp4a16_gemv_launch_overlap_modes_agree(dev, kind, N, K, M):
    """With launch overlap the producer fetches a first ring of weights before
    the previous kernel completes and activations after; CTA ranges that start
    in the middle of a scale span (NVFP4's spans are 4 units) must not make it
    wait on the consumers while activations are still to come.  Both modes
    give identical bits and no bounded wait runs out."""
    w = synthetic.weights(N, K, sigma=0.02, seed=81).to(dev)
    c, s, ts = qz.qz_fp4_quantize(w, kind)
    a0 = synthetic.activations(M, K, seed=82, device=dev)
    outs = {}
    try:
        for mode in (0, 1):
            qz.qz_set_launch_overlap(mode)
            ys = [qz.qz_fp4a16_gemv(a0, c, s, ts, N, K, kind) for _ in range(3)]
            torch.cuda.synchronize()
            assert qz.qz_device_status() == 0, f"a bounded wait ran out (overlap {mode})"
            assert all(torch.equal(ys[0], y) for y in ys[1:])
            outs[mode] = u16(ys[0])
    finally:
        qz.qz_set_launch_overlap(0)
    assert np.array_equal(outs[0], outs[1])
