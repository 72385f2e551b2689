"""GPTQ on the GPU vs the CPU oracle (needs a B200).

GPTQ explainer (azimuth.plus/paper/gptq): damped H = 2 X X^T from
calibration samples, Cholesky of H^-1, fixed column order, lazy batches of
128 columns.  Both sides run the compensation in fp64 and take every code in
fp32 from the compensated weight rounded to fp32, so codes, scales and zeros
are compared bit for bit: a difference could only come from a compensated
weight within about 1e-16 of a rounding boundary, and these seeded inputs
have none.  Calibration samples are synthetic N(0, 1) bf16 activations
(128 per layer unless stated), weights the usual N(0, sigma) with 0.1 %
outliers x20.
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic
import weight_only_quantization_wise_b200 as qz

pytestmark = pytest.mark.gpu


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


def assert_same(got, ref, what):
    (gc, gs, gz), (rc, rs, rz) = got, ref
    assert np.array_equal(u16(gs).reshape(rs.shape), rs), f"{what}: scales differ"
    if rz is None:
        assert gz is None
    else:
        assert np.array_equal(u8(gz).reshape(rz.shape), rz), f"{what}: zeros differ"
    c = u8(gc).reshape(rc.shape)
    if not np.array_equal(c, rc):
        bad = np.argwhere(c != rc)
        raise AssertionError(f"{what}: {len(bad)} code bytes differ, first {bad[:5].tolist()}")


CASES = [  # (N, K, n_samples, bits, symmetric, group_size)
    (64, 256, 128, 4, False, 128),
    (37, 384, 128, 4, False, 128),       # ragged rows, three blocks
    (100, 1024, 128, 4, False, 64),
    (16, 2048, 128, 8, True, 2048),      # per-channel: one group longer than a block
    (50, 512, 96, 4, True, 32),
    (33, 224, 200, 8, False, 32),        # K neither a multiple of 64 nor of 128
    (8, 1024, 1024, 4, False, 256),      # as many samples as features
]


@pytest.mark.parametrize("N,K,n,bits,sym,g", CASES)
def test_gptq_matches_oracle(dev, N, K, n, bits, sym, g):
    w = synthetic.weights(N, K, sigma=0.02, seed=N + K)
    x = synthetic.activations(n, K, seed=N + K + 1)
    ref = oracle.gptq_quantize(u16(w), u16(x), bits, sym, g)
    got = qz.qz_gptq_quantize(w.to(dev), x.to(dev), bits, sym, g)
    torch.cuda.synchronize()
    assert_same(got, ref, f"gptq N={N} K={K} n={n} bits={bits} sym={sym} g={g}")


def test_gptq_identity_hessian_is_round_to_nearest(dev):
    """One calibration sample per feature, x_t = e_t: H is a multiple of the
    identity, nothing is compensated, and GPTQ returns qz_quantize_pack's
    result."""
    N, K = 96, 512
    w = synthetic.weights(N, K, sigma=0.02, seed=31).to(dev)
    x = torch.eye(K, dtype=torch.bfloat16, device=dev)
    for bits, sym, g in ((4, False, 128), (8, True, K), (4, True, 32)):
        got = qz.qz_gptq_quantize(w, x, bits, sym, g)
        ref = qz.qz_quantize_pack(w, bits, sym, g)
        torch.cuda.synchronize()
        for a, b in zip(got, ref):
            assert (a is None and b is None) or torch.equal(a, b), (bits, sym, g)


def test_gptq_7b_layer_sampled_rows(dev):
    """A 4096 x 4096 layer with 128 calibration samples: the whole layer on
    the GPU, the oracle's factor in full and its column loop on sampled rows
    (rows are independent once the factor is known)."""
    N, K, g = 4096, 4096, 128
    w = synthetic.weights(N, K, sigma=0.02, seed=1)
    x = synthetic.activations(128, K, seed=77)
    c, s, z = qz.qz_gptq_quantize(w.to(dev), x.to(dev), 4, False, g)
    torch.cuda.synchronize()
    rng = np.random.default_rng(5)
    rows = np.array(sorted(set(rng.choice(N, size=48, replace=False).tolist()) | {0, N - 1}))
    _, U = oracle.gptq_hessian_factor(u16(x))
    rc, rs, rz, _ = oracle.gptq_quantize_with_factor(u16(w)[rows], U, 4, False, g)
    ti = torch.from_numpy(rows).to(dev)
    assert_same((c.index_select(0, ti), s.index_select(0, ti), z.index_select(0, ti)),
                (rc, rs, rz), "gptq 4096x4096 sampled rows")


def test_gptq_output_feeds_the_decode_gemv(dev):
    """GPTQ writes the packed format: the decode GEMV consumes it unchanged,
    within the matmul bound against the oracle's product over the oracle's
    dequantized GPTQ weights."""
    N, K, g = 512, 1024, 128
    w = synthetic.weights(N, K, sigma=0.02, seed=44)
    x = synthetic.activations(128, K, seed=45)
    a = synthetic.activations(4, K, seed=46)
    c, s, z = qz.qz_gptq_quantize(w.to(dev), x.to(dev), 4, False, g)
    y = qz.qz_w4a16_gemv(a.to(dev), c, s, z, N, K, g)
    torch.cuda.synchronize()
    rc, rs, rz = oracle.gptq_quantize(u16(w), u16(x), 4, False, g)
    w_hat = oracle.dequantize(rc, rs, rz, N, K, 4, False, g)
    y_ref, abs_ref = oracle.matmul_f64(u16(a), w_hat)
    yv = oracle.bf16_bits_to_f32(u16(y)).astype(np.float64)
    assert (np.abs(yv - y_ref) <= oracle.tolerance(y_ref, abs_ref)).all()
