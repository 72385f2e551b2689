"""CUDA path vs the CPU oracle on the same seeded inputs (needs a B200).

Bars (fixed before any kernel was written):
  * codes, scales, zeros: bit-exact;
  * dequantized bf16 weights: bit-exact;
  * matmul outputs: |y - y_ref| <= 8e-3 |y_ref| + 1e-4 sum_k |a_k w_k| against
    the oracle's fp64 product over its own bf16 dequantized weights, plus half
    the bf16 subnormal spacing (2^-134) so that outputs below 2^-126 can meet
    it at all (oracle.tolerance).
Large configurations are checked on sampled rows that the oracle computes on
its own; everything else is compared element by element.
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic
import weight_only_quantization_wise_b200 as qz

pytestmark = pytest.mark.gpu

FORMATS = [(4, False), (4, True), (8, False), (8, True)]


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


def u16(t):
    return synthetic.bf16_bits(t)


def u8(t):
    return t.detach().cpu().numpy().view(np.uint8)


def gpu_quantize(w_dev, bits, sym, g):
    ws = qz.Workspace(w_dev.device)
    c, s, z = qz.qz_quantize_pack(w_dev, bits, sym, g, workspace=ws)
    torch.cuda.synchronize()
    return u8(c), u16(s), (None if z is None else u8(z))


def to_dev_u8(a, dev):
    return torch.from_numpy(np.ascontiguousarray(a)).to(dev)


def to_dev_bf16(bits, dev):
    return synthetic.from_bf16_bits(bits, dev)


def assert_quant_equal(got, ref):
    (gc, gs, gz), (rc, rs, rz) = got, ref
    assert np.array_equal(gs.reshape(rs.shape), rs), "scales differ"
    if rz is None:
        assert gz is None
    else:
        assert np.array_equal(gz.reshape(rz.shape), rz), "zeros differ"
    if not np.array_equal(gc.reshape(rc.shape), rc):
        bad = np.argwhere(gc.reshape(rc.shape) != rc)
        raise AssertionError(f"codes differ at {len(bad)} bytes, first {bad[:5].tolist()}")


def check_tolerance(y_gpu_bits, y_ref, abs_ref, what=""):
    y = oracle.bf16_bits_to_f32(y_gpu_bits).astype(np.float64).reshape(y_ref.shape)
    bound = oracle.tolerance(y_ref, abs_ref)
    err = np.abs(y - y_ref)
    ratio = float((err / np.maximum(bound, 1e-300)).max())
    assert (err <= bound).all(), f"{what}: max error/bound = {ratio:.3f}"
    return ratio


def group_sizes(K):
    gs = [32, 64, 128, 256, K, 0]
    if (K // 2) % 8 == 0 and K // 2 not in gs and K % (K // 2) == 0:
        gs.append(K // 2)
    return [g for g in gs if g == 0 or K % g == 0]


SHAPES = [(1, 128), (37, 384), (64, 1024), (130, 2048)]


@pytest.mark.parametrize("bits,sym", FORMATS)
@pytest.mark.parametrize("N,K", SHAPES)
def test_quantize_pack_bit_exact(dev, bits, sym, N, K):
    w = synthetic.weights(N, K, sigma=0.02, seed=N * 7 + K)
    for g in group_sizes(K):
        ref = oracle.quantize_pack(u16(w), bits, sym, g)
        got = gpu_quantize(w.to(dev), bits, sym, g)
        assert_quant_equal(got, ref)


@pytest.mark.parametrize("bits,sym", FORMATS)
@pytest.mark.parametrize("N,K", SHAPES)
def test_dequantize_bit_exact(dev, bits, sym, N, K):
    w = synthetic.weights(N, K, sigma=0.02, seed=N * 11 + K)
    for g in group_sizes(K):
        c, s, z = oracle.quantize_pack(u16(w), bits, sym, g)
        ref = oracle.dequantize(c, s, z, N, K, bits, sym, g)
        out = qz.qz_dequantize(to_dev_u8(c, dev), to_dev_bf16(s, dev),
                               None if z is None else to_dev_u8(z, dev), N, K, bits, sym, g)
        torch.cuda.synchronize()
        assert np.array_equal(u16(out), ref), (bits, sym, g)


def edge_matrix():
    """Rows that exercise the degenerate and boundary cases of the method."""
    K = 256
    rows = []
    rows.append(np.zeros(K, np.float32))                          # all zero
    rows.append(np.full(K, 0.75, np.float32))                     # constant positive
    rows.append(np.full(K, -3.0, np.float32))                     # constant negative
    r = np.zeros(K, np.float32); r[:4] = [0.0, 15.0, 2.5, 3.5]; rows.append(r)   # ties (S=1)
    r = np.zeros(K, np.float32); r[:2] = [-1.5, 13.5]; rows.append(r)           # clamp at top
    rng = np.random.default_rng(0)
    rows.append((rng.normal(0, 1, K) * 1e-39).astype(np.float32))              # subnormal range
    rows.append((rng.normal(0, 1, K) * 1e30).astype(np.float32))               # huge range
    r = (rng.normal(0, 0.02, K)).astype(np.float32); r[77] = 3.0; rows.append(r)  # one outlier
    rows.append(np.abs(rng.normal(0, 1, K)).astype(np.float32))                # all positive
    rows.append(-np.abs(rng.normal(0, 1, K)).astype(np.float32))               # all negative
    r = np.zeros(K, np.float32); r[5] = -0.0; r[6] = 1e-45; rows.append(r)      # -0, min subnormal
    m = np.stack(rows)
    t = torch.from_numpy(m).to(torch.bfloat16)
    return t


@pytest.mark.parametrize("bits,sym", FORMATS)
def test_edge_groups_bit_exact(dev, bits, sym):
    w = edge_matrix()
    N, K = w.shape
    for g in (32, 128, 256, 0):
        ref = oracle.quantize_pack(u16(w), bits, sym, g)
        got = gpu_quantize(w.to(dev), bits, sym, g)
        assert_quant_equal(got, ref)
        c, s, z = ref
        wref = oracle.dequantize(c, s, z, N, K, bits, sym, g)
        out = qz.qz_dequantize(to_dev_u8(c, dev), to_dev_bf16(s, dev),
                               None if z is None else to_dev_u8(z, dev), N, K, bits, sym, g)
        torch.cuda.synchronize()
        assert np.array_equal(u16(out), wref)


@pytest.mark.parametrize("M", [1, 16, 17, 64])
def test_matmuls_on_edge_rows(dev, M):
    """The edge rows (all zero, constant, ties, top clamp, tiny and huge
    ranges, one outlier, one-signed, -0) through every matmul: the all-zero
    row gives exactly 0 and every output is within the tolerance of the fp64
    product over the oracle's dequantized weights."""
    w = edge_matrix()
    N, K = w.shape
    a = synthetic.activations(M, K, seed=90 + M)
    for bits, sym, g in ((4, False, 128), (8, True, K)):
        c, s, z = oracle.quantize_pack(u16(w), bits, sym, g)
        w_hat = oracle.dequantize(c, s, z, N, K, bits, sym, g)
        y_ref, abs_ref = oracle.matmul_f64(u16(a), w_hat)
        ad, cd, sd = a.to(dev), to_dev_u8(c, dev), to_dev_bf16(s, dev)
        if bits == 4:
            zd = to_dev_u8(z, dev)
            outs = [("gemm", qz.qz_w4a16_gemm(ad, cd, sd, zd, N, K, g))]
            if M <= 32:
                outs.append(("gemv", qz.qz_w4a16_gemv(ad, cd, sd, zd, N, K, g)))
        else:
            outs = [("gemm", qz.qz_w8a16_gemm(ad, cd, sd, N, K))]
            if M <= 32:
                outs.append(("gemv", qz.qz_w8a16_gemv(ad, cd, sd, N, K)))
        torch.cuda.synchronize()
        assert qz.qz_device_status() == 0
        for what, y in outs:
            yb = u16(y).reshape(M, N)
            assert (oracle.bf16_bits_to_f32(yb[:, 0]) == 0).all(), (bits, what)   # all-zero row
            check_tolerance(yb, y_ref, abs_ref, f"edge rows bits={bits} {what} M={M}")


# ---------------------------------------------------------------------------
# GEMV
# ---------------------------------------------------------------------------

GEMV_CASES = [  # (N, K, g)
    (1024, 1024, 128), (1000, 384, 128), (17, 128, 32), (96, 512, 64),
    (256, 2048, 256), (64, 1024, 1024), (4100, 1152, 128),
    # units of 256 k for M <= 16 (K % 256 == 0, K/g a multiple of 16): groups
    # of 128 (two per unit), 256 (one) and 512 (a group spans two units),
    # ragged rows
    (384, 2048, 128), (130, 4096, 256), (4100, 4096, 128), (256, 8192, 512),
    # ... with gathered scale/zero words (K/g not a multiple of 16)
    (300, 2816, 128), (130, 5632, 256),
]


def oracle_w4(w_bits, g):
    N, K = w_bits.shape
    c, s, z = oracle.quantize_pack(w_bits, 4, False, g)
    return c, s, z, oracle.dequantize(c, s, z, N, K, 4, False, g)


@pytest.mark.parametrize("N,K,g", GEMV_CASES)
@pytest.mark.parametrize("M", [1, 2, 5, 8, 9, 16])
def test_w4a16_gemv_tolerance(dev, N, K, g, M):
    w = synthetic.weights(N, K, sigma=0.02, seed=N + K + g)
    a = synthetic.activations(M, K, seed=M)
    c, s, z, w_hat = oracle_w4(u16(w), g)
    y_ref, abs_ref = oracle.matmul_f64(u16(a), w_hat)
    y = qz.qz_w4a16_gemv(a.to(dev), to_dev_u8(c, dev), to_dev_bf16(s, dev), to_dev_u8(z, dev),
                         N, K, g)
    torch.cuda.synchronize()
    check_tolerance(u16(y), y_ref, abs_ref, f"w4a16 M={M} N={N} K={K} g={g}")


def test_w4a16_gemv_two_half_units_onehot_and_fallback(dev):
    """Units of 256 k (up to 16 tokens, scale/zero tiles by TMA): one-hot
    activations read back the oracle's bf16 weights bit for bit; with a scale
    array that is not 16-byte aligned the call falls back to units of 128 k,
    within the bound and inside the workspace qz_workspace_bytes gives."""
    N, K, g = 300, 2048, 128
    w = synthetic.weights(N, K, sigma=0.02, seed=25)
    c, s, z, w_hat = oracle_w4(u16(w), g)
    rng = np.random.default_rng(3)
    ks = rng.choice(K, size=8, replace=False)
    a = np.zeros((8, K), np.uint16)
    a[np.arange(8), ks] = 0x3F80
    cd, zd = to_dev_u8(c, dev), to_dev_u8(z, dev)
    y = qz.qz_w4a16_gemv(to_dev_bf16(a, dev), cd, to_dev_bf16(s, dev), zd, N, K, g)
    torch.cuda.synchronize()
    assert np.array_equal(u16(y), w_hat[:, ks].T)
    # scales at a 2-byte offset inside a larger buffer
    buf = torch.empty(s.size + 1, dtype=torch.bfloat16, device=dev)
    s_off = buf[1:].view(s.shape)
    s_off.copy_(to_dev_bf16(s, dev))
    assert s_off.data_ptr() % 16 != 0
    act = synthetic.activations(5, K, seed=26)
    ws = torch.zeros(qz.qz_workspace_bytes(qz.QZ_OP_W4A16_GEMV, 5, N, K, g), dtype=torch.uint8,
                     device=dev)
    y2 = qz.qz_w4a16_gemv(act.to(dev), cd, s_off, zd, N, K, g, workspace=ws)
    torch.cuda.synchronize()
    y_ref, abs_ref = oracle.matmul_f64(u16(act), w_hat)
    check_tolerance(u16(y2), y_ref, abs_ref, "w4a16 misaligned scales")


@pytest.mark.parametrize("N,K,g", [(1024, 1024, 128), (37, 384, 32), (300, 4096, 128)])
def test_w4a16_gemv_onehot_is_exact(dev, N, K, g):
    """With one-hot activations y[m][n] = w_hat[n][k_m]: the in-register
    dequantization must reproduce the oracle's bf16 weights bit for bit."""
    w = synthetic.weights(N, K, sigma=0.02, seed=5)
    c, s, z, w_hat = oracle_w4(u16(w), g)
    rng = np.random.default_rng(1)
    ks = rng.choice(K, size=16, replace=False)
    a = np.zeros((16, K), np.uint16)
    a[np.arange(16), ks] = 0x3F80
    y = qz.qz_w4a16_gemv(to_dev_bf16(a, dev), to_dev_u8(c, dev), to_dev_bf16(s, dev),
                         to_dev_u8(z, dev), N, K, g)
    torch.cuda.synchronize()
    assert np.array_equal(u16(y), w_hat[:, ks].T)


@pytest.mark.parametrize("N,K", [(1024, 1024), (1000, 384), (17, 128), (4100, 1152)])
@pytest.mark.parametrize("M", [1, 3, 8, 16])
def test_w8a16_gemv_tolerance(dev, N, K, M):
    w = synthetic.weights(N, K, sigma=0.015, seed=N * 3 + K)
    a = synthetic.activations(M, K, seed=M + 100)
    c, s, _ = oracle.quantize_pack(u16(w), 8, True, K)
    w_hat = oracle.dequantize(c, s, None, N, K, 8, True, K)
    y_ref, abs_ref = oracle.matmul_f64(u16(a), w_hat)
    y = qz.qz_w8a16_gemv(a.to(dev), to_dev_u8(c, dev), to_dev_bf16(s, dev), N, K)
    torch.cuda.synchronize()
    check_tolerance(u16(y), y_ref, abs_ref, f"w8a16 M={M} N={N} K={K}")
    # one-hot rows reproduce w_hat exactly
    ks = np.arange(min(16, K)) * (K // 16)
    oh = np.zeros((16, K), np.uint16)
    oh[np.arange(16), ks] = 0x3F80
    y1 = qz.qz_w8a16_gemv(to_dev_bf16(oh, dev), to_dev_u8(c, dev), to_dev_bf16(s, dev), N, K)
    torch.cuda.synchronize()
    assert np.array_equal(u16(y1), w_hat[:, ks].T)


@pytest.mark.parametrize("N,K,g", [(1024, 1024, 128), (1000, 384, 128), (4100, 1152, 128),
                                   (256, 2048, 256), (96, 512, 64)])
@pytest.mark.parametrize("M", [17, 32, 33, 64])
@pytest.mark.parametrize("bits", [4, 8])
def test_gemv_wide_tolerance(dev, N, K, g, M, bits):
    """17..64 tokens: the decode GEMV keeps the activations in shared memory
    and reads them per code word (MB = 4 or 8 token groups)."""
    w = synthetic.weights(N, K, sigma=0.02, seed=N + K + M)
    a = synthetic.activations(M, K, seed=M + 7)
    if bits == 4:
        c, s, z, w_hat = oracle_w4(u16(w), g)
        y = qz.qz_w4a16_gemv(a.to(dev), to_dev_u8(c, dev), to_dev_bf16(s, dev),
                             to_dev_u8(z, dev), N, K, g)
    else:
        c, s, _ = oracle.quantize_pack(u16(w), 8, True, K)
        w_hat = oracle.dequantize(c, s, None, N, K, 8, True, K)
        y = qz.qz_w8a16_gemv(a.to(dev), to_dev_u8(c, dev), to_dev_bf16(s, dev), N, K)
    torch.cuda.synchronize()
    assert qz.qz_device_status() == 0
    y_ref, abs_ref = oracle.matmul_f64(u16(a), w_hat)
    check_tolerance(u16(y), y_ref, abs_ref, f"wide gemv bits={bits} M={M} N={N} K={K}")


@pytest.mark.parametrize("bits", [4, 8])
def test_gemv_wide_onehot_is_exact(dev, bits):
    """64 one-hot token rows read back 64 dequantized weights exactly."""
    N, K, g, M = 300, 1024, 128, 64
    w = synthetic.weights(N, K, sigma=0.02, seed=15)
    if bits == 4:
        c, s, z, w_hat = oracle_w4(u16(w), g)
    else:
        c, s, z = oracle.quantize_pack(u16(w), 8, True, K)
        w_hat = oracle.dequantize(c, s, None, N, K, 8, True, K)
    ks = np.random.default_rng(2).choice(K, size=M, replace=False)
    a = np.zeros((M, K), np.uint16)
    a[np.arange(M), ks] = 0x3F80
    if bits == 4:
        y = qz.qz_w4a16_gemv(to_dev_bf16(a, dev), to_dev_u8(c, dev), to_dev_bf16(s, dev),
                             to_dev_u8(z, dev), N, K, g)
    else:
        y = qz.qz_w8a16_gemv(to_dev_bf16(a, dev), to_dev_u8(c, dev), to_dev_bf16(s, dev), N, K)
    torch.cuda.synchronize()
    assert np.array_equal(u16(y), w_hat[:, ks].T)


def test_gemv_workspace_is_left_zeroed_and_results_repeat(dev):
    N, K, g, M = 4096, 4096, 128, 4
    nbytes = qz.qz_workspace_bytes(qz.QZ_OP_W4A16_GEMV, M, N, K, g)
    assert nbytes > 0
    w = synthetic.weights(N, K, seed=9, device=dev)
    a = synthetic.activations(M, K, seed=9, device=dev)
    c, s, z = qz.qz_quantize_pack(w, 4, False, g)
    ws = torch.zeros(nbytes, dtype=torch.uint8, device=dev)
    y1 = qz.qz_w4a16_gemv(a, c, s, z, N, K, g, workspace=ws)
    y2 = qz.qz_w4a16_gemv(a, c, s, z, N, K, g, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))
    # the counter region (after the partials) must be zero again
    subtasks = (N + 31) // 32                    # one counter per 32-row subtask
    plan_partials = nbytes - (-(-subtasks // 64)) * 64 * 4
    assert int(ws[plan_partials:].count_nonzero()) == 0


@pytest.mark.parametrize("overlap", [0, 1])
def test_gemv_large_layer_results_repeat_back_to_back(dev, overlap):
    """Decode GEMVs on a 70B-sized layer (28672 x 8192, int4 g128), M = 1
    and M = 8, launched back to back into separate outputs: the split-K sums
    are added in a fixed order, so every launch must give the same bits.  A
    consumer that released a ring stage before its shared-memory loads had
    returned would let the refill corrupt scattered tasks, differently on
    every launch."""
    N, K, g = 28672, 8192, 128
    w = synthetic.weights(N, K, sigma=0.015, seed=4, device=dev)
    c, s, z = qz.qz_quantize_pack(w, 4, False, g)
    qz.qz_set_launch_overlap(overlap)
    try:
        for M in (1, 8):
            a = synthetic.activations(M, K, seed=M, device=dev)
            nbytes = qz.qz_workspace_bytes(qz.QZ_OP_W4A16_GEMV, M, N, K, g)
            ws = torch.zeros(max(nbytes, 1), dtype=torch.uint8, device=dev)
            ys = [qz.qz_w4a16_gemv(a, c, s, z, N, K, g, workspace=ws) for _ in range(6)]
            torch.cuda.synchronize()
            for y in ys[1:]:
                assert torch.equal(y.view(torch.int16), ys[0].view(torch.int16)), M
    finally:
        qz.qz_set_launch_overlap(0)              # the library's default
    assert qz.qz_device_status() == 0


def test_explicit_side_stream_with_temporary_workspaces(dev):
    """Calls given an explicit side stream and no workspace: the binding
    allocates and zero-fills each temporary workspace, and the output, on
    that stream, so the fill is ordered before the kernel and the memory is
    not handed out again while the kernel still runs.  Results equal those of
    the same calls on the current stream."""
    N, K, g = 4096, 4096, 128
    w = synthetic.weights(N, K, seed=12, device=dev)
    c, s, z = qz.qz_quantize_pack(w, 4, False, g)
    a4 = synthetic.activations(4, K, seed=13, device=dev)
    a48 = synthetic.activations(48, K, seed=14, device=dev)
    assert qz.qz_workspace_bytes(qz.QZ_OP_W4A16_GEMV, 4, N, K, g) > 0
    assert qz.qz_workspace_bytes(qz.QZ_OP_W4A16_GEMM, 48, N, K, g) > 0
    ref_v = qz.qz_w4a16_gemv(a4, c, s, z, N, K, g)
    ref_m = qz.qz_w4a16_gemm(a48, c, s, z, N, K, g)
    torch.cuda.synchronize()
    side = torch.cuda.Stream(dev)
    side.wait_stream(torch.cuda.current_stream(dev))
    got = []
    for _ in range(4):
        got.append(qz.qz_w4a16_gemv(a4, c, s, z, N, K, g, stream=side))
        got.append(qz.qz_w4a16_gemm(a48, c, s, z, N, K, g, stream=side))
    side.synchronize()
    assert qz.qz_device_status() == 0
    for i, y in enumerate(got):
        assert torch.equal(y.view(torch.int16), (ref_v if i % 2 == 0 else ref_m).view(torch.int16))


def test_outputs_stay_inside_their_buffers(dev):
    """Guard bands around every output must be untouched (a stand-in for a
    memory checker, which this pool does not offer)."""
    N, K, g, M = 300, 1024, 128, 3
    pad = 4096
    w = synthetic.weights(N, K, seed=4, device=dev)
    a = synthetic.activations(M, K, seed=4, device=dev)

    def guarded(nbytes):
        buf = torch.full((nbytes + 2 * pad,), 0xA5, dtype=torch.uint8, device=dev)
        return buf, buf[pad:pad + nbytes]

    cb, sb, zb = qz.qz_packed_bytes(N, K, 4, False, g)
    cbuf, cv = guarded(cb)
    sbuf, sv = guarded(sb)
    zbuf, zv = guarded(zb)
    qz.qz_quantize_pack(w, 4, False, g, codes=cv, scales=sv.view(torch.bfloat16), zeros=zv)
    ybuf, yv = guarded(M * N * 2)
    qz.qz_w4a16_gemv(a, cv, sv.view(torch.bfloat16), zv, N, K, g, y=yv.view(torch.bfloat16))
    dbuf, dv = guarded(N * K * 2)
    qz.qz_dequantize(cv, sv.view(torch.bfloat16), zv, N, K, 4, False, g, out=dv.view(torch.bfloat16))
    torch.cuda.synchronize()
    for buf in (cbuf, sbuf, zbuf, ybuf, dbuf):
        assert bool((buf[:pad] == 0xA5).all()) and bool((buf[-pad:] == 0xA5).all())


# ---------------------------------------------------------------------------
# Full-size configurations, checked on sampled rows
# ---------------------------------------------------------------------------

def sample_rows(N, count, seed):
    rng = np.random.default_rng(seed)
    rows = set(rng.choice(N, size=min(count, N), replace=False).tolist())
    rows.update({0, N - 1})
    return np.array(sorted(rows))


def check_layer_sampled(dev, N, K, M, sigma, seed, bits, sym, g, rows=48):
    w = synthetic.weights(N, K, sigma=sigma, seed=seed, device=dev)
    a = synthetic.activations(M, K, seed=seed + 1000, device=dev)
    ws = qz.Workspace(dev)
    c, s, z = qz.qz_quantize_pack(w, bits, sym, g, workspace=ws)
    if bits == 4:
        y = qz.qz_w4a16_gemv(a, c, s, z, N, K, g, workspace=ws)
    else:
        y = qz.qz_w8a16_gemv(a, c, s, N, K, workspace=ws)
    torch.cuda.synchronize()
    idx = sample_rows(N, rows, seed)
    ti = torch.from_numpy(idx).to(dev)
    w_rows = u16(w.index_select(0, ti))
    ref = oracle.quantize_pack(w_rows, bits, sym, g)
    got = (u8(c.index_select(0, ti)), u16(s.index_select(0, ti)),
           None if z is None else u8(z.index_select(0, ti)))
    assert_quant_equal(got, ref)
    w_hat = oracle.dequantize(*ref, len(idx), K, bits, sym, g)
    y_ref, abs_ref = oracle.matmul_f64(u16(a), w_hat)
    return check_tolerance(u16(y)[:, idx], y_ref, abs_ref, f"N={N} K={K} M={M} bits={bits}")


def test_tiny_config_full(dev):
    """1024 x 1024, M = 1, seed 0: every code and every output."""
    N, K = 1024, 1024
    w = synthetic.weights(N, K, sigma=0.02, seed=0)
    a = synthetic.activations(1, K, seed=0)
    ref = oracle.quantize_pack(u16(w), 4, False, 128)
    got = gpu_quantize(w.to(dev), 4, False, 128)
    assert_quant_equal(got, ref)
    w_hat = oracle.dequantize(*ref, N, K, 4, False, 128)
    y_ref, abs_ref = oracle.matmul_f64(u16(a), w_hat)
    c, s, z = (to_dev_u8(got[0], dev), to_dev_bf16(got[1], dev), to_dev_u8(got[2], dev))
    y = qz.qz_w4a16_gemv(a.to(dev), c, s, z, N, K, 128)
    torch.cuda.synchronize()
    check_tolerance(u16(y), y_ref, abs_ref, "tiny")


@pytest.mark.parametrize("li,NK", list(enumerate(synthetic.DECODE_7B)))
def test_decode_7b_layers(dev, li, NK):
    N, K = NK
    check_layer_sampled(dev, N, K, 1, 0.02, 1 + li, 4, False, 128)


@pytest.mark.parametrize("M", synthetic.DECODE_70B_M)
@pytest.mark.parametrize("li,NK", list(enumerate(synthetic.DECODE_70B)))
@pytest.mark.parametrize("bits", [4, 8])
def test_decode_70b_layers(dev, M, li, NK, bits):
    N, K = NK
    sym = bits == 8
    g = 128 if bits == 4 else K
    check_layer_sampled(dev, N, K, M, 0.015, 4 + li, bits, sym, g, rows=24)


# ---------------------------------------------------------------------------
# Prefill GEMM (tcgen05)
# ---------------------------------------------------------------------------

GEMM_CASES = [  # (M, N, K, g); most have fewer tiles than CTAs, so CTAs share tiles' K steps
    (17, 128, 128, 128), (100, 200, 256, 64), (256, 128, 1024, 128),
    (300, 1000, 1024, 128), (512, 384, 2048, 256), (257, 130, 640, 128),
    (64, 256, 640, 640), (96, 192, 384, 192),      # groups of 10 and 3 stages
    (32, 1024, 4096, 128), (200, 512, 2048, 128),  # partial token tiles over many CTAs
    # on 148 SMs: 158 tiles, the last 10 (one token each) shared by 60 CTAs
    # after a whole wave; 16 full-token tiles over 148 CTAs; N % 4 == 2
    # (element-wise stores); 16 tiles of 64 K steps over 96 CTAs; 48 tokens
    # (paired CTAs: 8 tiles over 296)
    (257, 10112, 4096, 128), (512, 1024, 4096, 64), (257, 2050, 4096, 128), (300, 1000, 4096, 128),
    (48, 1024, 4096, 128),
    # one tile of 80 or 112 tokens shared by six CTAs
    (80, 100, 8192, 128), (112, 100, 8192, 128),
]


@pytest.mark.parametrize("M,N,K,g", GEMM_CASES)
def test_w4a16_gemm_tolerance(dev, M, N, K, g):
    w = synthetic.weights(N, K, sigma=0.02, seed=M + N + K)
    a = synthetic.activations(M, K, seed=M * 5)
    c, s, z, w_hat = oracle_w4(u16(w), g)
    y_ref, abs_ref = oracle.matmul_f64(u16(a), w_hat)
    y = qz.qz_w4a16_gemm(a.to(dev), to_dev_u8(c, dev), to_dev_bf16(s, dev), to_dev_u8(z, dev),
                         N, K, g)
    torch.cuda.synchronize()
    assert qz.qz_device_status() == 0
    check_tolerance(u16(y), y_ref, abs_ref, f"gemm M={M} N={N} K={K} g={g}")


@pytest.mark.parametrize("bits,M,N,K", [(4, 48, 1024, 4096), (8, 48, 1024, 4096),
                                         (4, 257, 10112, 4096), (8, 512, 1024, 4096)])
def test_gemm_split_k_repeats_and_leaves_workspace_zeroed(dev, bits, M, N, K):
    """Partials of shared tiles are added in K order: the same inputs give the
    same bits on every call, and each call leaves the arrival counters at
    zero (short token tiles over many CTAs; whole waves plus a shared tail)."""
    g = 128
    assert qz.qz_workspace_bytes(qz.QZ_OP_W4A16_GEMM, M, N, K, g) > 0
    w = synthetic.weights(N, K, sigma=0.02, seed=41, device=dev)
    a = synthetic.activations(M, K, seed=42, device=dev)
    ws = torch.zeros(qz.qz_workspace_bytes(qz.QZ_OP_W4A16_GEMM, M, N, K, g), dtype=torch.uint8,
                     device=dev)
    if bits == 4:
        c, s, z = qz.qz_quantize_pack(w, 4, False, g)
        run = lambda: qz.qz_w4a16_gemm(a, c, s, z, N, K, g, workspace=ws)
    else:
        c, s, _ = qz.qz_quantize_pack(w, 8, True, K)
        run = lambda: qz.qz_w8a16_gemm(a, c, s, N, K, workspace=ws)
    ys = [run() for _ in range(3)]
    torch.cuda.synchronize()
    assert qz.qz_device_status() == 0
    assert all(torch.equal(ys[0], yi) for yi in ys[1:])
    # the counters after the partials (one block of 64: at most 64 shared
    # tiles here) are back to zero; the layout is the one for this device's
    # SM count
    sms = min(torch.cuda.get_device_properties(dev).multi_processor_count, 148)
    used = qz.qz_workspace_bytes_for_sms(qz.QZ_OP_W4A16_GEMM, M, N, K, g, sms)
    assert used > 0
    assert int(ws[used - 64 * 4:used].count_nonzero()) == 0


def test_w4a16_gemm_onehot_is_exact(dev):
    """One-hot token rows read back single dequantized weights exactly."""
    M, N, K, g = 256, 256, 1024, 128
    w = synthetic.weights(N, K, sigma=0.02, seed=77)
    c, s, z, w_hat = oracle_w4(u16(w), g)
    ks = np.arange(M) * (K // M) + (np.arange(M) % (K // M))
    a = np.zeros((M, K), np.uint16)
    a[np.arange(M), ks] = 0x3F80
    y = qz.qz_w4a16_gemm(to_dev_bf16(a, dev), to_dev_u8(c, dev), to_dev_bf16(s, dev),
                         to_dev_u8(z, dev), N, K, g)
    torch.cuda.synchronize()
    assert np.array_equal(u16(y), w_hat[:, ks].T)


def test_prefill_config_sampled(dev):
    """M = 2048 tokens, N = K = 8192, seed 6: sampled weight rows, all tokens."""
    cfg = synthetic.PREFILL
    M, N, K = cfg["M"], cfg["N"], cfg["K"]
    w = synthetic.weights(N, K, sigma=cfg["sigma"], seed=cfg["seed"], device=dev)
    a = synthetic.activations(M, K, seed=cfg["seed"] + 1000, device=dev)
    c, s, z = qz.qz_quantize_pack(w, 4, False, 128)
    y = qz.qz_w4a16_gemm(a, c, s, z, N, K, 128)
    torch.cuda.synchronize()
    assert qz.qz_device_status() == 0
    idx = sample_rows(N, 24, 6)
    ti = torch.from_numpy(idx).to(dev)
    ref = oracle.quantize_pack(u16(w.index_select(0, ti)), 4, False, 128)
    got = (u8(c.index_select(0, ti)), u16(s.index_select(0, ti)), u8(z.index_select(0, ti)))
    assert_quant_equal(got, ref)
    w_hat = oracle.dequantize(*ref, len(idx), K, 4, False, 128)
    y_ref, abs_ref = oracle.matmul_f64(u16(a), w_hat)
    check_tolerance(u16(y)[:, idx], y_ref, abs_ref, "prefill 2048x8192x8192")


W8_GEMM_CASES = [  # (M, N, K): ragged token and row tiles, N % 8 != 0 (direct stores)
    (17, 128, 128), (100, 200, 256), (256, 128, 1024), (300, 1000, 1024),
    (257, 130, 640), (512, 384, 2048), (64, 36, 384), (257, 10112, 4096),
]


@pytest.mark.parametrize("M,N,K", W8_GEMM_CASES)
def test_w8a16_gemm_tolerance(dev, M, N, K):
    w = synthetic.weights(N, K, sigma=0.015, seed=M + 2 * N + K)
    a = synthetic.activations(M, K, seed=M * 7)
    c, s, _ = oracle.quantize_pack(u16(w), 8, True, K)
    w_hat = oracle.dequantize(c, s, None, N, K, 8, True, K)
    y_ref, abs_ref = oracle.matmul_f64(u16(a), w_hat)
    y = qz.qz_w8a16_gemm(a.to(dev), to_dev_u8(c, dev), to_dev_bf16(s, dev), N, K)
    torch.cuda.synchronize()
    assert qz.qz_device_status() == 0
    check_tolerance(u16(y), y_ref, abs_ref, f"w8 gemm M={M} N={N} K={K}")


def test_w8a16_gemm_onehot_is_exact(dev):
    """One-hot token rows read back single dequantized int8 weights exactly,
    including the extreme codes +-127 of every row."""
    M, N, K = 256, 256, 1024
    w = synthetic.weights(N, K, sigma=0.015, seed=78)
    c, s, _ = oracle.quantize_pack(u16(w), 8, True, K)
    w_hat = oracle.dequantize(c, s, None, N, K, 8, True, K)
    ks = np.arange(M) * (K // M) + (np.arange(M) % (K // M))
    a = np.zeros((M, K), np.uint16)
    a[np.arange(M), ks] = 0x3F80
    y = qz.qz_w8a16_gemm(to_dev_bf16(a, dev), to_dev_u8(c, dev), to_dev_bf16(s, dev), N, K)
    torch.cuda.synchronize()
    assert np.array_equal(u16(y), w_hat[:, ks].T)
    # the column of each row's extreme code
    kx = np.abs(c.view(np.int8).astype(np.int32)).argmax(axis=1)[:M]
    a2 = np.zeros((M, K), np.uint16)
    a2[np.arange(M), kx] = 0x3F80
    y2 = qz.qz_w8a16_gemm(to_dev_bf16(a2, dev), to_dev_u8(c, dev), to_dev_bf16(s, dev), N, K)
    torch.cuda.synchronize()
    assert np.array_equal(u16(y2), w_hat[:, kx].T)


@pytest.mark.parametrize("M", [1, 8, 256])
def test_w8a16_onehot_exact_across_the_scale_range(dev, M):
    """int8 scales from the smallest to the largest a finite bf16 weight can
    give (S = absmax / 127 up to about 2.7e36, down to subnormal bf16): the
    dequantized weight S*q is formed exactly and rounded once for every row,
    with no overflow of an intermediate, in the decode GEMV (M <= 32) and the
    tcgen05 GEMM."""
    N, K = 256, 512
    w = synthetic.weights(N, K, sigma=0.5, seed=91).float().numpy().astype(np.float64)
    # row magnitudes spread over the whole bf16 exponent range
    exps = np.linspace(-128, 126, N)
    w = np.clip(w * np.exp2(exps)[:, None], -3.3e38, 3.3e38)
    w = u16(torch.tensor(w, dtype=torch.float32).to(torch.bfloat16))
    c, s, _ = oracle.quantize_pack(w, 8, True, K)
    w_hat = oracle.dequantize(c, s, None, N, K, 8, True, K)
    ks = (np.arange(M) * 37) % K
    a = np.zeros((M, K), np.uint16)
    a[np.arange(M), ks] = 0x3F80
    fn = qz.qz_w8a16_gemv if M <= 32 else qz.qz_w8a16_gemm
    y = fn(to_dev_bf16(a, dev), to_dev_u8(c, dev), to_dev_bf16(s, dev), N, K)
    torch.cuda.synchronize()
    assert np.array_equal(u16(y), w_hat[:, ks].T)


def test_w8a16_gemm_small_m_matches_the_gemv(dev):
    """M <= 32 takes the decode kernel: the same bits as qz_w8a16_gemv."""
    N, K = 1000, 1024
    w = synthetic.weights(N, K, sigma=0.015, seed=5)
    c, s, _ = oracle.quantize_pack(u16(w), 8, True, K)
    cd, sd = to_dev_u8(c, dev), to_dev_bf16(s, dev)
    for M in (1, 16, 17, 32):
        a = synthetic.activations(M, K, seed=M).to(dev)
        y1 = qz.qz_w8a16_gemm(a, cd, sd, N, K)
        y2 = qz.qz_w8a16_gemv(a, cd, sd, N, K)
        torch.cuda.synchronize()
        assert torch.equal(y1, y2)


def test_w8a16_prefill_sampled(dev):
    """M = 2048 tokens, N = K = 8192 int8 per-channel: sampled rows, all tokens."""
    cfg = synthetic.PREFILL
    M, N, K = cfg["M"], cfg["N"], cfg["K"]
    w = synthetic.weights(N, K, sigma=cfg["sigma"], seed=cfg["seed"], device=dev)
    a = synthetic.activations(M, K, seed=cfg["seed"] + 1000, device=dev)
    c, s, _ = qz.qz_quantize_pack(w, 8, True, K)
    y = qz.qz_w8a16_gemm(a, c, s, N, K)
    torch.cuda.synchronize()
    assert qz.qz_device_status() == 0
    idx = sample_rows(N, 24, 8)
    ti = torch.from_numpy(idx).to(dev)
    ref = oracle.quantize_pack(u16(w.index_select(0, ti)), 8, True, K)
    got = (u8(c.index_select(0, ti)), u16(s.index_select(0, ti)), None)
    assert_quant_equal(got, ref)
    w_hat = oracle.dequantize(*ref, len(idx), K, 8, True, K)
    y_ref, abs_ref = oracle.matmul_f64(u16(a), w_hat)
    check_tolerance(u16(y)[:, idx], y_ref, abs_ref, "w8 prefill 2048x8192x8192")


def test_gemm_bounded_wait_reports_timeout_and_recovers(dev):
    """A 1 ns wait bound makes the first pipeline wait run out: the kernel
    must return with the error word set (no hang, no fault), and the next call
    with the default bound must be correct again."""
    M, N, K, g = 256, 256, 2048, 128
    w = synthetic.weights(N, K, seed=3, device=dev)
    a = synthetic.activations(M, K, seed=3, device=dev)
    c, s, z = qz.qz_quantize_pack(w, 4, False, g)
    assert qz.qz_device_status() == 0
    qz.qz_set_device_wait_limit(1)
    try:
        qz.qz_w4a16_gemm(a, c, s, z, N, K, g)
        st = qz.qz_device_status()
    finally:
        qz.qz_set_device_wait_limit(0)
    assert st == qz.QZ_ERR_DEVICE_TIMEOUT
    assert qz.qz_device_status() == 0                      # cleared by the read
    y = qz.qz_w4a16_gemm(a, c, s, z, N, K, g)
    torch.cuda.synchronize()
    assert qz.qz_device_status() == 0
    wb = u16(w)
    cref, sref, zref, w_hat = oracle_w4(wb, g)
    y_ref, abs_ref = oracle.matmul_f64(u16(a), w_hat)
    check_tolerance(u16(y), y_ref, abs_ref, "gemm after timeout")


@pytest.mark.parametrize("bits,sym", FORMATS)
@pytest.mark.parametrize("g", [128, 0, 4096])
def test_quantize_dense_bit_exact(dev, bits, sym, g):
    """2M values in one comparison.  About 0.3% of them land exactly on a
    half-way point of their group's grid, so the tie handling of the
    division-free path (round half to even) runs thousands of times."""
    N, K = 512, 4096
    w = synthetic.weights(N, K, sigma=0.02, seed=900 + bits + 2 * int(sym))
    ref = oracle.quantize_pack(u16(w), bits, sym, g)
    got = gpu_quantize(w.to(dev), bits, sym, g)
    assert_quant_equal(got, ref)


def _bf16_step(x, d):
    """The bf16 value d representable steps away from bf16 x (x > 0)."""
    b = np.array([x], np.float32).view(np.uint32)[0] >> 16
    return float(np.array([(int(b) + d) << 16], np.uint32).view(np.float32)[0])


def test_quantize_near_half_way_values(dev):
    """Values placed exactly on, and one bf16 step either side of, every
    half-way point of a group whose scale is exactly 1 (range [0, 15])."""
    K = 128
    vals = [0.0, 15.0]
    for j in range(15):
        h = j + 0.5
        vals += [h, _bf16_step(h, 1), _bf16_step(h, -1)]
    row = np.zeros(K, np.float32)
    row[:len(vals)] = vals
    w = torch.from_numpy(np.stack([row, -row[::-1].copy()])).to(torch.bfloat16)
    for bits, sym in FORMATS:
        for g in (128, 0):
            ref = oracle.quantize_pack(u16(w), bits, sym, g)
            got = gpu_quantize(w.to(dev), bits, sym, g)
            assert_quant_equal(got, ref)


@pytest.mark.parametrize("bits", [4, 8])
def test_gemv_launch_overlap_modes_agree(dev, bits):
    """Both launch-overlap modes give bit-identical results, also when GEMVs
    follow each other on the stream (each reads the previous one's output)."""
    N, K, M = 4096, 4096, 4
    w = synthetic.weights(N, K, sigma=0.02, seed=71).to(dev)
    if bits == 4:
        c, s, z = qz.qz_quantize_pack(w, 4, False, 128)
        run = lambda a: qz.qz_w4a16_gemv(a, c, s, z, N, K, 128)
    else:
        c, s, _ = qz.qz_quantize_pack(w, 8, True, K)
        run = lambda a: qz.qz_w8a16_gemv(a, c, s, N, K)
    a0 = synthetic.activations(M, K, seed=72, device=dev)
    outs = {}
    try:
        for mode in (0, 1):
            qz.qz_set_launch_overlap(mode)
            a = a0
            for _ in range(4):            # chained: each GEMV consumes the previous one's output
                a = run(a)
            torch.cuda.synchronize()
            outs[mode] = u16(a)
    finally:
        qz.qz_set_launch_overlap(0)
    assert np.array_equal(outs[0], outs[1])


@pytest.mark.parametrize("bits,sym", FORMATS)
def test_dequantize_leftover_chunks_bit_exact(dev, bits, sym):
    """N * K / 8 = 15 chunks: three groups of four and three left over."""
    N, K = 3, 40
    w = synthetic.weights(N, K, sigma=0.02, seed=91)
    for g in (8, 40, 0):
        c, s, z = oracle.quantize_pack(u16(w), bits, sym, g)
        ref = oracle.dequantize(c, s, z, N, K, bits, sym, g)
        out = qz.qz_dequantize(to_dev_u8(c, dev), to_dev_bf16(s, dev),
                               None if z is None else to_dev_u8(z, dev), N, K, bits, sym, g)
        torch.cuda.synchronize()
        assert np.array_equal(u16(out), ref), (bits, sym, g)
