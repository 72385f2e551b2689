"""Checks that pin the CPU oracle to facts fixed outside the oracle itself.

Each ``pin_*`` function raises ``AssertionError`` on a mismatch.  They are
collected by ``test_oracle_pins.py`` and re-run against deliberately broken
copies of the oracle by ``test_oracle_mutants.py`` (each planted mistake must
trip at least one pin).

Sources of truth used here, none of which is the oracle:
  * numbers printed on the pages (``golden/worked_examples.json``);
  * exact rational arithmetic (``fractions.Fraction``) for the closed forms
    q = nearest integer to x/S + Z, |x - S(q - Z)| <= S/2;
  * library routines: torch's fp32->bf16 conversion (RNE), numpy fp32/fp64
    arithmetic and matmul;
  * brute force over every code of tiny groups.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden",
                      "worked_examples.json")

FORMATS = [(4, False), (4, True), (8, False), (8, True)]


def golden():
    with open(GOLDEN) as f:
        return json.load(f)


def _bf16_value(bits: int) -> float:
    return float(np.array([bits << 16], dtype=np.uint32).view(np.float32)[0])


def _as_int_codes(codes, N, K, bits, symmetric):
    """Unpack codes to signed/unsigned integers, N x K (nibble order per the
    packing figure: even k in the low nibble)."""
    codes = np.asarray(codes, dtype=np.uint8)
    if bits == 8:
        return codes.view(np.int8).astype(np.int64).reshape(N, K)
    lo = (codes & 0x0F).astype(np.int64)
    hi = (codes >> 4).astype(np.int64)
    q = np.empty((N, K), dtype=np.int64)
    q[:, 0::2] = lo
    q[:, 1::2] = hi
    if symmetric:
        q = np.where(q >= 8, q - 16, q)
    return q


def _zeros_int(zeros, bits, symmetric, shape):
    if symmetric:
        return np.zeros(shape, dtype=np.int64)
    z = np.asarray(zeros, dtype=np.uint8)
    if bits == 8:
        return z.view(np.int8).astype(np.int64).reshape(shape)
    return z.astype(np.int64).reshape(shape)


def _bf16_round(values_f32: np.ndarray) -> np.ndarray:
    """bf16 bits of fp32 values via torch's conversion (round to nearest even)."""
    t = torch.from_numpy(np.ascontiguousarray(values_f32, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _random_bf16(shape, sigma, seed, outliers=True):
    g = torch.Generator().manual_seed(seed)
    w = torch.randn(shape, generator=g) * sigma
    if outliers:
        mask = torch.rand(shape, generator=g) < 1e-3
        w[mask] *= 20
    return w.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


# --------------------------------------------------------------------------
# Worked examples printed on the pages
# --------------------------------------------------------------------------

def pin_asym_int8_worked_example():
    """-1.8..2.4 onto int8: S ~ 0.0165, Z = -19, 0.5 -> 11 -> ~0.494 (error ~0.006);
    the range figure also puts -1.8 at -128, 0.0 at -19 and 2.4 at 127."""
    g = golden()["asym_int8"]
    lo, hi = g["range"]
    x = np.array([[lo, 0.0, g["x"], hi]], dtype=np.float32)
    codes, scales, zeros = oracle.quantize_pack(x, bits=8, symmetric=False, group_size=4)
    S = _bf16_value(int(scales[0, 0]))
    Z = int(zeros.view(np.int8)[0, 0])
    q = codes.view(np.int8)[0].astype(int).tolist()
    assert round(S, g["S_printed_decimals"]) == g["S_approx"], S
    assert Z == g["Z"], Z
    assert q == [-128, g["Z"], g["q"], 127], q
    w_hat = oracle.dequantize(codes, scales, zeros, 1, 4, bits=8, symmetric=False,
                              group_size=4)
    x_hat = _bf16_value(int(w_hat[0, 2]))
    assert round(x_hat, g["printed_decimals"]) == g["x_hat_approx"], x_hat
    assert round(abs(g["x"] - x_hat), g["printed_decimals"]) == g["error_approx"]


def pin_absmax_int8_ibm_example():
    """IBM vector, absmax 6.2 onto -127..127 (factor 127/6.2 ~ 20.5)."""
    g = golden()["absmax_int8"]
    x = np.array([g["x"]], dtype=np.float32)
    codes, scales, zeros = oracle.quantize_pack(x, bits=8, symmetric=True,
                                                group_size=len(g["x"]))
    assert zeros is None
    assert codes.view(np.int8)[0].astype(int).tolist() == g["q"]
    S = _bf16_value(int(scales[0, 0]))
    assert round(1.0 / S, 1) == g["scale_factor_approx"]
    assert round(g["qmax"] / g["absmax"], 1) == g["scale_factor_approx"]


def pin_nibble_order():
    """Packing figure: val1 (0101) low nibble, val2 (0011) high nibble."""
    g = golden()["nibble_packing"]
    # a group spanning [0, 15] has S = 1, Z = 0, so q equals x.
    x = np.array([[g["val1"], g["val2"], 15.0, 0.0]], dtype=np.float32)
    codes, scales, zeros = oracle.quantize_pack(x, bits=4, symmetric=False, group_size=4)
    assert _bf16_value(int(scales[0, 0])) == 1.0 and int(zeros[0, 0]) == 0
    assert int(codes[0, 0]) == g["byte"], hex(int(codes[0, 0]))
    assert int(codes[0, 1]) == 0x0F


def pin_code_ranges():
    g = golden()["int_ranges"]
    assert list(oracle.code_range(8, False)) == g["int8_asym"]
    assert list(oracle.code_range(8, True)) == g["int8_sym"]
    lo, hi = oracle.code_range(4, False)
    assert hi - lo + 1 == g["int4_count"]
    lo, hi = oracle.code_range(4, True)
    assert hi - lo + 1 <= g["int4_count"] and lo == -hi


def pin_sizes():
    """Bytes per parameter 2 / 1 / 0.5 -> 70B: 140 / 70 / 35 GB; 175B fp16 ~326 GB
    (the GPTQ page's figure is in GiB); group-128 metadata adds 3 bytes/group."""
    g = golden()["sizes"]
    N, K = 5_468_750, 12_800                 # 70e9 parameters, K % 128 == 0
    assert N * K == g["params_70b"]
    assert N * K * 2 / 1e9 == g["bf16_gb"]
    (c8, s8, z8) = oracle.packed_shapes(N, K, 8, True, K)
    (c4, s4, z4) = oracle.packed_shapes(N, K, 4, False, 128)
    assert math.prod(c8) / 1e9 == g["int8_gb"]
    assert math.prod(c4) / 1e9 == g["int4_gb"]
    meta = math.prod(s4) * 2 + math.prod(z4) * 1
    assert meta == g["params_70b"] / g["group_size_gptq_default"] * 3
    assert round(g["params_175b"] * 2 / 2**30) == g["fp16_175b_gb_printed"]
    # the oracle writes exactly those buffers
    w = _random_bf16((8, 256), 0.02, 1)
    c, s, z = oracle.quantize_pack(w, 4, False, 128)
    assert c.nbytes == 8 * 256 // 2 and s.nbytes == 8 * 2 * 2 and z.nbytes == 8 * 2


# --------------------------------------------------------------------------
# Closed forms and invariants
# --------------------------------------------------------------------------

def _check_format_invariants(w_bits, bits, symmetric, group_size, exact_rounding=True):
    N, K = w_bits.shape
    x = oracle.bf16_bits_to_f32(w_bits).astype(np.float64)
    codes, scales, zeros = oracle.quantize_pack(w_bits, bits, symmetric, group_size)
    q = _as_int_codes(codes, N, K, bits, symmetric)
    qmin, qmax = oracle.code_range(bits, symmetric)
    assert q.min() >= qmin and q.max() <= qmax
    gs = K if group_size == 0 else group_size
    if group_size == 0:
        S = np.full((N, K), _bf16_value(int(scales[0])), dtype=np.float64)
        Z = np.full((N, K), int(_zeros_int(zeros, bits, symmetric, (1,))[0]))
    else:
        sv = oracle.bf16_bits_to_f32(scales).astype(np.float64)
        S = np.repeat(sv, gs, axis=1)
        Z = np.repeat(_zeros_int(zeros, bits, symmetric, scales.shape), gs, axis=1)
    assert (Z >= qmin).all() and (Z <= qmax).all()
    # scale = smallest bf16 >= fp32 (range / code span), computed with numpy fp32
    xs = x.reshape(-1) if group_size == 0 else x.reshape(N, K // gs, gs)
    if symmetric:
        a = np.abs(xs).max(axis=-1).astype(np.float32)
        s32 = (a / np.float32(qmax)).astype(np.float32)
    else:
        mn = np.minimum(xs.min(axis=-1), 0).astype(np.float32)
        mx = np.maximum(xs.max(axis=-1), 0).astype(np.float32)
        s32 = ((mx - mn) / np.float32(qmax - qmin)).astype(np.float32)
    s32 = np.where(s32 == 0, np.float32(1.0), s32).astype(np.float32)
    near = _bf16_round(s32)
    near_v = oracle.bf16_bits_to_f32(near)
    up = np.where(near_v >= s32, near, near + 1).astype(np.uint16)
    assert np.array_equal(up.reshape(np.asarray(scales).shape), np.asarray(scales)), \
        "stored scale is not the smallest bf16 >= S"
    # range figure of the guide's "Mapping values to fewer bits": the low end
    # of the range lands on q_min (the range is widened to contain 0.0, so a
    # group with no negative value has Z == q_min)
    if not symmetric:
        qg = q.reshape(-1) if group_size == 0 else q.reshape(N, K // gs, gs)
        Zg = Z.reshape(-1)[:1] if group_size == 0 else Z.reshape(N, K // gs, gs)[..., 0]
        lo = xs.min(axis=-1)
        at_lo = np.take_along_axis(qg, xs.argmin(axis=-1)[..., None], axis=-1)[..., 0]
        neg = lo < 0
        assert (at_lo[neg] == qmin).all(), "the range minimum does not map to q_min"
        assert (Zg[~neg] == qmin).all(), "a group without negatives needs Z == q_min"
    # round trip: every element within half a step of its reconstruction
    err = np.abs(x - S * (q - Z))
    assert (err <= S / 2 * (1 + 1e-12)).all(), float((err / S).max())
    if exact_rounding:
        # q is the nearest code to x/S + Z (exact arithmetic), away from ties
        u = x / S + Z
        frac = u - np.floor(u)
        safe = np.abs(frac - 0.5) > 2.0 ** -16
        nearest = np.clip(np.floor(u + 0.5), qmin, qmax)
        assert np.array_equal(q[safe], nearest[safe].astype(np.int64))
    return codes, scales, zeros, q


def pin_roundtrip_and_nearest_all_formats():
    for bits, symmetric in FORMATS:
        w = _random_bf16((16, 512), 0.02, 100 + bits + int(symmetric))
        for g in (128, 512, 0, 32):
            _check_format_invariants(w, bits, symmetric, g)


def pin_brute_force_every_code():
    """Groups built so that every code of the format is hit exactly."""
    for bits, symmetric in FORMATS:
        qmin, qmax = oracle.code_range(bits, symmetric)
        s = 2.0 ** -4
        z0 = 0 if symmetric else (5 if bits == 4 else -3)
        j = np.arange(qmin, qmax + 1)
        x = ((j - z0) * s).astype(np.float32)[None, :]
        if bits == 4 and x.shape[1] % 2:
            x = np.concatenate([x, np.zeros((1, 1), np.float32)], axis=1)
        K = x.shape[1]
        codes, scales, zeros = oracle.quantize_pack(x, bits, symmetric, K)
        q = _as_int_codes(codes, 1, K, bits, symmetric)[0, : len(j)]
        assert _bf16_value(int(scales[0, 0])) == s
        assert np.array_equal(q, j), (bits, symmetric)
        w_hat = oracle.dequantize(codes, scales, zeros, 1, K, bits, symmetric, K)
        assert np.array_equal(oracle.bf16_bits_to_f32(w_hat[0, : len(j)]), x[0, : len(j)])


def pin_brute_force_argmin_tiny_groups():
    """On tiny random groups, q is the argmin over all codes of |x/S + Z - j|
    in exact rational arithmetic (skipping near-ties, where fp32 decides)."""
    rng = np.random.default_rng(7)
    for bits, symmetric in FORMATS:
        qmin, qmax = oracle.code_range(bits, symmetric)
        for trial in range(40):
            vals = rng.normal(0, 1, size=(1, 8)).astype(np.float32)
            if trial % 4 == 0:
                vals = np.abs(vals)
            codes, scales, zeros = oracle.quantize_pack(vals, bits, symmetric, 8)
            q = _as_int_codes(codes, 1, 8, bits, symmetric)[0]
            S = Fraction(_bf16_value(int(scales[0, 0])))
            Z = 0 if symmetric else int(_zeros_int(zeros, bits, symmetric, (1,))[0])
            for xi, qi in zip(vals[0], q):
                u = Fraction(float(xi)) / S + Z
                d = sorted((abs(u - c), c) for c in range(qmin, qmax + 1))
                if d[1][0] - d[0][0] > Fraction(1, 2 ** 15):
                    assert qi == d[0][1], (bits, symmetric, float(xi), int(qi), d[0][1])


def pin_ties_to_even():
    """x/S + Z exactly half-way: 2.5 -> 2, 3.5 -> 4, 0.5 -> 0 (S = 1, Z = 0)."""
    x = np.array([[0.0, 15.0, 2.5, 3.5, 0.5, 14.5]], dtype=np.float32)
    codes, scales, zeros = oracle.quantize_pack(x, 4, False, 6)
    q = _as_int_codes(codes, 1, 6, 4, False)[0].tolist()
    assert q == [0, 15, 2, 4, 0, 14], q
    # range [-1.5, 13.5]: S = 1, Z = 2; 13.5 lands on 15.5, whose even
    # neighbour 16 is outside the code range, so the clamp returns 15.
    x = np.array([[-1.5, 13.5, 0.0, 5.0]], dtype=np.float32)
    codes, scales, zeros = oracle.quantize_pack(x, 4, False, 4)
    assert int(zeros[0, 0]) == 2
    q = _as_int_codes(codes, 1, 4, 4, False)[0].tolist()
    assert q == [0, 15, 2, 7], q


def pin_special_groups():
    K = 128
    # all-zero group: S := 1, Z = 0 (int4 asym: q_min - round(0)), w_hat = +0
    z = np.zeros((1, K), np.float32)
    for bits, symmetric in FORMATS:
        codes, scales, zeros = oracle.quantize_pack(z, bits, symmetric, K)
        assert int(scales[0, 0]) == 0x3F80
        q = _as_int_codes(codes, 1, K, bits, symmetric)
        Zv = _zeros_int(zeros, bits, symmetric, (1,))[0]
        qmin, _ = oracle.code_range(bits, symmetric)
        assert (q == Zv).all() and Zv == (0 if symmetric else qmin)
        w_hat = oracle.dequantize(codes, scales, zeros, 1, K, bits, symmetric, K)
        assert (w_hat == 0).all()
    # constant positive group: range [0, c] -> every value takes the top code
    c = np.full((1, K), 0.75, np.float32)
    codes, scales, zeros = oracle.quantize_pack(c, 4, False, K)
    assert (_as_int_codes(codes, 1, K, 4, False) == 15).all() and int(zeros[0, 0]) == 0
    # constant negative group: range [c, 0] -> bottom code, Z at the top
    codes, scales, zeros = oracle.quantize_pack(-c, 4, False, K)
    assert (_as_int_codes(codes, 1, K, 4, False) == 0).all() and int(zeros[0, 0]) == 15
    # one outlier among small values keeps the half-step bound
    w = _random_bf16((4, K), 0.02, 3, outliers=False)
    w[0, 5] = _bf16_round(np.array([1.5], np.float32))[0]
    _check_format_invariants(w, 4, False, 128)


def pin_granularity():
    """Per-group = consecutive values along a row; per-channel = one scale per
    row; per-tensor = one scale for the matrix."""
    w = _random_bf16((6, 512), 0.02, 11)
    c, s, z = oracle.quantize_pack(w, 4, False, 128)
    for n in (0, 5):
        for j in (0, 3):
            cg, sg, zg = oracle.quantize_pack(w[n:n + 1, j * 128:(j + 1) * 128], 4, False, 128)
            assert np.array_equal(cg[0], c[n, j * 64:(j + 1) * 64])
            assert sg[0, 0] == s[n, j] and zg[0, 0] == z[n, j]
    c, s, z = oracle.quantize_pack(w, 8, True, 512)
    assert s.shape == (6, 1) and z is None
    for n in range(6):
        cr, sr, _ = oracle.quantize_pack(w[n:n + 1], 8, True, 512)
        assert np.array_equal(cr[0], c[n]) and sr[0, 0] == s[n, 0]
    c, s, z = oracle.quantize_pack(w, 8, False, 0)
    assert s.shape == (1,)
    cf, sf, zf = oracle.quantize_pack(w.reshape(1, -1), 8, False, 6 * 512)
    assert np.array_equal(cf.reshape(c.shape), c) and sf[0, 0] == s[0] and zf[0, 0] == z[0]


# --------------------------------------------------------------------------
# Conversions and the matmul
# --------------------------------------------------------------------------

def pin_bf16_rne_matches_torch():
    rng = np.random.default_rng(3)
    b = rng.integers(0, 2 ** 32, size=4000, dtype=np.uint64).astype(np.uint32)
    b = b[(b & 0x7F800000) != 0x7F800000]                       # finite only
    ties = (b & 0xFFFF0000) | 0x8000                             # exact ties
    sub = b & 0x807FFFFF                                         # subnormals
    allb = np.concatenate([b, ties, sub]).astype(np.uint32)
    f = allb.view(np.float32)
    mine = np.array([oracle.f32_to_bf16_rne(float(v)) for v in f], dtype=np.uint16)
    assert np.array_equal(mine, _bf16_round(f))


def pin_bf16_round_up():
    rng = np.random.default_rng(4)
    s = np.abs(rng.normal(0, 1, 3000)).astype(np.float32) * np.float32(1e-3)
    s = np.concatenate([s, np.array([1.0, 0.0625, 2.0 ** -130, 3e-39], np.float32)])
    for v in s:
        if v == 0:
            continue
        b = oracle.f32_to_bf16_up(float(v))
        up = _bf16_value(b)
        below = _bf16_value(b - 1)
        assert up >= v and below < v, (v, up, below)


def pin_dequant_closed_form():
    rng = np.random.default_rng(5)
    for bits, symmetric in FORMATS:
        N, K, g = 8, 256, 64
        qmin, qmax = oracle.code_range(bits, symmetric)
        q = rng.integers(qmin, qmax + 1, size=(N, K))
        if bits == 4:
            nib = (q & 0xF).astype(np.uint8)
            codes = (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)
        else:
            codes = q.astype(np.int8).view(np.uint8)
        sv = np.abs(rng.normal(0, 1e-3, (N, K // g))).astype(np.float32) + np.float32(1e-6)
        scales = _bf16_round(sv)
        if symmetric:
            zeros, Z = None, np.zeros((N, K // g), np.int64)
        else:
            Z = rng.integers(qmin, qmax + 1, size=(N, K // g))
            zeros = Z.astype(np.int8 if bits == 8 else np.uint8).view(np.uint8)
        got = oracle.dequantize(codes, scales, zeros, N, K, bits, symmetric, g)
        Sf = np.repeat(oracle.bf16_bits_to_f32(scales).astype(np.float64), g, axis=1)
        exact = Sf * (q - np.repeat(Z, g, axis=1))                   # exact in fp64
        assert np.array_equal(exact.astype(np.float32).astype(np.float64), exact)
        assert np.array_equal(got, _bf16_round(exact.astype(np.float32)))


def pin_matmul_f64():
    rng = np.random.default_rng(6)
    M, N, K = 3, 17, 96
    a = _bf16_round(rng.normal(0, 1, (M, K)).astype(np.float32))
    w = _bf16_round(rng.normal(0, 0.02, (N, K)).astype(np.float32))
    y, ya = oracle.matmul_f64(a, w)
    af = oracle.bf16_bits_to_f32(a).astype(np.float64)
    wf = oracle.bf16_bits_to_f32(w).astype(np.float64)
    assert np.allclose(y, af @ wf.T, rtol=1e-12, atol=1e-15)
    assert np.allclose(ya, np.abs(af) @ np.abs(wf).T, rtol=1e-12, atol=1e-15)
    onehot = np.zeros((1, K), np.uint16)
    onehot[0, 7] = 0x3F80                                              # 1.0
    y1, _ = oracle.matmul_f64(onehot, w)
    assert np.array_equal(y1[0], wf[:, 7])
    y0, _ = oracle.matmul_f64(a, np.zeros((N, K), np.uint16))
    assert (y0 == 0).all()


def pin_tolerance_reaches_bf16_outputs():
    """The bound admits the correctly rounded bf16 of the exact product at
    every magnitude: at least half a bf16 spacing, 2^-9 |y| for normal
    outputs (inside 8e-3 |y|) and 2^-134 for subnormal ones."""
    rng = np.random.default_rng(11)
    for scale in (1e3, 1.0, 1e-30, 1e-38, 1e-39, 1e-40):
        y = rng.normal(0, scale, 4000)
        ya = np.abs(y)                       # the smallest sum_k |a_k w_k| a product can have
        yb = oracle.bf16_bits_to_f32(_bf16_round(y.astype(np.float32))).astype(np.float64)
        finite = np.isfinite(yb)
        assert (np.abs(yb - y)[finite] <= oracle.tolerance(y, ya)[finite]).all(), scale
    # the subnormal term is negligible against normal outputs
    assert oracle.BF16_SUBNORMAL_HALF_SPACING == 2.0 ** -134
    assert oracle.tolerance(np.array([1e-30]), np.array([1e-30]))[0] == pytest.approx(8.1e-33)




# --------------------------------------------------------------------------
# GPTQ (GPTQ explainer, azimuth.plus/paper/gptq)
# --------------------------------------------------------------------------

def _gptq_inputs(N, K, n, seed):
    w = _random_bf16((N, K), 0.02, seed)
    x = _random_bf16((n, K), 1.0, seed + 1, outliers=False)
    return w, x


def pin_gptq_identity_hessian_is_rtn():
    """H = 2 X X^T proportional to the identity (one calibration sample per
    input feature, x_t = e_t): the inverse Hessian is diagonal, no weight is
    ever adjusted, and GPTQ reduces to the round-to-nearest quantizer."""
    N, K = 8, 256
    w = _random_bf16((N, K), 0.02, 311)
    x = np.zeros((K, K), np.uint16)
    x[np.arange(K), np.arange(K)] = 0x3F80                    # bf16 1.0
    for bits, symmetric in FORMATS:
        for g in (32, 128, K):
            got = oracle.gptq_quantize(w, x, bits, symmetric, g)
            ref = oracle.quantize_pack(w, bits, symmetric, g)
            for a, b in zip(got, ref):
                if b is None:
                    assert a is None
                else:
                    assert np.array_equal(a, b), (bits, symmetric, g)


def _obq_fixed_order(w_bits, x_bits, bits, symmetric, g, damp=oracle.GPTQ_DAMP):
    """OBQ as the page first describes it, with GPTQ's fixed column order:
    quantize column q of every row, move every later weight by
    -err / [Hinv]_qq * Hinv[q, k], then eliminate q from the inverse Hessian
    (Gaussian elimination).  No Cholesky, no batching.  The round-to-nearest
    quantizer of a value is restated here from the guide's formulas (scale
    and zero-point of the group, taken when its first column is reached)."""
    W = oracle.bf16_bits_to_f32(w_bits).astype(np.float64)
    X = oracle.bf16_bits_to_f32(x_bits).astype(np.float64).T       # K x n
    N, K = W.shape
    H = 2.0 * X @ X.T
    H += np.eye(K) * damp * np.mean(np.diag(H))
    Hinv = np.linalg.inv(H)
    qmin, qmax = oracle.code_range(bits, symmetric)
    codes = np.zeros((N, K), np.int64)
    S = np.zeros((N, K // g))
    Z = np.zeros((N, K // g), np.int64)
    for q in range(K):
        if q % g == 0:
            grp = W[:, q:q + g].astype(np.float32)
            _, sc, zz = oracle.quantize_pack(grp, bits, symmetric, g)     # group scale / zero
            S[:, q // g] = oracle.bf16_bits_to_f32(sc[:, 0])
            Z[:, q // g] = 0 if zz is None else _zeros_int(zz, bits, symmetric, zz.shape)[:, 0]
        s32 = S[:, q // g].astype(np.float32)
        u = (W[:, q].astype(np.float32) / s32 + Z[:, q // g].astype(np.float32)).astype(np.float32)
        c = np.clip(np.rint(u), qmin, qmax).astype(np.int64)
        codes[:, q] = c
        w_hat = S[:, q // g] * (c - Z[:, q // g])
        err = (W[:, q] - w_hat) / Hinv[q, q]
        W[:, q + 1:] -= np.outer(err, Hinv[q, q + 1:])
        W[:, q] = w_hat
        Hinv = Hinv - np.outer(Hinv[:, q], Hinv[q, :]) / Hinv[q, q]
    return codes, W


def pin_gptq_matches_sequential_obq():
    """The Cholesky form with lazy batches equals OBQ's sequential form with
    the fixed column order (the page's three innovations change the cost,
    not the result): same codes, same compensated weights."""
    for (bits, symmetric, N, K, g, block) in ((4, False, 6, 48, 16, 8), (4, False, 5, 40, 8, 128),
                                             (8, True, 4, 32, 32, 8), (4, True, 3, 64, 32, 16)):
        w, x = _gptq_inputs(N, K, 24, 400 + K)
        H, U = oracle.gptq_hessian_factor(x)
        codes, scales, zeros, w_out = oracle.gptq_quantize_with_factor(w, U, bits, symmetric, g,
                                                                       block)
        q = _as_int_codes(codes, N, K, bits, symmetric)
        ref_q, ref_w = _obq_fixed_order(w, x, bits, symmetric, g)
        assert np.array_equal(q, ref_q), (bits, symmetric, K, g, block)
        assert np.allclose(w_out, ref_w, rtol=0, atol=1e-9), float(np.abs(w_out - ref_w).max())


def pin_gptq_lazy_batch_is_a_reordering():
    """Blocks of 8 columns and one block of all columns give the same codes:
    the lazy update only postpones additions."""
    w, x = _gptq_inputs(16, 256, 64, 520)
    for bits, symmetric, g in ((4, False, 128), (4, False, 32), (8, True, 256)):
        a = oracle.gptq_quantize(w, x, bits, symmetric, g, block=8)
        b = oracle.gptq_quantize(w, x, bits, symmetric, g, block=256)
        for u, v in zip(a, b):
            assert (u is None and v is None) or np.array_equal(u, v), (bits, symmetric, g)


def pin_gptq_lowers_the_layer_error():
    """GPTQ's purpose: the layer output (W - W_hat) X^T is much smaller than
    with round-to-nearest on the same calibration data."""
    N, K = 64, 256
    w, x = _gptq_inputs(N, K, 128, 600)
    W = oracle.bf16_bits_to_f32(w).astype(np.float64)
    X = oracle.bf16_bits_to_f32(x).astype(np.float64)
    for bits, symmetric, g in ((4, False, 128), (4, True, 64)):
        errs = []
        for codes, scales, zeros in (oracle.gptq_quantize(w, x, bits, symmetric, g),
                                     oracle.quantize_pack(w, bits, symmetric, g)):
            w_hat = oracle.bf16_bits_to_f32(
                oracle.dequantize(codes, scales, zeros, N, K, bits, symmetric, g))
            errs.append(float((((W - w_hat) @ X.T) ** 2).sum()))
        assert errs[0] < 0.5 * errs[1], errs




# --------------------------------------------------------------------------
# FP4 with block scales (guide, section "FP4 with block scales")
# --------------------------------------------------------------------------

E2M1_PAGE_VALUES = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def pin_e2m1_values_and_layout():
    """Every code decodes to the page's list of values, and to the value the
    stated layout (1 sign, 2 exponent, 1 mantissa bit; exponent bias 1,
    subnormal when the exponent field is 0) gives."""
    for code in range(16):
        s, e, m = code >> 3, (code >> 1) & 3, code & 1
        layout = (m * 0.5) if e == 0 else 2.0 ** (e - 1) * (1 + m / 2)
        layout = -layout if s else layout
        v = oracle.e2m1_to_f64(code)
        assert v == layout, (code, v, layout)
        assert abs(v) == E2M1_PAGE_VALUES[code & 7]


def pin_e4m3_matches_torch():
    """E4M3 (guide, FP8 section: 4 exponent bits, 3 mantissa bits) decodes
    like torch's float8_e4m3fn for every finite byte."""
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for b in range(256):
        if np.isnan(ref[b]):
            continue
        assert oracle.e4m3_to_f64(b) == ref[b], b


def _fp4_blocks(w, codes, scales, ts, kind):
    N, K = w.shape
    bs = oracle.FP4_BLOCK[kind]
    x = oracle.bf16_bits_to_f32(w).astype(np.float64) if w.dtype == np.uint16 else w.astype(np.float64)
    q = np.zeros((N, K), np.float64)
    lo, hi = codes & 0xF, codes >> 4
    cod = np.empty((N, K), np.uint8)
    cod[:, 0::2], cod[:, 1::2] = lo, hi
    table = np.array([oracle.e2m1_to_f64(c) for c in range(16)])
    q = table[cod]
    if kind == oracle.FP4_MX:
        scale = np.ldexp(1.0, scales.astype(np.int64) - 127)
    else:
        e4 = torch.from_numpy(scales.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
        scale = (e4.astype(np.float32) * np.float32(ts)).astype(np.float64)   # fp32 product
    return x.reshape(N, K // bs, bs), q.reshape(N, K // bs, bs), scale, cod.reshape(N, K // bs, bs)


def pin_fp4_scales():
    """MXFP4: the scale is a power of two (E8M0, read by torch), the smallest
    that keeps the block's max |x| within 6.  NVFP4: s_t = amax / (6 x 448)
    and the block scale the smallest E4M3 value >= amax_b / (6 s_t)."""
    w = _random_bf16((24, 256), 0.02, 700)
    codes, scales, ts = oracle.fp4_quantize(w, oracle.FP4_MX)
    x, _, _, _ = _fp4_blocks(w, codes, scales, ts, oracle.FP4_MX)
    e8 = torch.from_numpy(scales.copy()).view(torch.float8_e8m0fnu).to(torch.float64).numpy()
    amax = np.abs(x).max(axis=-1)
    assert (amax <= 6 * e8).all() and (amax > 3 * e8).all()
    codes, scales, ts = oracle.fp4_quantize(w, oracle.FP4_NV)
    x, _, _, _ = _fp4_blocks(w, codes, scales, ts, oracle.FP4_NV)
    amax_t = np.float32(np.abs(x).max())
    assert ts == float(amax_t / np.float32(2688.0))
    e4 = torch.from_numpy(scales.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    grid = np.sort(np.unique(torch.arange(0, 127, dtype=torch.uint8).view(torch.float8_e4m3fn)
                             .to(torch.float64).numpy()))
    t = (np.abs(x).max(axis=-1).astype(np.float32) / np.float32(6.0 * np.float32(ts))).astype(np.float64)
    idx = np.searchsorted(grid, t, side="left")           # first grid value >= t
    assert np.array_equal(e4, grid[np.minimum(idx, len(grid) - 1)])


def pin_fp4_codes_nearest_and_roundtrip():
    """Every code is the nearest E2M1 value to x / scale (exact arithmetic,
    ties to the even mantissa bit), so |x - q scale| is at most half the gap
    between neighbouring E2M1 values times the scale."""
    w = _random_bf16((16, 512), 0.02, 710)
    vals = np.array(E2M1_PAGE_VALUES)
    for kind in (oracle.FP4_MX, oracle.FP4_NV):
        codes, scales, ts = oracle.fp4_quantize(w, kind)
        x, q, scale, cod = _fp4_blocks(w, codes, scales, ts, kind)
        u = x / scale[..., None]
        for i in np.ndindex(u.shape):
            a = abs(u[i])
            d = np.abs(vals - a)
            order = np.argsort(d, kind="stable")
            if d[order[1]] - d[order[0]] > 1e-6:
                assert abs(q[i]) == vals[order[0]], (kind, i, u[i], q[i])
            if a != 0 and q[i] != 0:
                assert np.sign(q[i]) == np.sign(u[i])
        gap = np.where(np.abs(q) < 2, 0.5, np.where(np.abs(q) < 4, 1.0, 2.0))
        assert (np.abs(u - q) <= gap / 2 + 1e-9).all()


def pin_fp4_ties_to_even():
    """x / scale exactly half-way: 0.25 -> 0, 0.75 -> 1, 1.25 -> 1, 1.75 -> 2,
    2.5 -> 2, 3.5 -> 4, 5 -> 4 (MXFP4 block with max 6 so the scale is 1)."""
    row = np.zeros((1, 32), np.float32)
    row[0, :8] = [6.0, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]
    codes, scales, _ = oracle.fp4_quantize(row, oracle.FP4_MX)
    assert scales[0, 0] == 127                                  # 2^0
    got = [oracle.e2m1_to_f64((codes[0, k // 2] >> (4 * (k % 2))) & 0xF) for k in range(8)]
    assert got == [6.0, 0.0, 1.0, 1.0, 2.0, 2.0, 4.0, 4.0], got


def pin_fp4_sizes():
    """Half a byte per weight plus one scale byte per block: 4.25 bits per
    weight for MXFP4, 4.5 for NVFP4 (plus one fp32 per tensor)."""
    N, K = 8, 256
    w = _random_bf16((N, K), 0.02, 720)
    for kind, bits in ((oracle.FP4_MX, 4.25), (oracle.FP4_NV, 4.5)):
        codes, scales, _ = oracle.fp4_quantize(w, kind)
        assert (codes.size + scales.size) * 8 / (N * K) == bits


def pin_fp4_dequant_closed_form():
    """The bf16 output is torch's bf16 rounding of the fp32 value of the
    definition; the exact values are code x scale(s)."""
    w = _random_bf16((8, 256), 0.02, 730)
    for kind in (oracle.FP4_MX, oracle.FP4_NV):
        codes, scales, ts = oracle.fp4_quantize(w, kind)
        w_hat, w_exact = oracle.fp4_dequantize(codes, scales, ts, 8, 256, kind)
        x, q, scale, _ = _fp4_blocks(w, codes, scales, ts, kind)
        if kind == oracle.FP4_MX:
            v32 = (q * scale[..., None]).astype(np.float32)
            exact = q * scale[..., None]
        else:
            e4 = torch.from_numpy(scales.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
            p = (q * e4[..., None]).astype(np.float32)                      # exact
            v32 = (p * np.float32(ts)).astype(np.float32)
            exact = q * e4[..., None] * np.float64(np.float32(ts))
        ref = torch.from_numpy(v32.reshape(8, 256)).to(torch.bfloat16).view(torch.int16).numpy()
        assert np.array_equal(w_hat, ref.view(np.uint16))
        assert np.array_equal(w_exact, exact.reshape(8, 256))


def _exact_int_products(M, N, K, seed):
    """Integer matrices times powers of two: every product and partial sum is
    exact in fp64, so the reference must equal integer arithmetic."""
    rng = np.random.default_rng(seed)
    ai = rng.integers(-7, 8, (M, K))
    wi = rng.integers(-6, 7, (N, K))
    exact = ai.astype(object).dot(wi.T.astype(object))              # Python integers
    exact_abs = np.abs(ai).astype(object).dot(np.abs(wi).T.astype(object))
    return ai, wi, np.array(exact, dtype=np.float64), np.array(exact_abs, dtype=np.float64)


def pin_matmul_f64_exact_integers():
    """bf16 activations x fp64 weights: small integers scaled by 2^-3 and 2^-5
    (exact in bf16 and fp64) give integer arithmetic scaled by 2^-8; the
    shape is not square, so a transposed operand cannot pass."""
    M, N, K = 3, 5, 40
    ai, wi, exact, exact_abs = _exact_int_products(M, N, K, 810)
    a_bits = (torch.from_numpy(ai * 0.125).to(torch.bfloat16).view(torch.int16).numpy()
              .view(np.uint16))
    y, ya = oracle.matmul_f64_exact(a_bits, wi * 0.03125)
    assert np.array_equal(y, exact / 256.0)
    assert np.array_equal(ya, exact_abs / 256.0)


def pin_matmul_f64_ab_integers():
    """fp64 x fp64: the same integer check, with fractional power-of-two
    scales on both operands, and a one-hot row that returns a weight column."""
    M, N, K = 4, 6, 72
    ai, wi, exact, exact_abs = _exact_int_products(M, N, K, 811)
    y, ya = oracle.matmul_f64_ab(ai * 0.5, wi * 0.0625)
    assert np.array_equal(y, exact / 32.0)
    assert np.array_equal(ya, exact_abs / 32.0)
    onehot = np.zeros((1, K))
    onehot[0, 9] = 1.0
    y1, _ = oracle.matmul_f64_ab(onehot, wi * 0.0625)
    assert np.array_equal(y1[0], wi[:, 9] * 0.0625)


# every pin_* function of this module (defined last, after all of them)
ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
