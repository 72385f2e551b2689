"""The NVFP4 quantize kernel's scale arithmetic, emulated on the CPU.

Quantization concepts guide, section "FP4 with block scales" (NVFP4: E4M3
block scales under one fp32 tensor scale).  The kernel forms the block scale
as the smallest E4M3 value >= fp32(amax_b / fp32(6 s_t)) without a division
or exponent functions, and this test checks that arithmetic against plain
definitions:

- E4M3 round-up from the fp32 bits: above 2^-6, (bits + 2^20 - 1) >> 20,
  less (127 - 7) << 3, clamped at 0x7E, must be the smallest E4M3 value >= t
  (the E4M3 grid from torch's float8_e4m3fn), at every grid point, both fp32
  neighbours of it, and random values from 2^-14 to 2^10.
- The quotient by Markstein's correction (Markstein 1990): with r = RN(1/d)
  and q0 = RN(x r), RN(q0 + RN-exact(x - q0 d) r) evaluated with two fused
  multiply-adds equals RN(x / d), checked in exact rational arithmetic on
  random and structured operands inside the range the kernel uses it in.
"""
from fractions import Fraction

import numpy as np
import torch


def e4m3_grid():
    b = torch.arange(0, 0x7F, dtype=torch.uint8)
    return b.view(torch.float8_e4m3fn).to(torch.float64).numpy()      # bytes 0..0x7E, increasing


def round_up_kernel(t32):
    """The kernel's E4M3 round-up, step by step in numpy (t > 0)."""
    t32 = np.asarray(t32, dtype=np.float32)
    u = t32.view(np.uint32).astype(np.int64)
    normal = ((u + 0xFFFFF) >> 20) - 960
    normal = np.minimum(normal, 0x7E)
    small = np.minimum(t32, np.float32(2.0 ** -6))                       # only used below 2^-6
    sub = np.ceil((small * np.float32(512.0)).astype(np.float64))        # t * 512 is exact
    return np.where(t32 < np.float32(2.0 ** -6), sub, normal).astype(np.int64)


def test_e4m3_round_up_from_bits():
    grid = e4m3_grid()
    assert (np.diff(grid) > 0).all()
    pts = grid[1:].astype(np.float32)
    ts = np.concatenate([
        pts, np.nextafter(pts, np.float32(np.inf)), np.nextafter(pts, np.float32(0)),
        np.exp2(np.random.default_rng(0).uniform(-14, 10, 20000)).astype(np.float32),
        np.array([448.0, 448.5, 480.0, 512.0, 1e6, 3e38], dtype=np.float32)])
    ts = ts[ts > 0]
    got = round_up_kernel(ts)
    want = np.minimum(np.searchsorted(grid, ts.astype(np.float64), side="left"), 0x7E)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, [(float(ts[i]), int(got[i]), int(want[i])) for i in bad[:5]]


def rn32(v: Fraction) -> Fraction:
    """Round a positive rational to the nearest fp32 (normal range), ties to
    even."""
    assert v > 0
    e = v.numerator.bit_length() - v.denominator.bit_length()
    if Fraction(2) ** e > v:
        e -= 1
    ulp = Fraction(2) ** (e - 23)
    m = v / ulp
    lo = m.numerator // m.denominator
    rem = m - lo
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and lo % 2 == 1):
        lo += 1
    return lo * ulp


def fma32(a: Fraction, b: Fraction, c: Fraction) -> Fraction:
    v = a * b + c
    if v == 0:
        return Fraction(0)
    return rn32(v) if v > 0 else -rn32(-v)


def markstein(x: Fraction, d: Fraction) -> Fraction:
    r = rn32(1 / d)
    q0 = rn32(x * r)
    rho = fma32(-q0, d, x)
    return fma32(rho, r, q0)


def f32(v) -> Fraction:
    return Fraction(float(np.float32(v)))


def test_markstein_quotient_is_correctly_rounded():
    rng = np.random.default_rng(1)
    cases = []
    # amax_b / (6 s_t) as the kernel forms it: bf16 block maxima, s_t from a
    # tensor maximum at least as large
    for _ in range(4000):
        amax_t = float(torch.tensor(np.exp2(rng.uniform(-60, 60)), dtype=torch.bfloat16))
        amax_b = float(torch.tensor(amax_t * rng.uniform(0.0, 1.0), dtype=torch.bfloat16))
        if amax_b < 2.0 ** -100:
            continue
        s_t = np.float32(np.float32(amax_t) / np.float32(2688.0))
        d6 = np.float32(np.float32(6.0) * s_t)
        cases.append((f32(amax_b), f32(d6)))
    # structured: divisors with few significant bits, quotients at and next
    # to E4M3 grid points (where a misrounded quotient would change the scale)
    grid = e4m3_grid()[1:]
    for d in (3.0, 6.0, 7.0, 0.75, 1.5 * 2 ** -20, 5.0 * 2 ** 30):
        for gval in grid[::3]:
            x = np.float32(gval * d)
            for xv in (x, np.nextafter(x, np.float32(np.inf)), np.nextafter(x, np.float32(0))):
                cases.append((f32(xv), f32(d)))
    for x, d in cases:
        q0 = rn32(x * rn32(1 / d))
        assert q0 >= Fraction(2) ** -100          # the kernel's range check
        assert markstein(x, d) == rn32(x / d), (float(x), float(d))
