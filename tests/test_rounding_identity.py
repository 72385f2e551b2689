"""The division-free rounding of the quantize kernels, checked on the CPU.

Quantization concepts guide (HF Transformers), section "Mapping values to
fewer bits": q = round(x / S + Z), clamped to the code range, with the
half-to-even rounding this library fixes.  The kernels never divide: with
r = 1/S rounded to nearest they compute

    m = fl( fl(x * r + (Z + C)) + (1.5 * 2^23 - C) ),   C = 192 (int4), 768 (int8)

(the inner step one fused multiply-add) and read the code from m's low
mantissa bits, clamping the asymmetric formats at q_max.  This file emulates
those two fp32 roundings in numpy -- float64 holds x * r + (Z + C) exactly,
and the cast to float32 rounds it once, to nearest even, as the FMA does --
and compares against the rational definition for EVERY finite bf16 x whose
x / S + Z lies in the reachable range, over all 128 bf16 scale significands
at several exponents (fp32-subnormal scales included) and a spread of zero
points.  It is a proof check of the identity the kernels rely on, not a test
of the CUDA code itself (the GPU parity tests do that).
"""
import numpy as np
import pytest

FORMATS = [(4, False), (4, True), (8, False), (8, True)]
EXPONENTS = [-134, -130, -20, -7, 0, 100]


def _all_bf16():
    b = np.arange(0x0001, 0x7F80, dtype=np.uint32) << 16      # positive finite bf16
    x = b.view(np.float32)
    return np.concatenate([x, -x, np.zeros(1, np.float32)])


def _code_range(bits, sym):
    if sym:
        q = (1 << (bits - 1)) - 1
        return -q, q
    return (0, 15) if bits == 4 else (-128, 127)


@pytest.mark.parametrize("bits,sym", FORMATS)
def test_division_free_rounding_matches_definition(bits, sym):
    qmin, qmax = _code_range(bits, sym)
    C = np.float32(192.0 if bits == 4 else 768.0)
    k_round = np.float32(12582912.0) - C
    xs_all = _all_bf16()
    zs = [0] if sym else sorted({qmin, qmin + 1, (qmin + qmax) // 2, qmax - 1, qmax})
    checked = 0
    for e in EXPONENTS:
        for ms in range(128, 256):
            S = np.float32(ms * 2.0 ** e)
            with np.errstate(all="ignore"):
                r = np.float32(1.0) / S                      # correctly rounded
            assert np.isfinite(r)
            x = xs_all[np.abs(xs_all.astype(np.float64)) <= (qmax - qmin + 0.5) * float(S)]
            q_exact = x.astype(np.float64) / float(S)        # exact ties stay exact
            for z in zs:
                t = q_exact + z
                if sym:    # S >= absmax / q_max, so |x / S| <= q_max
                    ok = np.abs(t) <= qmax
                else:      # the range contains 0 and (max - min) / S <= q_max - q_min
                    ok = (t >= qmin - 0.5) & (t <= qmax + 0.5)
                xx, tt = x[ok], t[ok]
                ref = np.clip(np.rint(tt), qmin, qmax).astype(np.int64)
                zc = np.float32(z) + C
                y = (xx.astype(np.float64) * float(r) + float(zc)).astype(np.float32)
                m = (y + k_round).astype(np.float32)
                b = m.view(np.uint32).astype(np.int64)
                if not sym:
                    b = np.minimum(b, 0x4B400000 + qmax)
                q = b - 0x4B400000
                bad = np.nonzero(q != ref)[0]
                assert len(bad) == 0, (e, ms, z, float(xx[bad[0]]), q[bad[0]], ref[bad[0]])
                checked += len(ref)
    assert checked > 10 ** 6
