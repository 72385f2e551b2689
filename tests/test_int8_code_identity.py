"""The int8 code-to-bf16 step of the decode GEMV and the tcgen05 GEMM, checked
on the CPU.

Quantization concepts guide (HF Transformers), section "Mapping values to
fewer bits": x_hat = S (q - Z), here int8 symmetric (Z = 0), rounded once to
bf16.  The kernels place each code byte b, XORed with 0x80 (u = q + 128),
in the low mantissa bits of the fp32 2^23, subtract 2^23 + 128 (two values
per sub.rn.f32x2), pack the pair to bf16 and multiply by (S, S) in bf16 with
one rounding.  This pins that the subtraction and the pack are exact for all
256 codes, so the one bf16 rounding of S*q is the definition's.

It also records why the kernels do not form S*q with one fma from a byte
placed higher in 2^23 (m = 2^23 + 256 u, s = S/256, c = -(2^23 + 2^15) s):
that intermediate is about 2^15 S and overflows fp32 for scales above 2^113,
which finite bf16 weights can produce (S = absmax / 127).
"""
import numpy as np


def test_subtraction_and_pack_are_exact_for_every_code():
    b = np.arange(256, dtype=np.uint32)
    u = b ^ 0x80
    m = (np.uint32(0x4B000000) | u).astype(np.uint32).view(np.float32)
    q = (m - np.float32(8388736.0)).astype(np.float32)          # 2^23 + 128, fp32 subtraction
    want = b.astype(np.uint8).view(np.int8).astype(np.float32)
    assert np.array_equal(q, want)
    # the bf16 pack keeps every q (|q| <= 128 fits in 8 significant bits)
    bf = (q.view(np.uint32) >> 16 << 16).view(np.float32)        # truncation to bf16
    assert np.array_equal(bf, q)


def test_the_one_fma_form_would_overflow_for_large_scales():
    # the largest int8 scale finite bf16 weights give: S = max bf16 / 127
    max_bf16 = np.float32(np.uint32(0x7F7F0000).view(np.float32))
    S = max_bf16 / np.float32(127.0)
    assert np.isfinite(S) and S > np.float32(2.0 ** 113)
    s = S * np.float32(1.0 / 256.0)
    with np.errstate(over="ignore"):
        c = s * np.float32(-8421376.0)                           # -(2^23 + 2^15) s
    assert not np.isfinite(c)
    # while S * q itself stays finite for every code the symmetric format
    # writes (|q| <= 127: S * 127 is the weights' absmax)
    assert np.float64(S) * 127.0 < np.finfo(np.float32).max
