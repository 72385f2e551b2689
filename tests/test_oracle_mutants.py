"""Planted mistakes in copies of the oracle must each trip at least one pin.

The lower clamp has no mutant: for all four formats x/S + Z >= q_min - 1/2
holds exactly in fp32 (the minimum defines Z through the same rounded
quotient) and round-half-even of q_min - 1/2 is q_min, so removing it changes
no result.

Every mutant below is a plausible slip in the oracle (a dropped term, a wrong
sign, rounding or index, a transposed operand), in the round-to-nearest
quantizer, the dequantization, the reference matmul and the GPTQ column loop.  The copy is compiled on the
CPU into a temporary directory; the real oracle is never modified.
"""
import os

import pytest

import oracle
import oracle_pins
from oracle import build as obuild

SRC = obuild.SRC

MUTANTS = {
    "nibble_order_swapped": (
        "if ((k & 1) == 0) *byte = (uint8_t)((*byte & 0xF0) | nib);\n        else              *byte = (uint8_t)((*byte & 0x0F) | (nib << 4));",
        "if ((k & 1) == 1) *byte = (uint8_t)((*byte & 0xF0) | nib);\n        else              *byte = (uint8_t)((*byte & 0x0F) | (nib << 4));"),
    "round_half_away": ("float r = rintf(u);", "float r = roundf(u);"),
    "no_clamp_high": ("if (c > qmax) c = qmax;", ""),
    "zero_point_sign": ("Z = qmin - (int32_t)rintf(vmin / Sf);",
                        "Z = qmin + (int32_t)rintf(vmin / Sf);"),
    "scale_rounded_to_nearest": ("uint16_t Sb = qzo_f32_to_bf16_up(S);",
                                 "uint16_t Sb = qzo_f32_to_bf16_rne(S);"),
    "range_without_zero": ("float vmin = 0.0f, vmax = 0.0f;",
                           "float vmin = x[0], vmax = x[0];"),
    "zero_point_from_unrounded_scale": ("Z = qmin - (int32_t)rintf(vmin / Sf);",
                                        "Z = qmin - (int32_t)rintf(vmin / S);"),
    "shift_before_divide": ("float u = x / Sf + (float)Z;",
                            "float u = (x + (float)Z) / Sf;"),
    "code_span_off_by_one": ("S = (vmax - vmin) / (float)(qmax - qmin);",
                             "S = (vmax - vmin) / (float)(qmax - qmin + 1);"),
    "symmetric_qmax_128": ("*qmax = (1 << (bits - 1)) - 1;", "*qmax = (1 << (bits - 1));"),
    "dequant_truncates": ("w_hat[n * K + k] = qzo_f32_to_bf16_rne(prod);",
                          "w_hat[n * K + k] = (uint16_t)(bits_of_f32(prod) >> 16);"),
    "dequant_drops_zero_point": ("float prod = Sf * (float)(q - Z);",
                                 "float prod = Sf * (float)q;"),
    "rne_ties_up": ("if (dropped > 0x8000u || (dropped == 0x8000u && kept_is_odd))",
                    "if (dropped >= 0x8000u)"),
    "matmul_transposed_operand": ("(double)qzo_bf16_to_f32(w_hat[n * K + k]);",
                                  "(double)qzo_bf16_to_f32(w_hat[k * N + n % K]);"),
    "matmul_abs_sum_signed": ("sa += fabs(p);", "sa += p;"),
    # GPTQ
    "gptq_error_not_scaled": ("double e = (W[j] - w_hat) / U[j * K + j];",
                              "double e = (W[j] - w_hat);"),
    "gptq_lazy_update_dropped": ("                W[k] -= v;\n", "\n"),
    "gptq_factor_transposed": ("for (int64_t k = j + 1; k < end; ++k) W[k] -= e * U[j * K + k];",
                               "for (int64_t k = j + 1; k < end; ++k) W[k] -= e * U[k * K + j];"),
    "gptq_group_scale_from_original_weights": ("for (int64_t k = 0; k < g; ++k) grp[k] = (float)W[j + k];",
                                               "for (int64_t k = 0; k < g; ++k) grp[k] = w[n * K + j + k];"),
    # FP4 with block scales
    "fp4_ties_away_from_zero": ("if (di < db || (di == db && (i % 2) == 0 && (best % 2) == 1)) best = i;",
                                "if (di <= db) best = i;"),
    "fp4_mx_scale_one_too_small": ("while ((double)amax > 6.0 * ldexp(1.0, e)) ++e;   /* smallest e */",
                                   "while ((double)amax > 12.0 * ldexp(1.0, e)) ++e;"),
    "fp4_nv_scale_rounded_down": ("if (qzo_e4m3_to_f64((uint8_t)b) >= (double)t) return (uint8_t)b;",
                                  "if (qzo_e4m3_to_f64((uint8_t)b) > (double)t) return (uint8_t)(b - 1);"),
    "fp4_nv_tensor_scale_without_fp8_range": ("s_t = amax > 0.0f ? amax / 2688.0f : 1.0f;",
                                              "s_t = amax > 0.0f ? amax / 6.0f : 1.0f;"),
    "fp4_e4m3_bias_off_by_one": ("ldexp(1.0 + m / 8.0, e - 7)", "ldexp(1.0 + m / 8.0, e - 8)"),
    "matmul_exact_transposed_weights": ("* w[n * K + k];\n                acc += p;",
                                        "* w[k * N + n % K];\n                acc += p;"),
    "matmul_ab_abs_sum_signed": ("sum_abs += fabs(t);", "sum_abs += t;"),
    "matmul_ab_transposed_activations": ("double t = a[m * K + k] * w[n * K + k];",
                                         "double t = a[k * M + m % K] * w[n * K + k];"),
    "gptq_no_damping": ("double lambda = mean > 0.0 ? damp * mean : 1.0;",
                        "double lambda = mean > 0.0 ? 0.0 : 1.0;"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path, monkeypatch):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not found exactly once"
    msrc = tmp_path / "mutant.c"
    msrc.write_text(src.replace(old, new))
    so = obuild.build(force=True, src=str(msrc), out=str(tmp_path / "libmutant.so"))
    monkeypatch.setattr(oracle, "_lib", oracle.load(so))
    caught = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin()
        except Exception as e:  # AssertionError, or a crash of the broken copy
            caught.append((pin.__name__, type(e).__name__))
            break
    assert caught, f"no pin detects the planted mistake '{name}'"


def test_mutation_sites_exist_in_real_oracle():
    src = open(SRC).read()
    for name, (old, _) in MUTANTS.items():
        assert src.count(old) == 1, name
    assert os.path.exists(obuild.build())
