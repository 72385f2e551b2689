"""The benchmark's accounting, on CPU: the algorithmic work per launch that
every GB/s and TFLOP/s figure divides, the roofline object, and the rule that
drops a DRAM-traffic record once its kernel source has changed.

The byte counts follow from the packed sizes of the quantization guide's
section "int8 and int4" (half a byte per int4 code, one per int8 code) with a
bf16 scale and a uint8 zero per group of 128, plus the bf16 activations and
outputs.  The figures below are those sizes worked out by hand for each
configuration and written to three or four digits; the functions must agree
to that precision.
"""
import hashlib
import json
import os

import pytest

import bench
import synthetic

MB = 1e6


@pytest.mark.parametrize("M,N,K,expect_mb,half_digit", [
    (1, 1024, 1024, 0.553, 5e-4),    # tiny configuration
    (1, 4096, 4096, 8.80, 5e-3),     # 7B-class decode layers
    (1, 11008, 4096, 23.63, 5e-3),
    (1, 4096, 11008, 23.63, 5e-3),
    (1, 28672, 8192, 123.0, 5e-2),   # 70B-class decode layers
    (1, 8192, 28672, 123.0, 5e-2),
])
def test_w4a16_gemv_bytes(M, N, K, expect_mb, half_digit):
    # equal to the stated figure to its printed precision
    assert abs(bench.w4_gemv_bytes(M, N, K) / MB - expect_mb) <= half_digit


def test_w4a16_gemv_bytes_terms():
    # codes N*K/2, scale + zero 3 bytes per group of 128, bf16 a and y
    M, N, K = 16, 256, 512
    assert bench.w4_gemv_bytes(M, N, K) == N * K // 2 + 3 * N * K // 128 + 2 * M * K + 2 * M * N


def test_w8a16_gemv_bytes():
    assert abs(bench.w8_gemv_bytes(1, 28672, 8192) / MB - 235.0) <= 0.05
    assert abs(bench.w8_gemv_bytes(1, 8192, 28672) / MB - 235.0) <= 0.05


def test_prefill_flops():
    assert bench.gemm_flops(2048, 8192, 8192) == pytest.approx(2.749e11, rel=5e-4)


def test_bulk_quantization_bytes():
    params = sum(N * K for N, K in synthetic.BULK_LAYER_SET) * synthetic.BULK_SETS
    assert params == 7_784_628_224
    b4 = sum(bench.quant_int4_bytes(N, K) for N, K in synthetic.BULK_LAYER_SET) * synthetic.BULK_SETS
    b8 = sum(bench.quant_int8_bytes(N, K) for N, K in synthetic.BULK_LAYER_SET) * synthetic.BULK_SETS
    assert b4 / params == pytest.approx(2.5234375)          # 2 + 1/2 + 3/128 bytes per parameter
    assert abs(b4 / 1e9 - 19.65) <= 0.01                    # 19.644 GB
    assert abs(b8 / 1e9 - 23.36) <= 0.005


def test_step_parts_cover_the_hot_path():
    names = [p[0] for p in bench.PARTS]
    assert names == ["quantize_pack_int4_g128", "quantize_pack_int8_per_channel",
                     "dequantize_int4", "w4a16_gemv_m1", "w8a16_gemv_m1",
                     "w4a16_gemv_70b_m1", "w8a16_gemv_70b_m1", "w4a16_gemm_prefill_m2048"]
    work = {p[0]: p[3] for p in bench.PARTS}
    assert work["w4a16_gemv_m1"] == sum(bench.w4_gemv_bytes(1, N, K) for N, K in synthetic.DECODE_7B)
    assert work["w4a16_gemv_70b_m1"] == sum(
        bench.w4_gemv_bytes(1, N, K) for N, K in synthetic.DECODE_70B)
    assert abs(work["w4a16_gemv_70b_m1"] / MB - 246.0) <= 0.1
    assert abs(work["w8a16_gemv_70b_m1"] / MB - 470.0) <= 0.1
    assert work["w4a16_gemm_prefill_m2048"] == sum(
        bench.gemm_flops(2048, N, K) for N, K in synthetic.DECODE_7B)
    launches = {p[0]: p[5] for p in bench.PARTS}
    assert launches["w4a16_gemv_70b_m1"] == 2 and launches["w4a16_gemv_m1"] == 3
    assert bench.LAUNCHES_PER_STEP == 3 * 6 + 2 * 2


PK = {"hbm_gbs": 6500.0, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0,
      "source": "measured"}


def test_roofline_object_hbm():
    r = bench.roofline_obj("w4a16_gemv_m1", 56e6, 0.05, 3, "hbm", PK,
                           {"w4a16_gemv_m1": {"dram_bytes_per_launch_set": 57e6}}, False)
    assert r["achieved"] == pytest.approx(1120.0)                # 56 MB in 50 us
    assert r["peak"] == 6500.0 and r["unit"] == "GB/s"
    assert r["frac"] == pytest.approx(1120.0 / 6500.0, abs=1e-4)
    assert r["traffic"] == 57e6 and r["peak_kind"] == "burst of measured"


def test_roofline_object_tensor_sustained():
    r = bench.roofline_obj("w4a16_gemm_prefill_m2048", 4.4e11, 0.4, 3, "tensor", PK, {}, True)
    assert r["achieved"] == pytest.approx(1100.0)
    assert r["peak"] == 1400.0 and r["unit"] == "TFLOP/s"
    assert r["peak_kind"] == "sustained of measured"
    assert r["traffic"] is None


def test_traffic_record_dropped_when_source_changes(tmp_path, monkeypatch):
    src = tmp_path / "k.cu"
    src.write_text("kernel v1\n")
    digest = hashlib.sha256(src.read_bytes()).hexdigest()[:16]
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps({"kernels": {
        "part": {"sources": ["k.cu"], "sources_sha256_16": digest,
                 "dram_bytes_per_launch_set": 123}}}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.ncu_traffic()["part"]["dram_bytes_per_launch_set"] == 123
    src.write_text("kernel v2\n")
    assert bench.ncu_traffic() == {}
    os.remove(tmp_path / "profiles" / "traffic.json")
    assert bench.ncu_traffic() == {}


def test_fp4_gemv_and_quantize_bytes():
    # half a byte per code plus one scale byte per 32 (MXFP4) or 16 (NVFP4)
    # values, bf16 activations and outputs; NVFP4 adds its fp32 tensor scale
    N, K = 28672, 8192
    assert bench.fp4_gemv_bytes(1, N, K, 0) == N * K // 2 + N * K // 32 + 2 * K + 2 * N
    assert bench.fp4_gemv_bytes(1, N, K, 1) == N * K // 2 + N * K // 16 + 4 + 2 * K + 2 * N
    assert abs(bench.fp4_gemv_bytes(1, N, K, 0) / MB - 124.85) <= 0.005   # 4.25 bits per weight
    assert abs(bench.fp4_gemv_bytes(1, N, K, 1) / MB - 132.19) <= 0.005   # 4.5 bits per weight
    assert bench.fp4_quant_bytes(N, K, 1) == 2 * N * K + N * K // 2 + N * K // 16


def test_gptq_flops_and_fp64_peak():
    """The leading-order count against multiply-adds counted one by one
    (2 flops each): the lower triangle of X^T X over n samples; the Cholesky
    (column j updates the (K-j-1)(K-j)/2 entries of the trailing triangle);
    the triangular inverse (entry (i, j), i > j, of L^-1 sums i - j terms);
    each quantized column j moves every later column of every row once."""
    N, K, n = 4096, 4096, 128
    f = bench.gptq_flops(N, K, n)
    hess = n * K * (K + 1) // 2
    chol = sum((K - j - 1) * (K - j) // 2 for j in range(K))
    trinv = sum(d * (K - d) for d in range(1, K))        # K - d entries at distance d
    updates = N * K * (K - 1) // 2
    exact = 2 * (hess + chol + trinv + updates)
    assert abs(f - exact) / exact < 1e-3
    assert abs(f / 1e9 - 116.68) <= 0.005    # 2.15 + 45.81 + 68.72
    assert abs(bench.FP64_PEAK_TFLOPS - 37.23) <= 0.01
