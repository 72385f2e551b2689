"""CUDA path vs the CPU oracle at full layer sizes, every element (needs a B200).

The elementwise kernels (quantize_pack, dequantize) walk their inputs with
grid-stride loops over grids sized to the device, so a layer of more than
about twenty million values takes second and later passes that the small
parity cases never reach.  These tests compare whole full-size layers bit for
bit:

  * dequantize of the 7B-class (4096, 11008) layer and of the 70B-class
    (28672, 8192) layer, int4 asymmetric group-128 and int8 symmetric
    per-channel, from codes the oracle packed (the expected values and the
    kernel's inputs both come from the oracle);
  * per-tensor (group_size 0) quantize_pack and dequantize of a 4096 x 5120
    matrix (21 M values), all four formats;
  * the bulk-quantization stack: 32 layer sets, 7.785e9 parameters, through
    quantize_pack at int4 asymmetric group-128 and int8 symmetric
    per-channel, every code, scale and zero of every layer.

Definitions: HF Transformers "Quantization concepts" guide, section "Mapping
values to fewer bits" (S, Z, q and the dequantization x = S (q - Z)),
section "Choose granularity" (per-tensor, per-channel, per-group).
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
    oracle.set_threads(oracle.max_threads())
    return torch.device("cuda:0")


def u16(t):
    return synthetic.bf16_bits(t)


def u8(t):
    return t.detach().cpu().numpy().view(np.uint8)


def to_dev_u8(a, dev):
    return torch.from_numpy(np.ascontiguousarray(a)).to(dev)


def first_difference(got, ref):
    bad = np.flatnonzero(got.reshape(-1) != ref.reshape(-1))
    return f"{bad.size} elements differ, first flat indices {bad[:5].tolist()}"


def check_dequantize_full(dev, N, K, bits, sym, g, seed):
    w = synthetic.weights(N, K, sigma=0.015, seed=seed, device=dev)
    wb = u16(w)
    del w
    c, s, z = oracle.quantize_pack(wb, bits, sym, g)
    del wb
    ref = oracle.dequantize(c, s, z, N, K, bits, sym, g)
    out = qz.qz_dequantize(to_dev_u8(c, dev), synthetic.from_bf16_bits(s, dev),
                           None if z is None else to_dev_u8(z, dev), N, K, bits, sym, g)
    torch.cuda.synchronize()
    got = u16(out)
    del out
    assert np.array_equal(got, ref), first_difference(got, ref)


@pytest.mark.parametrize("bits,sym,per_channel", [(4, False, False), (8, True, True)])
@pytest.mark.parametrize("N,K,seed", [(4096, 11008, 3), (28672, 8192, 4)])
def test_dequantize_full_layer_bit_exact(dev, N, K, seed, bits, sym, per_channel):
    """Every element of a full decode layer: 45 M and 235 M values (int4
    group-128, int8 per-channel)."""
    check_dequantize_full(dev, N, K, bits, sym, K if per_channel else 128, seed)


@pytest.mark.parametrize("bits,sym", FORMATS)
def test_per_tensor_quantize_and_dequantize_21m_values(dev, bits, sym):
    """group_size 0 (one scale and zero for the whole matrix) on 21 M values:
    the three-launch range / quantize / finish path over many grid passes."""
    N, K = 4096, 5120
    w = synthetic.weights(N, K, sigma=0.02, seed=17 + bits + int(sym), device=dev)
    wb = u16(w)
    ws = qz.Workspace(dev)
    c, s, z = qz.qz_quantize_pack(w, bits, sym, 0, workspace=ws)
    torch.cuda.synchronize()
    rc, rs, rz = oracle.quantize_pack(wb, bits, sym, 0)
    assert np.array_equal(u16(s).reshape(rs.shape), rs), "scale differs"
    if rz is not None:
        assert np.array_equal(u8(z).reshape(rz.shape), rz), "zero differs"
    gc = u8(c).reshape(rc.shape)
    assert np.array_equal(gc, rc), first_difference(gc, rc)
    ref = oracle.dequantize(rc, rs, rz, N, K, bits, sym, 0)
    out = qz.qz_dequantize(to_dev_u8(rc, dev), synthetic.from_bf16_bits(rs, dev),
                           None if rz is None else to_dev_u8(rz, dev), N, K, bits, sym, 0)
    torch.cuda.synchronize()
    got = u16(out)
    assert np.array_equal(got, ref), first_difference(got, ref)


def test_bulk_quantization_stack_every_code(dev):
    """32 layer sets (7.785e9 parameters) through quantize_pack, int4
    asymmetric group-128 and int8 symmetric per-channel: every code, scale
    and zero of every layer equals the oracle's."""
    total = 0
    ws = qz.Workspace(dev)
    for si in range(synthetic.BULK_SETS):
        for li, (N, K) in enumerate(synthetic.BULK_LAYER_SET):
            seed = 100 + si * 16 + li
            w = synthetic.weights(N, K, sigma=0.02, seed=seed, device=dev)
            wb = u16(w)
            for bits, sym, g in ((4, False, 128), (8, True, K)):
                c, s, z = qz.qz_quantize_pack(w, bits, sym, g, workspace=ws)
                torch.cuda.synchronize()
                rc, rs, rz = oracle.quantize_pack(wb, bits, sym, g)
                where = f"set {si} layer {li} ({N}x{K}) bits={bits}"
                assert np.array_equal(u16(s).reshape(rs.shape), rs), f"{where}: scales differ"
                if rz is not None:
                    assert np.array_equal(u8(z).reshape(rz.shape), rz), f"{where}: zeros differ"
                gc = u8(c).reshape(rc.shape)
                assert np.array_equal(gc, rc), f"{where}: " + first_difference(gc, rc)
                del c, s, z
            total += N * K
            del w, wb
    assert total == 7_784_628_224
