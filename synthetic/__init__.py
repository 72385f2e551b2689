"""Seeded synthetic inputs shared by the CUDA path's tests/benchmark and the CPU oracle.

This module holds no quantization arithmetic: it only draws random numbers and
rounds them to the input dtype (bf16, round-to-nearest-even, done by torch).

Recipe (stand-in for Llama-shaped linear layers; the pages use trained
OPT/BLOOM/Llama weights, which are not available here):
  weights      w ~ N(0, sigma) in fp32, then a Bernoulli(1e-3) outlier mask
               from the same generator multiplies those entries by 20, then
               bf16 RNE;
  activations  a ~ N(0, 1) in fp32, then bf16 RNE.
A ``torch.Generator`` seeded with ``seed`` on the target device drives both
draws, so the same (shape, sigma, seed, device) always yields the same tensor.
CPU and CUDA generators produce different streams; a parity test draws once
and hands the same tensor to both sides.
"""
import torch

OUTLIER_FRACTION = 1e-3
OUTLIER_FACTOR = 20.0


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def weights(N: int, K: int, sigma: float = 0.02, seed: int = 0, device="cpu",
            outlier_fraction: float = OUTLIER_FRACTION,
            outlier_factor: float = OUTLIER_FACTOR) -> torch.Tensor:
    """N x K bf16 weights: N(0, sigma) with a fraction of entries x outlier_factor."""
    g = _gen(seed, device)
    w = torch.randn((N, K), generator=g, device=device, dtype=torch.float32)
    w.mul_(sigma)
    if outlier_fraction > 0:
        mask = torch.rand((N, K), generator=g, device=device) < outlier_fraction
        w[mask] *= outlier_factor
    return w.to(torch.bfloat16)


def activations(M: int, K: int, seed: int = 0, device="cpu") -> torch.Tensor:
    """M x K bf16 activations ~ N(0, 1)."""
    g = _gen(seed, device)
    return torch.randn((M, K), generator=g, device=device,
                       dtype=torch.float32).to(torch.bfloat16)


def bf16_bits(t: torch.Tensor):
    """The uint16 bit patterns of a bf16 tensor as a CPU numpy array."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view("uint16")


def from_bf16_bits(bits, device="cpu") -> torch.Tensor:
    """Inverse of :func:`bf16_bits`."""
    import numpy as np
    arr = np.ascontiguousarray(bits, dtype=np.uint16)
    return torch.from_numpy(arr.view(np.int16)).view(torch.bfloat16).to(device)


# Layer shapes (N = output features, K = input features) of the workloads.
TINY = dict(N=1024, K=1024, M=1, sigma=0.02, seed=0)
DECODE_7B = [(4096, 4096), (11008, 4096), (4096, 11008)]
DECODE_70B = [(28672, 8192), (8192, 28672)]
DECODE_70B_M = [1, 4, 8, 16]
PREFILL = dict(M=2048, N=8192, K=8192, sigma=0.02, seed=6)
BULK_LAYER_SET = [(4096, 4096)] * 4 + [(14336, 4096)] * 2 + [(4096, 14336)]
BULK_SETS = 32
