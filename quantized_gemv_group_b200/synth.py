"""Seeded synthetic inputs shared by the tests, the bench and the oracle runs.

This module only draws random numbers; it holds none of the quantization or
product arithmetic.  The distributions restate the workloads of the pages:

* weights: fp32 draws from N(0, 0.02^2); about 0.1 % of the input (K)
  columns are multiplied by 20 as outliers ("Métodos de cuantización de LLM
  para ejecutar un modelo de 70B en una sola GPU", introduction: roughly
  0.1 % of hidden dimensions carry values up to 20x larger); cast to fp16
  with round-to-nearest;
* activations: N(0, 1) in fp16 or bf16;
* sign matrices: uniform random 32-bit words, i.e. exact Bernoulli(0.5) bits;
* channel scales s1, s2: fp16(|N(0, 0.02^2)| + 1e-3).

Every generator takes an explicit seed and device; tensors made on a CUDA
device use torch's Philox generator and are reproducible for a given torch
version.
"""
import torch


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=torch.device(device))
    g.manual_seed(int(seed))
    return g


def outlier_count(k: int, frac: float = 0.001) -> int:
    """Number of outlier K-columns: max(1, round(frac * k))."""
    return max(1, int(round(frac * k)))


def weight(n: int, k: int, seed: int, device="cpu", std: float = 0.02,
           outlier_frac: float = 0.001, outlier_mult: float = 20.0,
           dtype=torch.float16) -> torch.Tensor:
    """[n, k] row-major (out x in) weight with planted outlier columns."""
    g = _gen(seed, device)
    w = torch.randn(n, k, generator=g, device=device, dtype=torch.float32) * std
    if outlier_frac > 0:
        cols = torch.randperm(k, generator=g, device=device)[: outlier_count(k, outlier_frac)]
        w[:, cols] *= outlier_mult
    return w.to(dtype)


def activations(M: int, k: int, seed: int, device="cpu", dtype=torch.float16) -> torch.Tensor:
    g = _gen(seed, device)
    return torch.randn(M, k, generator=g, device=device, dtype=torch.float32).to(dtype)


def sign_words(rows: int, cols: int, seed: int, device="cpu") -> torch.Tensor:
    """[rows, cols/32] int32 tensor of uniform random bits (canonical sign words)."""
    assert cols % 32 == 0
    g = _gen(seed, device)
    return torch.randint(-(2 ** 31), 2 ** 31, (rows, cols // 32), generator=g,
                         device=device, dtype=torch.int64).to(torch.int32)


def channel_scales(d: int, seed: int, device="cpu", std: float = 0.02) -> torch.Tensor:
    g = _gen(seed, device)
    return (torch.randn(d, generator=g, device=device, dtype=torch.float32).abs() * std
            + 1e-3).to(torch.float16)


def pm1(rows: int, cols: int, seed: int, device="cpu") -> torch.Tensor:
    """[rows, cols] int8 tensor of +-1 values."""
    g = _gen(seed, device)
    return (torch.randint(0, 2, (rows, cols), generator=g, device=device, dtype=torch.int8) * 2 - 1)


def tensor_seed(layer: int, proj: int) -> int:
    """Seed of the tensor (layer, projection) in the layered workloads."""
    return 1000 * layer + proj


def bits_u16(t: torch.Tensor):
    """uint16 numpy view of a half-precision tensor's bit patterns (on host)."""
    import numpy as np
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def words_u32(t: torch.Tensor):
    import numpy as np
    return t.detach().contiguous().cpu().numpy().view(np.uint32)
