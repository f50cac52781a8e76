"""Seeded synthetic inputs for the mHC layer.

This module only draws random numbers and sets parameter initialisations; it
holds none of the layer's arithmetic, so both the CUDA path and the fp64
oracle can take their inputs from it.  Every tensor is created on the CPU
from ``torch.Generator().manual_seed(seed)`` so that a test, the benchmark
and the oracle see bit-identical values.

Recipes (std is the second argument of N(., .)):

* tiny forward: T=64, n=4, C=256, x ~ N(0,1) fp32, phi ~ N(0, 0.02)
  [nC, n^2+2n] fp32, alpha = 0.01, bias 4 on the diagonal H_res logits and 0
  elsewhere, F = fixed random linear map W [C, C] with std 1/16
  (variance 1/C), seed 0.
* forward bf16: T=8192, n=4, C=4096, x ~ N(0,1) bf16, f_out ~ N(0,1) bf16.
* forward+backward: T=16384, n=4, C=7168, x, grad_x_next, grad_h_in, f_out
  ~ N(0,1) bf16.
* Sinkhorn: logits ~ N(0, 2) fp32 [B, n, n].
* depth stack: per layer l, phi drawn with seed l and a scalar gain
  s_l ~ U(0.5, 1.5) standing for F_l(h) = s_l * h.
"""
from __future__ import annotations

import torch


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def n_map(n: int) -> int:
    """Number of mapping logits per token: n pre + n post + n*n residual."""
    return n * n + 2 * n


def bias_init(n: int, diag: float = 4.0) -> torch.Tensor:
    """Bias with ``diag`` on the diagonal residual logits, zero elsewhere."""
    b = torch.zeros(n_map(n), dtype=torch.float32)
    for i in range(n):
        b[2 * n + i * n + i] = diag
    return b


def _normal(shape, std: float, g: torch.Generator, dtype: torch.dtype) -> torch.Tensor:
    t = torch.randn(*shape, generator=g, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(dtype) if dtype != torch.float32 else t


def layer_params(n: int, C: int, seed: int, phi_std: float = 0.02, alpha: float = 0.01,
                 diag: float = 4.0) -> dict:
    """phi [nC, n^2+2n] fp32 ~ N(0, phi_std), alpha [1], b [n^2+2n]."""
    g = _gen(seed)
    phi = _normal((n * C, n_map(n)), phi_std, g, torch.float32)
    return dict(phi=phi, alpha=torch.tensor([alpha], dtype=torch.float32), b=bias_init(n, diag))


def activations(T: int, n: int, C: int, seed: int, dtype: torch.dtype = torch.bfloat16,
                backward: bool = True) -> dict:
    """x [T,n,C], f_out [T,C] and (with backward) grad_x_next [T,n,C], grad_h_in [T,C],
    all ~ N(0,1) in ``dtype``."""
    g = _gen(seed + 1000)
    out = dict(x=_normal((T, n, C), 1.0, g, dtype), f_out=_normal((T, C), 1.0, g, dtype))
    if backward:
        out["grad_x_next"] = _normal((T, n, C), 1.0, g, dtype)
        out["grad_h_in"] = _normal((T, C), 1.0, g, dtype)
    return out


def layer_inputs(T: int, n: int, C: int, seed: int = 0, dtype: torch.dtype = torch.bfloat16,
                 backward: bool = True) -> dict:
    """Parameters plus activations for one layer."""
    d = layer_params(n, C, seed)
    d.update(activations(T, n, C, seed, dtype, backward))
    return d


def tiny_forward(seed: int = 0) -> dict:
    """T=64, n=4, C=256 fp32 inputs and the fixed random F = W [C, C] (std 1/16)."""
    T, n, C = 64, 4, 256
    d = layer_inputs(T, n, C, seed, torch.float32, backward=True)
    g = _gen(seed + 2000)
    d["W"] = _normal((C, C), 1.0 / 16.0, g, torch.float32)
    return d


def sinkhorn_logits(B: int, n: int, seed: int = 0, std: float = 2.0) -> torch.Tensor:
    """[B, n, n] fp32 logits ~ N(0, std)."""
    return _normal((B, n, n), std, _gen(seed + 3000), torch.float32)


def depth_gain(l: int) -> float:
    """Scalar s_l ~ U(0.5, 1.5) for layer l of the depth stack (F_l(h) = s_l h)."""
    g = _gen(l + 4000)
    return float(0.5 + torch.rand(1, generator=g).item())


def depth_stack_chunk(T: int, n: int, C: int, chunk: int,
                      dtype: torch.dtype = torch.bfloat16) -> dict:
    """One token chunk of the depth-stack workload: the stack input x_0 [T,n,C] and the
    upstream gradient of the last layer's output G_L [T,n,C], both ~ N(0,1).  Chunk k
    draws from its own seed, so any chunk can be regenerated alone."""
    g = _gen(chunk + 6000)
    return dict(x0=_normal((T, n, C), 1.0, g, dtype), G_last=_normal((T, n, C), 1.0, g, dtype))


def token_sample(T: int, k: int, seed: int = 0) -> torch.Tensor:
    """Sorted random subset of k distinct token indices in [0, T) (always includes the
    first and last token)."""
    g = _gen(seed + 5000)
    k = min(k, T)
    idx = torch.randperm(T, generator=g)[:k]
    idx = torch.unique(torch.cat([idx, torch.tensor([0, T - 1])]))
    return idx
