"""Seeded synthetic inputs for the NF4 weight path.

This module holds random draws and dtype casts only; none of the method's
arithmetic.  The tests feed the same tensors to the CUDA library and to the CPU
oracle, the benchmark feeds them to the CUDA library, so parity never depends on
two random streams agreeing.

Workloads (no trained weights or datasets are available, so these stand in for
the 7B / 70B models the pages talk about; shapes follow the Llama-7B / 70B
linears):

* ``weight_normal``: W ~ N(0, std^2) drawn in fp32, optionally rounded to bf16;
* ``weight_student_t``: Student-t(nu) scaled to a target std, then a seeded set
  of input columns (a fraction of K) multiplied by a factor to plant outliers;
* ``activations``: X ~ N(0, 1) rounded to bf16;
* ``llama7b_stack``: the 32 x 7 linear shapes of a 7B decoder stack.

Seeds: ``seed = 1000 * config + tensor_index`` (config 1's W uses seed 0).
"""
from __future__ import annotations

import math

import torch

__all__ = ["weight_normal", "weight_student_t", "activations", "llama7b_stack", "LLAMA7B_LINEARS",
           "seed_for"]

# (name, out_features N, in_features K) of one Llama-7B decoder layer.
LLAMA7B_LINEARS = (
    ("q_proj", 4096, 4096), ("k_proj", 4096, 4096), ("v_proj", 4096, 4096),
    ("o_proj", 4096, 4096), ("gate_proj", 11008, 4096), ("up_proj", 11008, 4096),
    ("down_proj", 4096, 11008),
)


def seed_for(config: int, index: int) -> int:
    return 1000 * config + index


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def weight_normal(n: int, k: int, seed: int, std: float = 0.02, dtype=torch.bfloat16,
                  device="cpu") -> torch.Tensor:
    """[n, k] weight, N(0, std^2) drawn in fp32 then cast to ``dtype``."""
    g = _gen(seed, device)
    w = torch.randn((n, k), generator=g, device=device, dtype=torch.float32)
    w.mul_(std)
    return w if dtype == torch.float32 else w.to(dtype)


def weight_student_t(n: int, k: int, seed: int, nu: int = 4, std: float = 0.015,
                     outlier_frac: float = 0.001, outlier_scale: float = 20.0,
                     dtype=torch.bfloat16, device="cpu") -> torch.Tensor:
    """[n, k] heavy-tailed weight: t = z / sqrt(chi2_nu / nu) with chi2_nu a sum of
    nu squared normals, scaled by std / sqrt(nu / (nu - 2)) so its std is ``std``;
    then round(outlier_frac * k) seeded input columns are multiplied by
    ``outlier_scale``."""
    g = _gen(seed, device)
    z = torch.randn((n, k), generator=g, device=device, dtype=torch.float32)
    chi2 = torch.zeros_like(z)
    for _ in range(nu):
        e = torch.randn((n, k), generator=g, device=device, dtype=torch.float32)
        chi2.addcmul_(e, e)
        del e
    chi2.div_(nu).sqrt_()
    z.div_(chi2)
    del chi2
    z.mul_(std / math.sqrt(nu / (nu - 2.0)))
    n_out = int(round(outlier_frac * k))
    if n_out > 0:
        cols = torch.randperm(k, generator=g, device=device)[:n_out]
        z[:, cols] *= outlier_scale
    return z if dtype == torch.float32 else z.to(dtype)


def activations(m: int, k: int, seed: int, device="cpu") -> torch.Tensor:
    """[m, k] bf16 activations, N(0, 1) drawn in fp32 then rounded to bf16."""
    g = _gen(seed, device)
    return torch.randn((m, k), generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)


def llama7b_stack(n_layers: int = 32):
    """List of (layer, name, N, K) for the 7B-shaped stack (32 x 7 = 224 linears)."""
    return [(li, name, n, k) for li in range(n_layers) for (name, n, k) in LLAMA7B_LINEARS]
