"""Seeded synthetic inputs shaped like the model cards' layers.

This module only draws random numbers; it holds none of the quantizer's or the
matmul's arithmetic, so both the CUDA path's tests/bench and the CPU oracle can
take their inputs from here.  Everything is generated on the host with numpy's
PCG64 (``default_rng(seed)``) and returned as CPU torch tensors; bf16 values are
fp32 draws rounded to nearest even by torch.

Distributions (the pages quantize BF16 checkpoints of these models):
  * ``gaussian_with_outliers``: N(0, std^2) fp32 plus round(frac * O * I)
    positions (without replacement) set to +-k_sigma * std with random sign.
  * ``student_t``: Student-t with 4 degrees of freedom scaled to std 0.02
    (var(t_4) = 2, so t * std / sqrt(2)), drawn as z / sqrt(chi2_4 / 4) with
    chi2_4 = -2 ln(u1 u2); fp32 or rounded to bf16.
  * ``activations``: N(0, 1) rounded to bf16.
  * ``router_logits``: N(0, 1) fp32.
  * ``sign_vectors``: the two +-1 vectors of length 128 of the TQ3 rotation,
    fair coin flips (the producer's own generator for its seed is not known;
    these stand in for it).
"""

from __future__ import annotations

import math

import numpy as np
import torch


def _rng(seed: int) -> np.random.Generator:
    return np.random.default_rng(seed)


def gaussian_with_outliers(out_f: int, in_f: int, std: float = 0.02, frac: float = 0.001,
                           k_sigma: float = 20.0, seed: int = 0) -> torch.Tensor:
    rng = _rng(seed)
    w = rng.standard_normal((out_f, in_f), dtype=np.float32) * np.float32(std)
    n_out = int(round(frac * out_f * in_f))
    if n_out:
        pos = rng.choice(out_f * in_f, size=n_out, replace=False)
        sign = np.where(rng.random(n_out) < 0.5, -1.0, 1.0).astype(np.float32)
        w.reshape(-1)[pos] = sign * np.float32(k_sigma * std)
    return torch.from_numpy(w)


def student_t(shape, std: float = 0.02, df4_seed: int = 0, dtype=torch.bfloat16,
              chunk: int = 1 << 24) -> torch.Tensor:
    """Student-t(4) scaled to standard deviation ``std``."""
    rng = _rng(df4_seed)
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.float32)
    scale = std / math.sqrt(2.0)
    for s in range(0, n, chunk):
        m = min(chunk, n - s)
        z = rng.standard_normal(m)
        u = rng.random((2, m))
        chi2 = -2.0 * np.log((1.0 - u[0]) * (1.0 - u[1]))   # 1-u in (0, 1]
        out[s:s + m] = (z / np.sqrt(chi2 / 4.0) * scale).astype(np.float32)
    t = torch.from_numpy(out.reshape(shape))
    return t.to(dtype) if dtype != torch.float32 else t


def activations(rows: int, cols: int, seed: int = 1, dtype=torch.bfloat16) -> torch.Tensor:
    rng = _rng(seed)
    x = torch.from_numpy(rng.standard_normal((rows, cols), dtype=np.float32))
    return x.to(dtype) if dtype != torch.float32 else x


def router_logits(tokens: int, experts: int, seed: int = 2) -> torch.Tensor:
    rng = _rng(seed)
    return torch.from_numpy(rng.standard_normal((tokens, experts), dtype=np.float32))


def sign_vectors(seed: int = 42) -> torch.Tensor:
    """int8 [2][128] of +-1: row 0 is applied before the FWHT, row 1 after it."""
    bits = _rng(seed).integers(0, 2, size=(2, 128))
    return torch.from_numpy((1 - 2 * bits).astype(np.int8))


def uniform(shape, lo: float, hi: float, seed: int) -> np.ndarray:
    """Plain fp64 uniforms (used for rotated-domain probe values in tests)."""
    return _rng(seed).uniform(lo, hi, size=shape)


def student_t_device(shape, std: float = 0.02, seed: int = 0, dtype=torch.bfloat16,
                     device="cuda") -> torch.Tensor:
    """The same Student-t(4) recipe drawn on the device with torch's seeded
    generator (a different random stream from ``student_t``): used where the
    host would take too long to draw a large benchmark workload."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    n = int(np.prod(shape))
    out = torch.empty(n, dtype=dtype, device=device)
    scale = std / math.sqrt(2.0)
    chunk = 1 << 26
    for s in range(0, n, chunk):
        m = min(chunk, n - s)
        z = torch.randn(m, generator=g, device=device)
        u = torch.rand(2, m, generator=g, device=device)
        chi2 = -2.0 * torch.log((1.0 - u[0]) * (1.0 - u[1]))
        out[s:s + m] = (z / torch.sqrt(chi2 / 4.0) * scale).to(dtype)
    return out.view(shape)


def activations_device(rows: int, cols: int, seed: int = 1, dtype=torch.bfloat16, device="cuda") -> torch.Tensor:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return torch.randn(rows, cols, generator=g, device=device).to(dtype)
