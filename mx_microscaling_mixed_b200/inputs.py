"""Seeded synthetic inputs shaped like the MXSens workloads.

This module holds none of the method's arithmetic: it only draws random
weights, calibration activations, layer activations and K/V tensors with the
shapes and outlier structure of the workloads the MXSens pages evaluate
(LLaMA-2/3 linear layers; W4A4KV4, [TS §4]).  The pages' real weights and
WikiText-2 / C4 calibration text are not available, so these draws stand in
for them.  Both the CUDA path and the CPU oracle consume the SAME bytes drawn
here (the oracle reads them back from the device), so nothing downstream
depends on the generator's numbers being reproducible across devices.

Recipes (one per workload):
  parity   W 256x256 fp32 N(0, 0.02^2); 5 columns (2%) x20 and 26 columns
           (10%) x3, disjoint, chosen by a seeded permutation; calibration
           X 128x256 fp32 N(0,1) and activations A 128x256 fp32 N(0,1) with
           the same 31 channels x10.
  attn     W 4096x4096 bf16 N(0, 0.02^2) with 3% of columns replaced by
           0.02 * Student-t(3); X 2048x4096 bf16 N(0,1) with 8 seeded outlier
           channels x50; A (M x 4096) drawn like X.
  mlp      gate/up W 14336x4096 as attn; down W 4096x14336 with X and A
           ~ Laplace(0, 0.1) plus 0.5% elementwise spikes x100.
  kv       K/V cache tokens x heads x head_dim bf16 N(0,1).
Student-t(3) = Z / sqrt(chi2_3 / 3); Laplace(0, b) = -b sgn(u) ln(1 - 2|u|),
u ~ U(-1/2, 1/2).
"""
from __future__ import annotations

import torch


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def outlier_columns(K: int, count: int, g: torch.Generator, device) -> torch.Tensor:
    """`count` distinct column indices from a seeded permutation of range(K)."""
    return torch.randperm(K, generator=g, device=device)[:count]


def _normal(shape, std, g, device):
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32) * std


def _student_t3(shape, g, device):
    z = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    c = torch.randn((3,) + tuple(shape), generator=g, device=device, dtype=torch.float32)
    chi2 = (c * c).sum(0)
    return z / torch.sqrt(chi2 / 3.0)


def _laplace(shape, b, g, device):
    u = torch.rand(shape, generator=g, device=device, dtype=torch.float32) - 0.5
    u = u.clamp(-0.4999999, 0.4999999)
    return -b * torch.sign(u) * torch.log1p(-2.0 * u.abs())


def parity_layer(device="cpu", seed: int = 0, M: int = 128, K: int = 256, N: int = 256,
                 T: int = 128):
    """The small parity workload (fp32 throughout)."""
    g = _gen(device, seed)
    W = _normal((N, K), 0.02, g, device)
    cols = outlier_columns(K, round(0.02 * K) + round(0.10 * K), g, device)
    extreme, mild = cols[:round(0.02 * K)], cols[round(0.02 * K):]
    W[:, extreme] *= 20.0
    W[:, mild] *= 3.0
    X = _normal((T, K), 1.0, g, device)
    X[:, cols] *= 10.0
    A = _normal((M, K), 1.0, g, device)
    A[:, cols] *= 10.0
    return {"W": W, "X": X, "A": A, "outlier_cols": cols}


def attn_weight(device, seed: int, N: int = 4096, K: int = 4096, std: float = 0.02,
                t_frac: float = 0.03):
    g = _gen(device, seed)
    W = _normal((N, K), std, g, device)
    cols = outlier_columns(K, round(t_frac * K), g, device)
    W[:, cols] = std * _student_t3((N, cols.numel()), g, device)
    return W.to(torch.bfloat16)


def gaussian_acts(device, seed: int, rows: int, K: int = 4096, n_outlier: int = 8,
                  scale: float = 50.0):
    """N(0,1) activations with `n_outlier` fixed channels scaled up."""
    g = _gen(device, seed)
    cols = outlier_columns(K, n_outlier, _gen(device, seed ^ 0x5EED), device)
    X = _normal((rows, K), 1.0, g, device)
    X[:, cols] *= scale
    return X.to(torch.bfloat16)


def laplace_acts(device, seed: int, rows: int, K: int = 14336, b: float = 0.1,
                 spike_frac: float = 0.005, spike: float = 100.0):
    g = _gen(device, seed)
    X = _laplace((rows, K), b, g, device)
    mask = torch.rand((rows, K), generator=g, device=device) < spike_frac
    X = torch.where(mask, X * spike, X)
    return X.to(torch.bfloat16)


def attn_layer(device="cuda", seed: int = 2000, M: int = 2048, T: int = 2048,
               N: int = 4096, K: int = 4096):
    """Llama-3-8B-shaped attention projection."""
    return {"W": attn_weight(device, seed, N, K),
            "X": gaussian_acts(device, seed + 1, T, K),
            "A": gaussian_acts(device, seed + 2, M, K)}


def mlp_down_layer(device="cuda", seed: int = 3000, M: int = 2048, T: int = 2048,
                   N: int = 4096, K: int = 14336):
    return {"W": attn_weight(device, seed, N, K),
            "X": laplace_acts(device, seed + 1, T, K),
            "A": laplace_acts(device, seed + 2, M, K)}


def kv_cache(device="cuda", seed: int = 4000, tokens: int = 8192, heads: int = 8,
             head_dim: int = 128):
    g = _gen(device, seed)
    return _normal((tokens, heads, head_dim), 1.0, g, device).to(torch.bfloat16)


def random_matrix(rows: int, cols: int, *, device="cpu", seed: int = 0,
                  dtype=torch.float32, std: float = 1.0, outlier_frac: float = 0.05,
                  outlier_scale: float = 30.0):
    """Generic N(0, std^2) matrix with a fraction of scaled columns (test sizes)."""
    g = _gen(device, seed)
    X = _normal((rows, cols), std, g, device)
    n_out = int(round(outlier_frac * cols))
    if n_out:
        X[:, outlier_columns(cols, n_out, g, device)] *= outlier_scale
    return X.to(dtype)
