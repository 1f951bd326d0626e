"""Seeded synthetic inputs shaped like the workloads the pages describe.

This module holds none of the method's arithmetic: it only draws random numbers and
rounds them to the storage dtype.  Both the CUDA path and the CPU oracle are fed from
here, and nothing else is shared between them.

Recipes (all seeds fixed):
  * Gaussian sketch matrix S [m, d]: fp16 of numpy ``default_rng(7).standard_normal``.
  * One-layer cache with outlier channels: K, V fp16 [1, 8, 512, 128] ~ N(0, 1) with
    channels 3 and 77 scaled by 10, then a query fp16 [1, 8, 128] ~ N(0, 1); seed 0.
  * Throughput sweep: [N, D] fp32 or fp16 ~ N(0, 1), k = max(1, round(0.01 D)) columns
    (drawn without replacement, shared by all rows) scaled by 20, N = floor(total / D);
    an fp32 query [D] ~ N(0, 1) from the same stream; seed 2000 + sweep index.
  * Model-shaped caches: N(0, 1) * sigma_c with sigma_c = exp(0.5 z), z ~ N(0, 1), one
    sigma per (cache tensor, head, channel), shared across batch and tokens, rounded to
    fp16.  Queries fp16 ~ N(0, 1).

Host draws use numpy PCG64 (bit-reproducible everywhere).  Caches too large to draw on
the host quickly are drawn on the GPU with torch's seeded Philox generator (same
distribution, different stream); the recipe name says which.
"""
from __future__ import annotations

import numpy as np

SKETCH_SEED = 7


def sketch_matrix(m: int = 256, d: int = 128, seed: int = SKETCH_SEED) -> np.ndarray:
    """Gaussian JL matrix S [m, d] with i.i.d. N(0, 1) entries, stored as fp16."""
    rng = np.random.default_rng(seed)
    return rng.standard_normal((m, d)).astype(np.float16)


def sketch_matrix_f64(m: int, d: int, seed: int) -> np.ndarray:
    """The same distribution kept in fp64 (for statistical checks of the estimator)."""
    return np.random.default_rng(seed).standard_normal((m, d))


def outlier_layer(seed: int = 0, batch: int = 1, heads: int = 8, tokens: int = 512,
                  head_dim: int = 128, outlier_channels=(3, 77), factor: float = 10.0):
    """One layer's K, V fp16 [B, H, T, D] ~ N(0,1) with outlier channels, then q [B, H, D]."""
    rng = np.random.default_rng(seed)
    shape = (batch, heads, tokens, head_dim)
    out = []
    for _ in range(2):
        x = rng.standard_normal(shape, dtype=np.float32)
        for c in outlier_channels:
            if c < head_dim:
                x[..., c] *= np.float32(factor)
        out.append(x.astype(np.float16))
    q = rng.standard_normal((batch, heads, head_dim), dtype=np.float32).astype(np.float16)
    return out[0], out[1], q


def sweep_rows(total: int, d: int) -> int:
    return total // d


def sweep_matrix(total: int, d: int, dtype, sweep_index: int, n_rows: int | None = None):
    """Throughput-sweep matrix [N, D] (N = total // D unless n_rows is given) with 1% of
    columns scaled by 20, and an fp32 query [D]."""
    rng = np.random.default_rng(2000 + sweep_index)
    n = sweep_rows(total, d) if n_rows is None else n_rows
    k = max(1, int(round(0.01 * d)))
    cols = rng.choice(d, k, replace=False)
    x = rng.standard_normal((n, d), dtype=np.float32)
    x[:, cols] *= np.float32(20.0)
    q = rng.standard_normal((d,), dtype=np.float32)
    return x.astype(dtype), q, np.sort(cols)


def channel_std(rng: np.random.Generator, shape) -> np.ndarray:
    """Per-channel standard deviations drawn from LogNormal(0, 0.5)."""
    return np.exp(0.5 * rng.standard_normal(shape)).astype(np.float32)


def lognormal_cache(seed: int, batch: int, heads: int, tokens: int, head_dim: int = 128,
                    n_tensors: int = 1):
    """n_tensors fp16 caches [B, H, T, D] ~ N(0,1) * sigma(head, channel), host-drawn."""
    rng = np.random.default_rng(seed)
    out = []
    for _ in range(n_tensors):
        sig = channel_std(rng, (1, heads, 1, head_dim))
        x = rng.standard_normal((batch, heads, tokens, head_dim), dtype=np.float32) * sig
        out.append(x.astype(np.float16))
    return out


def gaussian_queries(seed: int, batch: int, heads: int, head_dim: int = 128) -> np.ndarray:
    rng = np.random.default_rng(seed)
    return rng.standard_normal((batch, heads, head_dim), dtype=np.float32).astype(np.float16)


# --- device-side draws for the large caches (same distributions) ---------------------

def lognormal_cache_device(seed: int, shape, n_sigma_dims, device, out=None):
    """Draw an fp16 cache of ``shape`` on ``device`` with torch's seeded generator.

    ``shape`` is [..., H, T, D]; one sigma is drawn per index of every axis except the
    batch and token axes (the axes listed in ``n_sigma_dims`` are kept in sigma's shape,
    the others are broadcast).  Drawn one leading slice at a time to bound temporaries.
    """
    import torch

    g = torch.Generator(device=device)
    g.manual_seed(seed)
    shape = tuple(int(s) for s in shape)
    sig_shape = tuple(s if i in n_sigma_dims else 1 for i, s in enumerate(shape))
    sig = torch.exp(0.5 * torch.randn(sig_shape, generator=g, device=device))
    if out is None:
        out = torch.empty(shape, dtype=torch.float16, device=device)
    lead = shape[0]
    for i in range(lead):
        chunk = torch.randn(shape[1:], generator=g, device=device, dtype=torch.float32)
        chunk.mul_(sig[i if sig_shape[0] > 1 else 0])
        out[i].copy_(chunk)
        del chunk
    return out


def gaussian_queries_device(seed: int, shape, device):
    import torch

    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return torch.randn(tuple(shape), generator=g, device=device).to(torch.float16)


def sweep_matrix_device(total: int, d: int, dtype, sweep_index: int, device):
    """The throughput-sweep recipe drawn on the device (for the 1e9-element points): the
    scaled columns and the fp32 query come from numpy (seed 2000 + sweep index), the
    matrix from torch's seeded generator."""
    import torch

    rng = np.random.default_rng(2000 + sweep_index)
    n = sweep_rows(total, d)
    k = max(1, int(round(0.01 * d)))
    cols = np.sort(rng.choice(d, k, replace=False))
    q = rng.standard_normal((d,), dtype=np.float32)
    g = torch.Generator(device=device)
    g.manual_seed(2000 + sweep_index)
    tdt = torch.float16 if dtype == np.float16 else torch.float32
    x = torch.empty((n, d), dtype=tdt, device=device)
    factor = torch.ones(d, dtype=torch.float32, device=device)
    factor[torch.from_numpy(cols).to(device)] = 20.0
    step = max(1, (1 << 28) // d)
    for r0 in range(0, n, step):
        r1 = min(n, r0 + step)
        chunk = torch.randn((r1 - r0, d), generator=g, device=device, dtype=torch.float32)
        x[r0:r1].copy_(chunk.mul_(factor))
    return x, q, cols
