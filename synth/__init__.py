"""Seeded synthetic inputs for the IsoQuant compressor and decode attention.

This module only draws data.  It holds none of the method's arithmetic (no
rotation, codebook, quantiser or attention), so both the float64 oracle and
the CUDA path can consume what it produces without sharing method code.

Every generator is deterministic in its seed.  The CPU generators use NumPy's
``Generator(PCG64(seed))`` and draw in float64 before casting with round to
nearest even; the GPU generators (``*_torch``) use a seeded
``torch.Generator`` on the target device for sizes a CPU generator cannot
produce in reasonable time, with the same recipe.

Workload recipes (the shapes of the pages' experiments; see the design notes):

* ``tiny_kv``: K and V rows N(0, 1)^d times a per-row radius
  r ~ LogNormal(0, 0.5); K first, then V, then the query N(0, 1)^d.
* ``unit_vectors``: normalised N(0, I_d) draws ("synthetic normalised
  vectors" of the IsoQuant stage-1 evaluation).
* ``student_t_kv``: i.i.d. Student-t (nu = 4) entries, built from the
  definition t = Z / sqrt(chi2_4 / 4) with chi2_4 a sum of four squared
  normals; per head, 4 distinct "outlier" channels drawn once and scaled by
  10 (K and V separately); rotary position embedding applied to K only
  (rotate-half pairs (i, i + d/2), angle p * base^(-2i/d), p = token index,
  base 1e6).  This stands in for the KV of a Qwen3-30B-A3B-shaped attention
  layer, whose real activations are not available here.
* ``ragged_lengths``: integer sequence lengths uniform in [lo, hi].
"""

from __future__ import annotations

import math

import numpy as np

__all__ = [
    "rng",
    "tiny_kv",
    "unit_vectors",
    "student_t_kv",
    "ragged_lengths",
    "queries",
    "student_t_kv_torch",
    "queries_torch",
    "random_packed_torch",
]


def rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def _cast(a: np.ndarray, dtype) -> np.ndarray:
    return np.asarray(a, dtype=np.float64).astype(dtype)


def tiny_kv(n: int = 4096, d: int = 128, seed: int = 0, dtype=np.float32):
    """K [1][n][d], V [1][n][d], q [1][1][d]: N(0,1)^d rows times LogNormal(0, 0.5)."""
    g = rng(seed)
    k = g.standard_normal((n, d)) * g.lognormal(0.0, 0.5, (n, 1))
    v = g.standard_normal((n, d)) * g.lognormal(0.0, 0.5, (n, 1))
    q = g.standard_normal((d,))
    return (_cast(k, dtype)[None], _cast(v, dtype)[None], _cast(q, dtype)[None, None])


def unit_vectors(n: int, d: int, seed: int, dtype=np.float32, n_heads: int = 1):
    """[n_heads][n][d] normalised N(0, I_d) samples, cast to ``dtype``."""
    g = rng(seed)
    x = g.standard_normal((n_heads, n, d))
    x /= np.sqrt(np.sum(x * x, axis=-1, keepdims=True))
    return _cast(x, dtype)


def _rope_rotate_half(x: np.ndarray, positions: np.ndarray, base: float) -> np.ndarray:
    """Rotary embedding, rotate-half convention, on the last axis of x [..., T, d]."""
    d = x.shape[-1]
    half = d // 2
    inv = base ** (-2.0 * np.arange(half) / d)
    ang = positions[:, None].astype(np.float64) * inv[None, :]
    cos, sin = np.cos(ang), np.sin(ang)
    a, b = x[..., :half], x[..., half:]
    return np.concatenate([a * cos - b * sin, a * sin + b * cos], axis=-1)


def _student_t4(g: np.random.Generator, shape) -> np.ndarray:
    z = g.standard_normal(shape)
    chi2 = np.zeros(shape)
    for _ in range(4):
        w = g.standard_normal(shape)
        chi2 += w * w
    return z / np.sqrt(chi2 / 4.0)


def student_t_kv(n_heads: int, t: int, d: int, seed: int, batch: int = 1,
                 dtype=np.float16, outliers: int = 4, outlier_scale: float = 10.0,
                 rope_base: float = 1e6):
    """K, V [batch][n_heads][t][d]: Student-t (nu=4) with outlier channels, RoPE on K."""
    g = rng(seed)
    out = []
    for is_key in (True, False):
        x = _student_t4(g, (batch, n_heads, t, d))
        for h in range(n_heads):
            ch = g.choice(d, size=outliers, replace=False)
            x[:, h, :, ch] *= outlier_scale
        if is_key:
            x = _rope_rotate_half(x, np.arange(t), rope_base)
        out.append(_cast(x, dtype))
    return out[0], out[1]


def queries(batch: int, hq: int, d: int, seed: int, dtype=np.float16):
    """[batch][hq][d] N(0, 1) queries."""
    return _cast(rng(seed).standard_normal((batch, hq, d)), dtype)


def ragged_lengths(batch: int, lo: int, hi: int, seed: int) -> np.ndarray:
    """int32 lengths uniform on the integers [lo, hi] (inclusive)."""
    return rng(seed).integers(lo, hi + 1, size=batch).astype(np.int32)


# ---------------------------------------------------------------------------
# Device-side generators for sizes beyond a CPU generator's reach
# ---------------------------------------------------------------------------

def student_t_kv_torch(batch: int, n_heads: int, t: int, d: int, seed: int,
                       device, outliers: int = 4, outlier_scale: float = 10.0,
                       rope_base: float = 1e6, chunk_tokens: int = 8192):
    """Same recipe as ``student_t_kv``, drawn with a seeded torch.Generator on
    ``device``; returns float16 K, V [batch][n_heads][t][d].

    Drawn in float32 chunks of ``chunk_tokens`` tokens to bound the transient
    memory; the stream differs from the NumPy generator's, the distribution
    does not.
    """
    import torch

    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    cpu_gen = torch.Generator()
    cpu_gen.manual_seed(seed)
    half = d // 2
    inv = rope_base ** (-2.0 * torch.arange(half, dtype=torch.float64) / d)
    result = []
    for is_key in (True, False):
        x = torch.empty((batch, n_heads, t, d), dtype=torch.float16, device=device)
        scale = torch.ones((n_heads, d), dtype=torch.float32)
        for h in range(n_heads):
            ch = torch.randperm(d, generator=cpu_gen)[:outliers]
            scale[h, ch] = outlier_scale
        scale = scale.to(device)
        for t0 in range(0, t, chunk_tokens):
            t1 = min(t, t0 + chunk_tokens)
            shape = (batch, n_heads, t1 - t0, d)
            z = torch.randn(shape, generator=gen, device=device)
            chi2 = torch.zeros(shape, device=device)
            for _ in range(4):
                w = torch.randn(shape, generator=gen, device=device)
                chi2.addcmul_(w, w)
            v = z / torch.sqrt(chi2 / 4.0)
            del z, chi2
            v *= scale[None, :, None, :]
            if is_key:
                pos = torch.arange(t0, t1, dtype=torch.float64)
                ang = (pos[:, None] * inv[None, :]).to(device)
                cos = torch.cos(ang).float()
                sin = torch.sin(ang).float()
                a, b = v[..., :half].clone(), v[..., half:].clone()
                v[..., :half] = a * cos - b * sin
                v[..., half:] = a * sin + b * cos
            x[:, :, t0:t1] = v.half()
            del v
        result.append(x)
    return result[0], result[1]


def queries_torch(batch: int, hq: int, d: int, seed: int, device):
    """[batch][hq][d] float16 N(0, 1) queries from a seeded device generator."""
    import torch

    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    return torch.randn((batch, hq, d), generator=gen, device=device).half()


def random_packed_torch(shape, seed: int, device):
    """Uniform random bytes of the given shape (a packed-code stand-in)."""
    import torch

    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    return torch.randint(0, 256, shape, generator=gen, device=device, dtype=torch.uint8)


def lognormal_norms(shape, seed: int, mean: float = math.log(16.0), sigma: float = 0.25):
    """Positive float16 norms (a stored-scale stand-in) from LogNormal(mean, sigma)."""
    return rng(seed).lognormal(mean, sigma, shape).astype(np.float16)
