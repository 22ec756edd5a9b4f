"""Shared helpers of the test suite: tolerance checks that compare the CUDA
path with the float64 oracle, and GPU fixtures."""

from __future__ import annotations

import math
import os
import re

import numpy as np
import pytest

import oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "isoq.h")

# Tolerances (each is justified in the design notes):
#   codes: bit-exact except coordinates whose float64 rotated value lies within
#          CODE_BAND (unit-sphere units) of a decision threshold;
#   norms: float16 bit-exact except where the float64 norm lies within
#          NORM_BAND (relative) of a float16 rounding midpoint;
#   dequantised values: within DEQ_REL of the vector's norm (float32 output);
#   attention outputs: ATT_F16 max-abs (float16 output, plus the output's own
#          float16 rounding) and ATT_F32 max-abs (float32 output).
CODE_BAND = 1e-5
NORM_BAND = 1e-6
DEQ_REL = 1e-6
ATT_F16 = 2e-3
ATT_F32 = 1e-5


def header_functions():
    """Names of the functions declared in include/isoq.h."""
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(isoq_\w+)\s*\(", text)))


def gpu_available() -> bool:
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


def require_gpu():
    if not gpu_available():
        pytest.skip("needs a CUDA GPU")


def boundary_distance(y, thresholds):
    """Distance of each rotated coordinate to its nearest decision threshold."""
    y = np.asarray(y, dtype=np.float64)
    return np.min(np.abs(y[..., None] - np.asarray(thresholds)[None, :]), axis=-1)


def check_codes(gpu_packed, oracle_packed, oracle_y, bits, d, band=CODE_BAND):
    """Asserts codes agree except near a boundary; returns the mismatch count."""
    _, thresholds = O.make_codebook(d, bits)
    gc = O.bitunpack(np.asarray(gpu_packed), bits, d)
    oc = O.bitunpack(np.asarray(oracle_packed), bits, d)
    mism = gc != oc
    n = int(mism.sum())
    if n:
        dist = boundary_distance(np.asarray(oracle_y)[mism], thresholds)
        assert np.all(dist < band), f"{n} code mismatches, worst boundary distance {dist.max():.3g}"
        assert np.all(np.abs(gc[mism] - oc[mism]) == 1), "mismatched codes are not adjacent"
    return n


def check_norms(gpu_norms16, oracle_norms16, x_f64, band=NORM_BAND):
    """Asserts float16 norms agree bit for bit except at rounding midpoints."""
    g = np.asarray(gpu_norms16, dtype=np.float16)
    o = np.asarray(oracle_norms16, dtype=np.float16)
    mism = g.view(np.uint16) != o.view(np.uint16)
    n = int(mism.sum())
    if n:
        s = np.sqrt(np.sum(np.asarray(x_f64, dtype=np.float64) ** 2, axis=-1))[mism]
        mid = 0.5 * (g[mism].astype(np.float64) + o[mism].astype(np.float64))
        assert np.all(np.abs(s - mid) <= band * s), f"{n} norm mismatches away from a midpoint"
        ulps = np.abs(g[mism].view(np.uint16).astype(np.int64) - o[mism].view(np.uint16).astype(np.int64))
        assert np.all(ulps == 1)
    return n


def f16_half_ulp(v):
    """Half a float16 ulp at |v| (the float16 output's own rounding bound)."""
    a = np.abs(np.asarray(v, dtype=np.float64))
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -14)))
    return 2.0 ** (e - 11)


def check_attention(gpu_out, oracle_out, dtype, label=None):
    """Asserts the attention output is within the stated max-abs tolerance.

    float16 outputs: |err| <= 2e-3 + half a float16 ulp of the oracle's value,
    per element (the stated 2e-3 max-abs plus the output format's own
    rounding, which matters only where |o| > 4).
    float32 outputs: 1e-5 max-abs.

    Returns the largest absolute error.  When ISOQ_ATTENTION_LOG names a
    file, one JSON line per call is appended to it with the largest absolute
    error, the largest |o| and the smallest margin to the bar, so that a test
    run records how close each case came.
    """
    g = np.asarray(gpu_out, dtype=np.float64)
    o = np.asarray(oracle_out, dtype=np.float64)
    err = np.abs(g - o)
    if dtype == np.float16:
        tol = ATT_F16 + f16_half_ulp(o)
    else:
        tol = ATT_F32 + 0.0 * o
    _record_attention(label, dtype, err, o, tol)
    worst = float(np.max(err - tol)) if err.size else 0.0
    assert np.all(err <= tol), f"attention error exceeds tolerance by {worst:.3g} (max err {err.max():.3g})"
    return float(err.max()) if err.size else 0.0


def _record_attention(label, dtype, err, o, tol):
    path = os.environ.get("ISOQ_ATTENTION_LOG")
    if not path or not err.size:
        return
    import json
    if label is None:
        label = os.environ.get("PYTEST_CURRENT_TEST", "?").split(" ")[0]
    rec = {"case": label, "dtype": "f16" if dtype == np.float16 else "f32",
           "max_abs_err": float(err.max()), "max_abs_o": float(np.abs(o).max()),
           "min_margin": float(np.min(tol - err)),
           "max_err_where_abs_o_le_1": float(err[np.abs(o) <= 1].max()) if np.any(np.abs(o) <= 1) else None}
    with open(path, "a") as f:
        f.write(json.dumps(rec) + "\n")


def scale_for(d):
    return 1.0 / math.sqrt(d)
