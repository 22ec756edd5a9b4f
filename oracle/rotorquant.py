"""Float64 CPU oracle of the RotorQuant comparator (blockwise 3-D Clifford rotors).

TEST INFRASTRUCTURE ONLY, like ``oracle.isoquant``: imported by the tests, the
package smoke check and the benchmark's CPU legs, never by the product, and
sharing no code with the CUDA library.

Sources, cited by page title and section:

  [RT]  "RotorQuant" (the page on rotor-based KV-cache quantisation): each
        head vector is split into groups of three dimensions, the last group
        padded; each group is rotated by its own rotor with the sandwich
        product R v reverse(R); the rotated coordinates are Lloyd-Max
        quantised and packed; reconstruction inverts the rotation.  Its
        sparse rotor step keeps only the scalar and the three bivector
        coefficients of R.
  [IQ]  "IsoQuant" (arXiv 2603.28430), abstract: RotorQuant's forward
        rotation costs about 2,408 FMAs at d = 128; IsoQuant is compared
        with it on the stage-1 quantize-dequantize path.

Readings (the pages leave these open; the design notes list them):

  * Algebra Cl(3,0), e_i e_i = +1.  Multivectors are 8 components in the
    order (1, e1, e2, e3, e12, e13, e23, e123).  A rotor is
    R = s + p12 e12 + p13 e13 + p23 e23 with s^2 + |p|^2 = 1; its reverse
    negates the bivector part.
  * Groups: G = ceil(d / 3); group k holds dimensions 3k, 3k+1, 3k+2, the
    missing ones of the last group are zero.  All 3G rotated coordinates are
    quantised and stored (the padded coordinate does not stay zero).
  * Rotors: per head and group, four normals of the same SplitMix64 +
    Box-Muller stream as ``oracle.isoquant.make_params``, normalised, stored
    float32 [n_heads][G][4] as (s, p12, p13, p23).
  * Norm, codebook and scale as IsoQuant: s = ||x|| over the d real
    coordinates, x_hat = x / s, Lloyd-Max for N(0, 1/d) with code
    #{k : y > t_k}, float16 norm.
  * Packing: the 3G codes as one LSB-first bitstream, code i at bits
    [b i, b i + b), padded with zero bits to whole 32-bit words.
  * Cost: the pages' 2,408 FMAs at d = 128 are 43 groups x 56, which is the
    sandwich evaluated as the sparse rotor times the full 8-component
    multivector (8 outputs x 4 terms) and then that product times the dense
    8-component reverse for the three vector outputs (3 x 8 terms).
    ``sandwich`` follows that evaluation and counts it.
"""

from __future__ import annotations

import math

import numpy as np

from .isoquant import SplitMix64, gaussian_stream, make_codebook, quantize_scalar

# Blade bitmasks in the component order (1, e1, e2, e3, e12, e13, e23, e123).
BLADES = (0b000, 0b001, 0b010, 0b100, 0b011, 0b101, 0b110, 0b111)
_INDEX = {m: i for i, m in enumerate(BLADES)}


def _blade_product(a: int, b: int):
    """e_A e_B = sign * e_(A xor B) for Euclidean basis blades (bitmasks):
    the sign counts the transpositions that bring the product to canonical
    order, (-1)^#{(i in A, j in B) : j < i}."""
    swaps = 0
    x = a >> 1
    while x:
        swaps += bin(x & b).count("1")
        x >>= 1
    return (-1.0 if swaps & 1 else 1.0), a ^ b


# TABLE[i][j] = (sign, k): component i times component j lands on k.
TABLE = [[(_blade_product(BLADES[i], BLADES[j])[0], _INDEX[BLADES[i] ^ BLADES[j]]) for j in range(8)]
         for i in range(8)]
GRADE = tuple(bin(m).count("1") for m in BLADES)


def geometric_product(a, b):
    """Dense geometric product of multivectors [..., 8] (64 terms)."""
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    out = np.zeros(np.broadcast_shapes(a.shape, b.shape), dtype=np.float64)
    for i in range(8):
        for j in range(8):
            sgn, k = TABLE[i][j]
            out[..., k] += sgn * a[..., i] * b[..., j]
    return out


def reverse(a):
    """Reverse: grade k scaled by (-1)^(k (k - 1) / 2)."""
    a = np.asarray(a, dtype=np.float64)
    return a * np.array([(-1.0) ** (g * (g - 1) // 2) for g in GRADE])


def rotor_multivector(r):
    """(s, p12, p13, p23) [..., 4] -> multivector [..., 8]."""
    r = np.asarray(r, dtype=np.float64)
    out = np.zeros(r.shape[:-1] + (8,), dtype=np.float64)
    out[..., 0] = r[..., 0]
    out[..., 4:7] = r[..., 1:4]
    return out


def embed_vector(v):
    """3-vector [..., 3] -> multivector [..., 8] (grade 1 only)."""
    v = np.asarray(v, dtype=np.float64)
    out = np.zeros(v.shape[:-1] + (8,), dtype=np.float64)
    out[..., 1:4] = v
    return out


def sandwich(v, r, counter=None):
    """R v reverse(R) for 3-vectors v [..., 3] and rotors r [..., 4]
    ([RT] rotor sandwich), evaluated as the cost figure implies: first the
    sparse rotor (scalar + bivector terms only) times the embedded
    8-component multivector, all 8 outputs; then that product times the
    8-component reverse, the three vector outputs only.  ``counter`` (a
    one-element list) accumulates the multiply-adds: 32 + 24 per group."""
    x = embed_vector(v)
    rm = rotor_multivector(r)
    t = np.zeros(np.broadcast_shapes(x.shape, rm.shape), dtype=np.float64)
    for i in (0, 4, 5, 6):                 # the rotor's nonzero components
        for j in range(8):
            sgn, k = TABLE[i][j]
            t[..., k] += sgn * rm[..., i] * x[..., j]
    rr = reverse(rm)
    out = np.zeros(t.shape[:-1] + (3,), dtype=np.float64)
    for i in range(8):
        for j in range(8):
            sgn, k = TABLE[i][j]
            if k in (1, 2, 3):
                out[..., k - 1] += sgn * t[..., i] * rr[..., j]
    if counter is not None:
        groups = int(np.prod(out.shape[:-1], dtype=np.int64))
        counter[0] += (4 * 8 + 3 * 8) * groups
    return out


def sandwich_inverse(v, r):
    """reverse(R) v R: the inverse rotation (R reverse(R) = 1 for a unit rotor)."""
    rm = rotor_multivector(r)
    out = geometric_product(geometric_product(reverse(rm), embed_vector(v)), rm)
    return out[..., 1:4]


def n_groups(d: int) -> int:
    return (d + 2) // 3


def make_rotors(d: int, seed: int, n_heads: int = 1) -> np.ndarray:
    """Per-head, per-group unit rotors, float32 [n_heads][G][4] (s, p12, p13, p23):
    four normals of the shared generator per group, normalised in double."""
    g = gaussian_stream(SplitMix64(seed))
    out = np.empty((n_heads, n_groups(d), 4), dtype=np.float32)
    for h in range(n_heads):
        for k in range(n_groups(d)):
            v = [next(g) for _ in range(4)]
            n = math.sqrt(v[0] * v[0] + v[1] * v[1] + v[2] * v[2] + v[3] * v[3])
            out[h, k] = [v[0] / n, v[1] / n, v[2] / n, v[3] / n]
    return out


def packed_words(d: int, bits: int) -> int:
    """32-bit words per packed vector: ceil(3 G b / 32)."""
    return (3 * n_groups(d) * bits + 31) // 32


def packed_bytes(d: int, bits: int) -> int:
    return 4 * packed_words(d, bits)


def bitpack(codes, bits: int):
    """LSB-first bitstream of codes [..., n] into uint8 [..., 4 * ceil(n b / 32)]."""
    codes = np.asarray(codes, dtype=np.int64)
    n = codes.shape[-1]
    nbytes = 4 * ((n * bits + 31) // 32)
    out = np.zeros(codes.shape[:-1] + (nbytes,), dtype=np.int64)
    for i in range(n):
        for k in range(bits):
            pos = bits * i + k
            out[..., pos // 8] |= ((codes[..., i] >> k) & 1) << (pos % 8)
    return out.astype(np.uint8)


def bitunpack(packed, bits: int, n: int):
    packed = np.asarray(packed, dtype=np.int64)
    codes = np.zeros(packed.shape[:-1] + (n,), dtype=np.int64)
    for i in range(n):
        for k in range(bits):
            pos = bits * i + k
            codes[..., i] |= ((packed[..., pos // 8] >> (pos % 8)) & 1) << k
    return codes


def rotate(xhat, rotors_head, counter=None):
    """Pad x_hat [..., d] to 3G and rotate each group by its rotor -> [..., 3G]."""
    xhat = np.asarray(xhat, dtype=np.float64)
    d = xhat.shape[-1]
    g = n_groups(d)
    pad = np.zeros(xhat.shape[:-1] + (3 * g,), dtype=np.float64)
    pad[..., :d] = xhat
    groups = pad.reshape(xhat.shape[:-1] + (g, 3))
    return sandwich(groups, np.asarray(rotors_head, dtype=np.float64), counter).reshape(pad.shape)


def rotate_inverse(y, rotors_head, d: int):
    """Inverse rotation of each group, then the first d coordinates."""
    y = np.asarray(y, dtype=np.float64)
    g = n_groups(d)
    groups = y.reshape(y.shape[:-1] + (g, 3))
    back = sandwich_inverse(groups, np.asarray(rotors_head, dtype=np.float64))
    return back.reshape(y.shape)[..., :d]


def quantize(x, rotors, bits: int, return_rotated: bool = False):
    """RotorQuant stage-1 compression of x [n_heads][n_vec][d] ([RT]).

    Per vector: s = ||x||; x_hat = x / s (0 when s = 0); pad to 3G; rotate
    each group (sandwich); code = #{k : y > t_k} with IsoQuant's Lloyd-Max
    thresholds for N(0, 1/d); pack the 3G codes.  Returns (packed uint8
    [n_heads][n_vec][4 W], norms float16 [n_heads][n_vec]) and optionally y.
    """
    x = np.asarray(x, dtype=np.float64)
    n_heads, n_vec, d = x.shape
    _, thresholds = make_codebook(d, bits)
    packed = np.empty((n_heads, n_vec, packed_bytes(d, bits)), dtype=np.uint8)
    norms = np.empty((n_heads, n_vec), dtype=np.float16)
    ys = np.empty((n_heads, n_vec, 3 * n_groups(d))) if return_rotated else None
    for h in range(n_heads):
        s = np.sqrt(np.sum(x[h] * x[h], axis=-1))
        safe = np.where(s > 0, s, 1.0)
        xhat = np.where(s[:, None] > 0, x[h] / safe[:, None], 0.0)
        y = rotate(xhat, rotors[h])
        packed[h] = bitpack(quantize_scalar(y, thresholds), bits)
        norms[h] = s.astype(np.float16)
        if return_rotated:
            ys[h] = y
    if return_rotated:
        return packed, norms, ys
    return packed, norms


def dequantize(packed, norms, rotors, bits: int, d: int):
    """Reconstruction s16 * (inverse group rotations of c[codes])[:d]."""
    centroids, _ = make_codebook(d, bits)
    packed = np.asarray(packed)
    n_heads, n_vec, _ = packed.shape
    out = np.empty((n_heads, n_vec, d), dtype=np.float64)
    for h in range(n_heads):
        c = centroids[bitunpack(packed[h], bits, 3 * n_groups(d))]
        out[h] = rotate_inverse(c, rotors[h], d) * np.asarray(norms[h], dtype=np.float64)[:, None]
    return out


def rotation_fma_count(d: int) -> int:
    """Multiply-adds of one vector's forward rotation, counted by running it."""
    counter = [0]
    rotate(np.zeros((d,)), np.tile([1.0, 0.0, 0.0, 0.0], (n_groups(d), 1)), counter)
    return counter[0]
