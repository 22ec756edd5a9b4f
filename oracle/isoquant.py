"""Float64 CPU oracle of IsoQuant KV compression and compressed-space decode attention.

TEST INFRASTRUCTURE ONLY.  The test suite, the package smoke check and the
benchmark's CPU-baseline / reference leg are the only code allowed to import
this module.  The product (the CUDA library behind ``include/isoq.h`` and its
Python binding) never imports, links or calls it, and this module imports
nothing from the product.  It is deliberately plain and slow: every step is
written out in float64 in the order the sources give it, vectorised only across
independent vectors, with no blocking, fusion or reordering of one vector's
arithmetic.

Sources, cited by page title and section:

  [RQ]  "RotaryQuant: Fitting 120B MoE Models on Consumer Hardware via Fused
        Compressed-Space Attention" (arXiv 2608.08081):
        §3.2 Algorithm 1 and Steps 1-4, eq. (2), "Rotation cost analysis";
        §3.3 eq. (5); §3.4 Table 2 (kernels A-D); Appendix A (inner-product
        preservation, compressed-space attention); Appendix B (SO(4)
        quaternion parameterisation).
  [IQ]  "IsoQuant: Hardware-Aligned SO(4) Isoclinic Rotations for LLM KV Cache
        Compression" (arXiv 2603.28430), abstract: T(v) = q_L v conj(q_R),
        IsoQuant-Full and IsoQuant-Fast, FMA counts 1,024 / 512 at d = 128.

Readings taken where the pages are silent (each is listed with its reason in
the repository's design notes):

  * WHT: H_d is the +-1 Sylvester matrix in natural order,
    H_ij = (-1)^popcount(i & j); the orthonormal transform is H_d / sqrt(d);
    no random sign diagonal.  The rotation is R = R_SO4 o (H_d / sqrt(d)).
  * A 4-block (x0, x1, x2, x3) is the quaternion x0 + x1 i + x2 j + x3 k,
    real part first, Hamilton convention ij = k.
  * Full: u = q_L (x) v (x) conj(q_R); Fast: u = q_L (x) v (left-isoclinic,
    q_R stored as the identity (1, 0, 0, 0)).
  * Parameters: per head d/4 blocks of 8 floats (q_L then q_R, each w,x,y,z),
    Haar-random unit quaternions from SplitMix64 + Box-Muller (see
    ``make_params``), rounded to float32.
  * Codebook: Lloyd-Max for N(0, 1/d), 2^b levels, the same for K and V and
    all heads; code = #{k : y > t_k} (ties go to the lower code).
  * Bit-pack: b = 2, 4: LSB-first little-endian bitstream per vector, code
    i at bits [b*i, b*i + b).  b = 3: 32-code groups of three little-endian
    32-bit words; codes 32k+8r+j in bits [4j, 4j+3) of word r, bit r of code
    32k+24+j in bit 4j+3 of word r.  Vectors are contiguous with no padding.
  * Scale: s = ||x||_2 is stored as float16 (round to nearest even); the
    vector is normalised by the unrounded s; dequantisation multiplies by the
    stored float16 s.  s = 0 gives x_hat = 0.
  * Decode attention: q is not normalised; q~ = R_K q; scores use the
    K-rotation of the query's KV head kvh = qh // G; the output is
    o = R_V^T o~; softmax is the natural-exponent softmax with the maximum
    subtracted; tokens j >= min(seq_len[b], Tmax) are masked; seq_len <= 0
    gives a zero output row.
"""

from __future__ import annotations

import math

import numpy as np

FULL = 0        # [IQ] IsoQuant-Full, after the WHT ([RQ] v3: R_SO4 o H_d)
FAST = 1        # [IQ] IsoQuant-Fast: left isoclinic factor only, after the WHT
PLANAR = 2      # [IQ] the 2-D special case, after the WHT (reading: see make_params)
BLOCK_SO4 = 3   # [RQ] §4.6 Table 8 v2: block SO(4) (Full map) without the WHT
SO3 = 4         # [RQ] §4.6 Table 8 v1: single-quaternion conjugation q v conj(q), no WHT
VARIANTS = (FULL, FAST, PLANAR, BLOCK_SO4, SO3)

_MASK64 = (1 << 64) - 1


# ---------------------------------------------------------------------------
# Parameter generator: SplitMix64 -> uniform (0, 1] -> Box-Muller -> Haar S^3
# ---------------------------------------------------------------------------

class SplitMix64:
    """SplitMix64 generator (Steele, Lea & Flood, "Fast splittable
    pseudorandom number generators", OOPSLA 2014).

    The state is a 64-bit counter advanced by the odd constant
    0x9E3779B97F4A7C15 each call; the output is the counter passed through
    the published three-step xor-shift-multiply finaliser.
    """

    def __init__(self, seed: int):
        self.state = int(seed) & _MASK64

    def next_u64(self) -> int:
        self.state = (self.state + 0x9E3779B97F4A7C15) & _MASK64
        z = self.state
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _MASK64
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _MASK64
        return z ^ (z >> 31)

    def next_uniform(self) -> float:
        """A uniform double in (0, 1]: the top 53 bits, plus one, times 2^-53."""
        return float((self.next_u64() >> 11) + 1) * 2.0 ** -53


def gaussian_stream(rng: SplitMix64):
    """Standard normal draws by the Box-Muller transform (Box & Muller 1958).

    Each pair of uniforms (u1, u2) yields r cos(2 pi u2) and then
    r sin(2 pi u2), with r = sqrt(-2 ln u1), in that order.
    """
    while True:
        u1 = rng.next_uniform()
        u2 = rng.next_uniform()
        r = math.sqrt(-2.0 * math.log(u1))
        theta = 2.0 * math.pi * u2
        yield r * math.cos(theta)
        yield r * math.sin(theta)


def _unit4(v):
    n = math.sqrt(v[0] * v[0] + v[1] * v[1] + v[2] * v[2] + v[3] * v[3])
    return [v[0] / n, v[1] / n, v[2] / n, v[3] / n]


def make_params(d: int, variant: int, seed: int, n_heads: int = 1) -> np.ndarray:
    """Per-head SO(4) block parameters, float32 [n_heads][d/4][8].

    [RQ] Appendix B: each of the d/4 blocks stores a pair of unit quaternions
    (q_L, q_R), 8 floats per block, 256 floats per head at d = 128.
    [RQ] §3.2 calls them learnable while its checklist says no training is
    done; this oracle draws them at random.  A normalised N(0, I_4) draw is
    uniform (Haar) on S^3.  Draw order: heads, then blocks, then q_L (4
    normals), then q_R (4 normals).  IsoQuant-Fast ([IQ]) keeps only q_L: its
    q_L equals Full's for the same seed (q_R's draws are still consumed) and
    its q_R slot holds the identity (1, 0, 0, 0).

    Every variant consumes the same eight normals per block:
      BLOCK_SO4 ([RQ] Table 8 v2) stores Full's pair unchanged;
      SO3 ([RQ] Table 8 v1, v -> q v conj(q)) stores q_L in both slots;
      PLANAR ([IQ]'s 2-D special case, a reading: the pages name it without
      detail) restricts both quaternions to the complex line span{1, i}:
      q_L = (a0, a1, 0, 0) / |(a0, a1)| from the first two of q_L's normals,
      q_R likewise from q_R's, so each is uniform on that circle.  For such
      a pair the block map q_L v conj(q_R) rotates the coordinate pairs
      (v0, v1) and (v2, v3) of the block independently (see ``planar_forward``).
    """
    if d % 4:
        raise ValueError("d must be a multiple of 4")
    g = gaussian_stream(SplitMix64(seed))
    out = np.empty((n_heads, d // 4, 8), dtype=np.float32)
    for h in range(n_heads):
        for i in range(d // 4):
            a = [next(g) for _ in range(4)]
            b = [next(g) for _ in range(4)]
            if variant == PLANAR:
                ql = _unit4([a[0], a[1], 0.0, 0.0])
                qr = _unit4([b[0], b[1], 0.0, 0.0])
            else:
                ql, qr = _unit4(a), _unit4(b)
            if variant == FAST:
                qr = [1.0, 0.0, 0.0, 0.0]
            elif variant == SO3:
                qr = ql
            out[h, i, 0:4] = ql
            out[h, i, 4:8] = qr
    return out


# ---------------------------------------------------------------------------
# Lloyd-Max scalar quantiser for a Gaussian source
# ---------------------------------------------------------------------------

_SQRT2 = math.sqrt(2.0)
_INV_SQRT_2PI = 1.0 / math.sqrt(2.0 * math.pi)


def _phi(x: float) -> float:
    """Standard normal density (0 at +-inf)."""
    if math.isinf(x):
        return 0.0
    return _INV_SQRT_2PI * math.exp(-0.5 * x * x)


def _cell_mass(a: float, b: float) -> float:
    """P(a < X < b) for X ~ N(0, 1), using the tail form that keeps precision."""
    if a >= 0.0:
        # both edges in the upper tail: Q(a) - Q(b), Q(x) = erfc(x / sqrt 2) / 2
        return 0.5 * (math.erfc(a / _SQRT2) - math.erfc(b / _SQRT2))
    if b <= 0.0:
        return 0.5 * (math.erfc(-b / _SQRT2) - math.erfc(-a / _SQRT2))
    return 1.0 - 0.5 * math.erfc(b / _SQRT2) - 0.5 * math.erfc(-a / _SQRT2)


def _normal_quantile(p: float) -> float:
    """Inverse of the standard normal CDF by bisection (initialisation only)."""
    lo, hi = -40.0, 40.0
    for _ in range(200):
        mid = 0.5 * (lo + hi)
        if 0.5 * math.erfc(-mid / _SQRT2) < p:
            lo = mid
        else:
            hi = mid
    return 0.5 * (lo + hi)


def lloyd_max_gaussian(bits: int, sigma: float = 1.0, tol: float = 2e-15,
                       max_iter: int = 100000):
    """Lloyd-Max quantiser for N(0, sigma^2) with 2^bits levels.

    [RQ] §3.2 Step 3: each rotated coordinate is quantised with a Lloyd-Max
    optimal codebook (Lloyd 1982; Max 1960).  Lloyd's iteration alternates the
    two optimality conditions: thresholds at the midpoints of adjacent
    centroids, and each centroid the conditional mean of its cell,
    E[X | a < X < b] = (phi(a) - phi(b)) / (Phi(b) - Phi(a)) in sigma units.
    It starts from the Gaussian quantiles (k + 1/2) / L and stops when no
    centroid moves by more than ``tol`` (sigma units).  The Gaussian density
    is log-concave and even, so the fixed point is unique and odd-symmetric
    (c_k = -c_{L-1-k}, middle threshold 0); each iterate is symmetrised,
    (c_k - c_{L-1-k}) / 2, so that rounding cannot break that symmetry.

    Returns (centroids[L], thresholds[L-1]) as float64, scaled by sigma.
    """
    levels = 1 << bits

    def symmetrise(c):
        return [0.5 * (c[k] - c[levels - 1 - k]) for k in range(levels)]

    c = symmetrise([_normal_quantile((k + 0.5) / levels) for k in range(levels)])
    for _ in range(max_iter):
        t = [0.5 * (c[k] + c[k + 1]) for k in range(levels - 1)]
        edges = [-math.inf] + t + [math.inf]
        new_c = []
        for k in range(levels):
            a, b = edges[k], edges[k + 1]
            new_c.append((_phi(a) - _phi(b)) / _cell_mass(a, b))
        new_c = symmetrise(new_c)
        delta = max(abs(x - y) for x, y in zip(new_c, c))
        c = new_c
        if delta <= tol:
            break
    t = [0.5 * (c[k] + c[k + 1]) for k in range(levels - 1)]
    return np.array(c) * sigma, np.array(t) * sigma


def make_codebook(d: int, bits: int):
    """Codebook for the post-rotation marginal of a unit vector in R^d.

    Reading of [RQ] §3.2 Step 3 ("post-rotation marginal"): after the WHT each
    coordinate of a unit vector has variance 1/d ([RQ] §3.2, "Why structured
    rotation works"); the codebook is Lloyd-Max for N(0, 1/d).
    """
    return lloyd_max_gaussian(bits, sigma=1.0 / math.sqrt(d))


# ---------------------------------------------------------------------------
# Walsh-Hadamard transform and quaternion block maps
# ---------------------------------------------------------------------------

def wht(x, counter=None):
    """Unnormalised Walsh-Hadamard transform H_d x along the last axis.

    [RQ] §3.2 Step 2 / eq. (2) and "Rotation cost analysis": the WHT is
    applied by its butterfly, d log2 d operations.  Stage h (h = 1, 2, 4, ...,
    d/2) replaces each pair (x_i, x_{i+h}), i with bit h clear, by
    (x_i + x_{i+h}, x_i - x_{i+h}).  The product of the stages is the Sylvester
    matrix in natural order.  ``counter`` (a one-element list) accumulates the
    number of add/subtract operations.
    """
    y = np.array(x, dtype=np.float64, copy=True)
    d = y.shape[-1]
    if d & (d - 1):
        raise ValueError("d must be a power of two")
    h = 1
    while h < d:
        for start in range(0, d, 2 * h):
            a = y[..., start:start + h].copy()
            b = y[..., start + h:start + 2 * h].copy()
            y[..., start:start + h] = a + b
            y[..., start + h:start + 2 * h] = a - b
            if counter is not None:
                counter[0] += 2 * h
        h *= 2
    return y


def hamilton(p, q, counter=None):
    """Quaternion product p (x) q on arrays [..., 4] ordered (w, x, y, z).

    Hamilton's rules i^2 = j^2 = k^2 = ijk = -1.  Each output component is a
    sum of four products, so one product is 16 multiply-adds; ``counter`` (a
    one-element list) accumulates that count per product and per vector.
    """
    p = np.asarray(p, dtype=np.float64)
    q = np.asarray(q, dtype=np.float64)
    pw, px, py, pz = p[..., 0], p[..., 1], p[..., 2], p[..., 3]
    qw, qx, qy, qz = q[..., 0], q[..., 1], q[..., 2], q[..., 3]
    out = np.empty(np.broadcast_shapes(p.shape, q.shape), dtype=np.float64)
    out[..., 0] = pw * qw - px * qx - py * qy - pz * qz
    out[..., 1] = pw * qx + px * qw + py * qz - pz * qy
    out[..., 2] = pw * qy - px * qz + py * qw + pz * qx
    out[..., 3] = pw * qz + px * qy - py * qx + pz * qw
    if counter is not None:
        counter[0] += 16 * int(np.prod(out.shape[:-1], dtype=np.int64))
    return out


def qconj(q):
    """Quaternion conjugate (w, -x, -y, -z)."""
    q = np.asarray(q, dtype=np.float64)
    return q * np.array([1.0, -1.0, -1.0, -1.0])


def planar_forward(v, ql, qr, counter=None):
    """The 2-D special case ([IQ] abstract) written as plane rotations.

    With q_L = (cos a, sin a, 0, 0) and q_R = (cos b, sin b, 0, 0), Hamilton's
    rules give q_L v = rotation of both pairs (v0, v1) and (v2, v3) by a, and
    v conj(q_R) = rotation of (v0, v1) by -b and of (v2, v3) by +b; so the
    block map is the plane rotation by a - b on the first pair and by a + b
    on the second, with cos(a -+ b) = w_L w_R +- x_L x_R and
    sin(a -+ b) = x_L w_R -+ w_L x_R.  Four multiply-adds per pair
    (``counter``), d * 2 per vector.
    """
    v = np.asarray(v, dtype=np.float64)
    ql = np.asarray(ql, dtype=np.float64)
    qr = np.asarray(qr, dtype=np.float64)
    c1 = ql[..., 0] * qr[..., 0] + ql[..., 1] * qr[..., 1]
    s1 = ql[..., 1] * qr[..., 0] - ql[..., 0] * qr[..., 1]
    c2 = ql[..., 0] * qr[..., 0] - ql[..., 1] * qr[..., 1]
    s2 = ql[..., 1] * qr[..., 0] + ql[..., 0] * qr[..., 1]
    u = np.empty(np.broadcast_shapes(v.shape, ql.shape), dtype=np.float64)
    u[..., 0] = c1 * v[..., 0] - s1 * v[..., 1]
    u[..., 1] = s1 * v[..., 0] + c1 * v[..., 1]
    u[..., 2] = c2 * v[..., 2] - s2 * v[..., 3]
    u[..., 3] = s2 * v[..., 2] + c2 * v[..., 3]
    if counter is not None:
        counter[0] += 8 * int(np.prod(u.shape[:-1], dtype=np.int64))
    return u


def so4_forward(v, ql, qr, variant, counter=None):
    """[IQ] abstract / [RQ] Algorithm 1: T(v) = q_L v conj(q_R) per 4-block.

    v: [..., nblk, 4]; ql, qr: [nblk, 4].  Full (and the no-WHT BLOCK_SO4,
    and SO3 whose q_R = q_L) applies both products; Fast keeps only the left
    isoclinic factor, T(v) = q_L v; PLANAR applies its two plane rotations.
    """
    if variant == PLANAR:
        return planar_forward(v, ql, qr, counter)
    u = hamilton(ql, v, counter)
    if variant != FAST:
        u = hamilton(u, qconj(qr), counter)
    return u


def so4_inverse(u, ql, qr, variant):
    """Inverse block map: conj(q_L) u q_R (Full and every variant but Fast)
    or conj(q_L) u (Fast).

    [RQ] §3.4 / Table 2 kernel D: the inverse rotation uses the transposed
    SO(4) blocks; for unit quaternions the transpose of v -> q_L v conj(q_R)
    is u -> conj(q_L) u q_R.
    """
    v = hamilton(qconj(ql), u)
    if variant != FAST:
        v = hamilton(v, qr)
    return v


def uses_wht(variant: int) -> bool:
    """[RQ] §4.6 Table 8: v3 (FULL, and FAST and PLANAR built the same way)
    composes the block map with the WHT; v1 (SO3) and v2 (BLOCK_SO4) do not."""
    return variant in (FULL, FAST, PLANAR)


def rotate(xhat, params_head, variant):
    """R x = R_SO4(H_d x / sqrt(d)) along the last axis ([RQ] eq. (2));
    R x = R_SO4 x for the variants without the WHT."""
    xhat = np.asarray(xhat, dtype=np.float64)
    d = xhat.shape[-1]
    p = np.asarray(params_head, dtype=np.float64).reshape(d // 4, 8)
    z = wht(xhat) / math.sqrt(d) if uses_wht(variant) else xhat
    blocks = z.reshape(z.shape[:-1] + (d // 4, 4))
    return so4_forward(blocks, p[:, 0:4], p[:, 4:8], variant).reshape(xhat.shape)


def rotate_inverse(y, params_head, variant):
    """R^T y = H_d (R_SO4^T y) / sqrt(d) ([RQ] Appendix A: R^-1 = R^T);
    R_SO4^T y for the variants without the WHT."""
    y = np.asarray(y, dtype=np.float64)
    d = y.shape[-1]
    p = np.asarray(params_head, dtype=np.float64).reshape(d // 4, 8)
    blocks = y.reshape(y.shape[:-1] + (d // 4, 4))
    v = so4_inverse(blocks, p[:, 0:4], p[:, 4:8], variant).reshape(y.shape)
    return wht(v) / math.sqrt(d) if uses_wht(variant) else v


# ---------------------------------------------------------------------------
# Scalar quantiser and bit-pack
# ---------------------------------------------------------------------------

def quantize_scalar(y, thresholds):
    """Lloyd-Max code of each coordinate: #{k : y > t_k} ([RQ] Algorithm 1)."""
    y = np.asarray(y, dtype=np.float64)
    codes = np.zeros(y.shape, dtype=np.int64)
    for t in thresholds:
        codes += (y > t)
    return codes


def packed_bytes(d: int, bits: int) -> int:
    """Bytes per packed vector, d * b / 8 ([RQ] §3.2 Step 4: 48 at d=128, b=3)."""
    return d * bits // 8


def _bitpack_lsb_first(codes, bits: int):
    codes = np.asarray(codes, dtype=np.int64)
    d = codes.shape[-1]
    out = np.zeros(codes.shape[:-1] + (packed_bytes(d, bits),), dtype=np.int64)
    for i in range(d):
        for k in range(bits):
            pos = bits * i + k
            out[..., pos // 8] |= ((codes[..., i] >> k) & 1) << (pos % 8)
    return out.astype(np.uint8)


def _bitunpack_lsb_first(packed, bits: int, d: int):
    packed = np.asarray(packed, dtype=np.int64)
    codes = np.zeros(packed.shape[:-1] + (d,), dtype=np.int64)
    for i in range(d):
        for k in range(bits):
            pos = bits * i + k
            codes[..., i] |= ((packed[..., pos // 8] >> (pos % 8)) & 1) << k
    return codes


def _words_to_bytes(words):
    """Little-endian bytes of a list of 32-bit word arrays."""
    out = []
    for w in words:
        for byte in range(4):
            out.append((w >> (8 * byte)) & 0xFF)
    return np.stack(out, axis=-1)


def _bitpack3_groups(codes):
    """BitPack_3 in 32-code groups of three little-endian 32-bit words.

    Group k holds codes 32k .. 32k+31 at bytes 12k .. 12k+11 (words w0, w1,
    w2).  For r in {0, 1, 2} and j in 0..7: bits [4j, 4j+3) of w_r hold code
    32k + 8r + j, and bit 4j+3 of w_r holds bit r of code 32k + 24 + j.
    """
    codes = np.asarray(codes, dtype=np.int64)
    d = codes.shape[-1]
    if d % 32:
        raise ValueError("3-bit packing needs d to be a multiple of 32")
    groups = []
    for k in range(d // 32):
        words = [np.zeros(codes.shape[:-1], dtype=np.int64) for _ in range(3)]
        for r in range(3):
            for j in range(8):
                words[r] |= (codes[..., 32 * k + 8 * r + j] & 7) << (4 * j)
                words[r] |= ((codes[..., 32 * k + 24 + j] >> r) & 1) << (4 * j + 3)
        groups.append(_words_to_bytes(words))
    return np.concatenate(groups, axis=-1).astype(np.uint8)


def _bitunpack3_groups(packed, d: int):
    packed = np.asarray(packed, dtype=np.int64)
    codes = np.zeros(packed.shape[:-1] + (d,), dtype=np.int64)
    for k in range(d // 32):
        words = []
        for r in range(3):
            base = 12 * k + 4 * r
            words.append(packed[..., base] | (packed[..., base + 1] << 8) |
                         (packed[..., base + 2] << 16) | (packed[..., base + 3] << 24))
        for r in range(3):
            for j in range(8):
                codes[..., 32 * k + 8 * r + j] = (words[r] >> (4 * j)) & 7
        for j in range(8):
            codes[..., 32 * k + 24 + j] = sum(((words[r] >> (4 * j + 3)) & 1) << r for r in range(3))
    return codes


def bitpack(codes, bits: int):
    """BitPack_b ([RQ] Algorithm 1): d codes of b bits in d*b/8 bytes.

    b = 2 and b = 4: LSB-first bitstream, code i at bits [b*i, b*i + b)
    (written bit by bit: bit k of code i goes to stream position b*i + k).
    b = 3: 32-code groups of three 32-bit words (``_bitpack3_groups``), a bit
    order chosen so that the codes sit in 4-bit fields.  The pages fix only
    the size (48 bytes at d = 128); the order within a vector is a reading.
    codes: integer array [..., d]; returns uint8 [..., d*b/8].
    """
    if bits == 3:
        return _bitpack3_groups(codes)
    return _bitpack_lsb_first(codes, bits)


def bitunpack(packed, bits: int, d: int):
    """Inverse of ``bitpack``: uint8 [..., d*b/8] -> int64 codes [..., d]."""
    if bits == 3:
        return _bitunpack3_groups(packed, d)
    return _bitunpack_lsb_first(packed, bits, d)


# ---------------------------------------------------------------------------
# Algorithm 1: quantise, and its inverse
# ---------------------------------------------------------------------------

def quantize(x, params, bits: int, variant: int, return_rotated: bool = False):
    """IsoQuant compression of every vector ([RQ] §3.2, Algorithm 1).

    x: [n_heads][n_vec][d] (any real dtype; its values are taken exactly);
    params: [n_heads][d/4][8].  Per vector: s = ||x||_2 (Step 1);
    x_hat = x / s (x_hat = 0 when s = 0); y = R_SO4(H_d x_hat / sqrt d)
    (Step 2, eq. 2); code_i = #{k : y_i > t_k} (Step 3); BitPack_b (Step 4).
    Returns (packed uint8 [n_heads][n_vec][d*b/8], norms float16
    [n_heads][n_vec]) and, with ``return_rotated``, also y (float64), whose
    distance to the nearest threshold tells how close each code is to a
    decision boundary.
    """
    x = np.asarray(x, dtype=np.float64)
    n_heads, n_vec, d = x.shape
    _, thresholds = make_codebook(d, bits)
    packed = np.empty((n_heads, n_vec, packed_bytes(d, bits)), dtype=np.uint8)
    norms = np.empty((n_heads, n_vec), dtype=np.float16)
    ys = np.empty_like(x) if return_rotated else None
    for h in range(n_heads):
        s = np.sqrt(np.sum(x[h] * x[h], axis=-1))
        safe = np.where(s > 0, s, 1.0)
        xhat = np.where(s[:, None] > 0, x[h] / safe[:, None], 0.0)
        y = rotate(xhat, params[h], variant)
        packed[h] = bitpack(quantize_scalar(y, thresholds), bits)
        norms[h] = s.astype(np.float16)
        if return_rotated:
            ys[h] = y
    if return_rotated:
        return packed, norms, ys
    return packed, norms


def dequantize(packed, norms, params, bits: int, variant: int, d: int):
    """Reconstruction s16 * R^T c[codes] ([RQ] §3.4 kernel D, Appendix A).

    packed: uint8 [n_heads][n_vec][d*b/8]; norms: float16 [n_heads][n_vec].
    Returns float64 [n_heads][n_vec][d]: x = float(s16) * H_d(R_SO4^T c) / sqrt d.
    """
    centroids, _ = make_codebook(d, bits)
    packed = np.asarray(packed)
    n_heads, n_vec, _ = packed.shape
    out = np.empty((n_heads, n_vec, d), dtype=np.float64)
    for h in range(n_heads):
        c = centroids[bitunpack(packed[h], bits, d)]
        out[h] = rotate_inverse(c, params[h], variant) * \
            np.asarray(norms[h], dtype=np.float64)[:, None]
    return out


# ---------------------------------------------------------------------------
# Decode attention: compressed space (A) and reconstructed (B)
# ---------------------------------------------------------------------------

def _softmax_weights(z):
    m = np.max(z)
    p = np.exp(z - m)
    return p / np.sum(p)


def _valid_len(seq_len, tmax):
    return int(min(max(int(seq_len), 0), tmax))


def decode_attention(q, packed_k, packed_v, norms_k, norms_v, seq_lens,
                     params_k, params_v, bits: int, variant: int, scale: float):
    """Fused decode attention in the rotated domain ([RQ] Appendix A, §3.4).

    q: [B][Hq][d]; packed_k/v: uint8 [B][Hkv][Tmax][d*b/8];
    norms_k/v: float16 [B][Hkv][Tmax]; seq_lens: [B];
    params_k/v: [Hkv][d/4][8].  For each (b, qh), kvh = qh // (Hq / Hkv),
    T = min(seq_len[b], Tmax):
      q~ = R_K q;   z_j = s^K_j <q~, c[codeK_j]> * scale;
      alpha = softmax(z);   o~ = sum_j alpha_j s^V_j c[codeV_j];
      o = R_V^T o~   (the inverse rotation is applied once, to the output).
    Returns float64 [B][Hq][d]; rows with T = 0 are zero.
    """
    q = np.asarray(q, dtype=np.float64)
    bsz, hq, d = q.shape
    hkv, tmax = packed_k.shape[1], packed_k.shape[2]
    group = hq // hkv
    centroids, _ = make_codebook(d, bits)
    out = np.zeros((bsz, hq, d), dtype=np.float64)
    for b in range(bsz):
        t = _valid_len(seq_lens[b], tmax)
        if t == 0:
            continue
        for kvh in range(hkv):
            kt = centroids[bitunpack(packed_k[b, kvh, :t], bits, d)] * \
                np.asarray(norms_k[b, kvh, :t], dtype=np.float64)[:, None]
            vt = centroids[bitunpack(packed_v[b, kvh, :t], bits, d)] * \
                np.asarray(norms_v[b, kvh, :t], dtype=np.float64)[:, None]
            for g in range(group):
                qh = kvh * group + g
                q_rot = rotate(q[b, qh], params_k[kvh], variant)
                alpha = _softmax_weights((kt @ q_rot) * scale)
                out[b, qh] = rotate_inverse(alpha @ vt, params_v[kvh], variant)
    return out


def prefill_attention(q, packed_k, packed_v, norms_k, norms_v, seq_lens,
                      params_k, params_v, bits: int, variant: int, scale: float):
    """Causal attention of a chunk of Tq new queries over the packed cache
    that already holds them ([RQ] §3.4 "early termination via causal
    masking" in kernel A; Figure 1's path with T_q > 1).

    q: [B][Tq][Hq][d]; the cache as in ``decode_attention``, with
    seq_lens[b] the cache length including the chunk.  Query t of row b sits
    at position p = seq_lens[b] - Tq + t and attends to tokens
    j <= p (and j < Tmax); a query with p < 0 gets a zero row.  Each query
    row is the compressed-space decode of ``decode_attention`` with
    p + 1 tokens.  Returns float64 [B][Tq][Hq][d].
    """
    q = np.asarray(q, dtype=np.float64)
    bsz, tq, hq, d = q.shape
    out = np.zeros((bsz, tq, hq, d), dtype=np.float64)
    for b in range(bsz):
        for t in range(tq):
            pos = int(seq_lens[b]) - tq + t
            if pos < 0:
                continue
            out[b, t] = decode_attention(q[b:b + 1, t], packed_k[b:b + 1], packed_v[b:b + 1],
                                         norms_k[b:b + 1], norms_v[b:b + 1], [pos + 1],
                                         params_k, params_v, bits, variant, scale)[0]
    return out


def decode_attention_reconstructed(q, packed_k, packed_v, norms_k, norms_v,
                                   seq_lens, params_k, params_v, bits: int,
                                   variant: int, scale: float):
    """Ordinary attention over the dequantised K and V ([RQ] Figure 1, top).

    K_hat_j = dequantize(codeK_j, s^K_j), V_hat_j likewise;
    o = sum_j softmax(<q, K_hat_j> * scale)_j V_hat_j.  By orthogonality of R
    ([RQ] Appendix A) this equals ``decode_attention`` up to rounding.
    """
    q = np.asarray(q, dtype=np.float64)
    bsz, hq, d = q.shape
    hkv, tmax = packed_k.shape[1], packed_k.shape[2]
    group = hq // hkv
    out = np.zeros((bsz, hq, d), dtype=np.float64)
    for b in range(bsz):
        t = _valid_len(seq_lens[b], tmax)
        if t == 0:
            continue
        for kvh in range(hkv):
            k_hat = dequantize(packed_k[b, kvh:kvh + 1, :t], norms_k[b, kvh:kvh + 1, :t],
                               params_k[kvh:kvh + 1], bits, variant, d)[0]
            v_hat = dequantize(packed_v[b, kvh:kvh + 1, :t], norms_v[b, kvh:kvh + 1, :t],
                               params_v[kvh:kvh + 1], bits, variant, d)[0]
            for g in range(group):
                qh = kvh * group + g
                alpha = _softmax_weights((k_hat @ q[b, qh]) * scale)
                out[b, qh] = alpha @ v_hat
    return out


def decode_append(k_new, v_new, packed_k, packed_v, norms_k, norms_v, seq_lens,
                  params_k, params_v, bits: int, variant: int):
    """One decode step's cache write ([RQ] Figure 1 and Appendix D: during
    decode each new K and V entry is compressed once and stored in the packed
    cache, which attention then reads).

    k_new, v_new: [B][Hkv][d]; cache arrays as in ``decode_attention``.
    For each batch row b with t = max(seq_lens[b], 0) < Tmax, the new vectors
    of every KV head are compressed by ``quantize`` (Algorithm 1) and stored
    at position t, and the row's length becomes t + 1.  A row already
    holding Tmax tokens is left unchanged and reported.
    Returns (packed_k, packed_v, norms_k, norms_v, seq_lens, full_rows) as
    new arrays; full_rows lists the rows that could not take the token.
    """
    packed_k, packed_v = np.array(packed_k), np.array(packed_v)
    norms_k, norms_v = np.array(norms_k), np.array(norms_v)
    lens = np.array(seq_lens, dtype=np.int64)
    tmax = packed_k.shape[2]
    full_rows = []
    for b in range(lens.shape[0]):
        t = max(int(lens[b]), 0)
        if t >= tmax:
            full_rows.append(b)
            continue
        pk, nk = quantize(np.asarray(k_new[b])[:, None, :], params_k, bits, variant)
        pv, nv = quantize(np.asarray(v_new[b])[:, None, :], params_v, bits, variant)
        packed_k[b, :, t], norms_k[b, :, t] = pk[:, 0], nk[:, 0]
        packed_v[b, :, t], norms_v[b, :, t] = pv[:, 0], nv[:, 0]
        lens[b] = t + 1
    return packed_k, packed_v, norms_k, norms_v, lens, full_rows


def split_partials(z, values, bounds):
    """Split-K partial states of softmax attention for one query row.

    z: scores [T]; values: [T][d]; bounds: increasing token offsets
    [0, t1, ..., T].  For each split k over [bounds[k], bounds[k+1]):
    m_k = max z, l_k = sum exp(z - m_k), acc_k = sum exp(z - m_k) v.
    Empty splits give (m = -inf, l = 0, acc = 0).
    """
    parts = []
    for k in range(len(bounds) - 1):
        lo, hi = bounds[k], bounds[k + 1]
        if hi <= lo:
            parts.append((-math.inf, 0.0, np.zeros(values.shape[1])))
            continue
        m = float(np.max(z[lo:hi]))
        p = np.exp(z[lo:hi] - m)
        parts.append((m, float(np.sum(p)), p @ values[lo:hi]))
    return parts


def combine_partials(parts):
    """Merge split-K partials: m* = max m_k, l = sum l_k e^(m_k - m*),
    o = sum acc_k e^(m_k - m*) / l (the flash-decode combine; [RQ] §2
    "Efficient attention" names FlashAttention as the analogue)."""
    m_star = max(m for m, _, _ in parts)
    l_tot = 0.0
    acc = np.zeros_like(parts[0][2])
    for m, l_k, a in parts:
        if l_k == 0.0:
            continue
        w = math.exp(m - m_star)
        l_tot += l_k * w
        acc = acc + a * w
    return acc / l_tot


# ---------------------------------------------------------------------------
# Operation counts the pages quote
# ---------------------------------------------------------------------------

def wht_op_count(d: int) -> int:
    """Add/subtract operations of one butterfly WHT, counted by running it."""
    counter = [0]
    wht(np.zeros((d,)), counter)
    return counter[0]


def so4_fma_count(d: int, variant: int) -> int:
    """Multiply-adds of the block rotation of one vector, counted by running it."""
    counter = [0]
    blocks = np.zeros((d // 4, 4))
    q = np.tile(np.array([1.0, 0.0, 0.0, 0.0]), (d // 4, 1))
    so4_forward(blocks, q, q, variant, counter)
    return counter[0]
