"""Pins of the float64 oracle against facts fixed outside the oracle itself.

Each test checks the oracle against something it does not compute the same
way: a value printed on the method's pages or in the literature
(``tests/golden``), a closed form, an algebraic law, an independent
construction (the Sylvester recursion, quadrature, a dense matrix), or brute
force on a tiny case.  A dropped term, a wrong sign, a wrong index or a
transposed operand anywhere in the oracle fails at least one of them.
"""

import math
import os

import numpy as np
import pytest
from scipy import integrate

import oracle as O
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand_unit_quats(g, n):
    q = g.standard_normal((n, 4))
    return q / np.linalg.norm(q, axis=1, keepdims=True)


def _read_golden_pairs(name):
    rows = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            parts = [p.strip() for p in line.split("|")]
            rows[parts[0]] = float(parts[1])
    return rows


# ---------------------------------------------------------------------------
# Walsh-Hadamard transform
# ---------------------------------------------------------------------------

def _sylvester(d):
    h = np.array([[1.0]])
    while h.shape[0] < d:
        h = np.block([[h, h], [h, -h]])
    return h


@pytest.mark.parametrize("d", [4, 8, 16, 128, 256, 512])
def test_wht_equals_sylvester_recursion(d):
    # Column j of the transform is the transform of basis vector e_j.
    m = O.wht(np.eye(d)).T
    np.testing.assert_array_equal(m, _sylvester(d))


@pytest.mark.parametrize("d", [8, 128])
def test_wht_entries_closed_form(d):
    m = O.wht(np.eye(d)).T
    i, j = np.meshgrid(np.arange(d), np.arange(d), indexing="ij")
    popc = np.vectorize(lambda v: bin(int(v)).count("1"))(i & j)
    np.testing.assert_array_equal(m, (-1.0) ** popc)


@pytest.mark.parametrize("d", [128, 256, 512])
def test_wht_hht_is_d_identity_and_parseval(d):
    m = O.wht(np.eye(d))
    np.testing.assert_array_equal(m @ m.T, d * np.eye(d))
    g = np.random.default_rng(1)
    x = g.standard_normal((64, d))
    x /= np.linalg.norm(x, axis=1, keepdims=True)
    y = O.wht(x) / math.sqrt(d)
    np.testing.assert_allclose(np.sum(y * y, axis=1), 1.0, atol=1e-13)
    # A spike is spread to +-1/sqrt(d) in every coordinate: variance 1/d each
    # (RotaryQuant §3.2, "Why structured rotation works").
    spike = np.zeros(d)
    spike[3] = 1.0
    np.testing.assert_allclose(np.abs(O.wht(spike) / math.sqrt(d)), 1 / math.sqrt(d), atol=1e-15)


def test_wht_op_count_matches_pages():
    figs = _read_golden_pairs("page_figures.txt")
    assert O.wht_op_count(128) == figs["wht_fmas_d128"] == 128 * 7
    for d in (256, 512):
        assert O.wht_op_count(d) == d * int(math.log2(d))


# ---------------------------------------------------------------------------
# Quaternion algebra and the SO(4) block maps
# ---------------------------------------------------------------------------

ONE = np.array([1.0, 0, 0, 0])
I_ = np.array([0, 1.0, 0, 0])
J_ = np.array([0, 0, 1.0, 0])
K_ = np.array([0, 0, 0, 1.0])


def test_hamilton_basis_rules():
    h = O.hamilton
    for u in (I_, J_, K_):
        np.testing.assert_array_equal(h(u, u), -ONE)
    np.testing.assert_array_equal(h(I_, J_), K_)
    np.testing.assert_array_equal(h(J_, K_), I_)
    np.testing.assert_array_equal(h(K_, I_), J_)
    np.testing.assert_array_equal(h(J_, I_), -K_)
    np.testing.assert_array_equal(h(K_, J_), -I_)
    np.testing.assert_array_equal(h(I_, K_), -J_)
    np.testing.assert_array_equal(h(h(I_, J_), K_), -ONE)
    np.testing.assert_array_equal(h(ONE, I_), I_)


def test_hamilton_laws():
    g = np.random.default_rng(2)
    p, q, r = g.standard_normal((3, 100, 4))
    h = O.hamilton
    np.testing.assert_allclose(np.linalg.norm(h(p, q), axis=1),
                               np.linalg.norm(p, axis=1) * np.linalg.norm(q, axis=1), rtol=1e-14)
    np.testing.assert_allclose(h(h(p, q), r), h(p, h(q, r)), atol=1e-12)
    np.testing.assert_allclose(O.qconj(h(p, q)), h(O.qconj(q), O.qconj(p)), atol=1e-14)
    # p conj(p) = |p|^2 (real)
    pp = h(p, O.qconj(p))
    np.testing.assert_allclose(pp[:, 0], np.sum(p * p, axis=1), rtol=1e-14)
    np.testing.assert_allclose(pp[:, 1:], 0.0, atol=1e-14)


def _block_matrix(ql, qr, variant):
    cols = [O.so4_forward(e[None, :], ql[None, :], qr[None, :], variant)[0]
            for e in np.eye(4)]
    return np.stack(cols, axis=1)


def _left_matrix(q):
    """q (x) v as a matrix acting on v = (w, x, y, z), rows typed out from
    Hamilton's rules (RotaryQuant Appendix B; IsoQuant abstract)."""
    w, x, y, z = q
    return np.array([[w, -x, -y, -z],
                     [x, w, -z, y],
                     [y, z, w, -x],
                     [z, -y, x, w]])


def _right_matrix(p):
    """v (x) p as a matrix acting on v, rows typed out from Hamilton's rules."""
    w, x, y, z = p
    return np.array([[w, -x, -y, -z],
                     [x, w, z, -y],
                     [y, -z, w, x],
                     [z, y, -x, w]])


@pytest.mark.parametrize("variant", [O.FULL, O.FAST, O.BLOCK_SO4, O.SO3])
def test_block_maps_equal_explicit_4x4_matrices(variant):
    """RotaryQuant §3.3 / Appendix B: T(v) = q_L v conj(q_R) is the 4x4 matrix
    L(q_L) R(conj q_R) (Full, and the no-WHT block map; v1 repeats q_L in the
    right slot), and IsoQuant-Fast keeps L(q_L) alone.  The matrices are typed
    out independently of the oracle's Hamilton product; the inverse map is
    their transpose.  Checked on random inputs, including non-unit
    quaternions (the identities are algebraic)."""
    g = np.random.default_rng(11)
    for trial in range(40):
        ql, qr = g.standard_normal((2, 4))
        if trial % 2 == 0:
            ql, qr = ql / np.linalg.norm(ql), qr / np.linalg.norm(qr)
        if variant == O.SO3:
            qr = ql
        conj_qr = qr * np.array([1.0, -1.0, -1.0, -1.0])
        m = _left_matrix(ql) if variant == O.FAST else _left_matrix(ql) @ _right_matrix(conj_qr)
        v = g.standard_normal((7, 4))
        fwd = O.so4_forward(v[:, None, :], ql[None, :], qr[None, :], variant)[:, 0]
        scale = np.max(np.abs(v)) * np.sum(ql * ql) * max(1.0, np.sum(qr * qr))
        np.testing.assert_allclose(fwd, v @ m.T, rtol=0, atol=4e-15 * scale)
        inv = O.so4_inverse(v[:, None, :], ql[None, :], qr[None, :], variant)[:, 0]
        np.testing.assert_allclose(inv, v @ m, rtol=0, atol=4e-15 * scale)


def _complex_line(g, n):
    a = g.standard_normal((n, 2))
    a /= np.linalg.norm(a, axis=1, keepdims=True)
    return np.concatenate([a, np.zeros((n, 2))], axis=1)


@pytest.mark.parametrize("variant", O.VARIANTS)
def test_block_map_is_rotation_in_so4(variant):
    g = np.random.default_rng(3)
    draw = _complex_line if variant == O.PLANAR else _rand_unit_quats
    for ql, qr in zip(draw(g, 50), draw(g, 50)):
        if variant == O.SO3:
            qr = ql
        m = _block_matrix(ql, qr, variant)
        np.testing.assert_allclose(m.T @ m, np.eye(4), atol=1e-14)
        assert abs(np.linalg.det(m) - 1.0) < 1e-13  # SO(4), not a reflection
        v = g.standard_normal(4)
        np.testing.assert_allclose(np.linalg.norm(m @ v), np.linalg.norm(v), rtol=1e-14)
        back = O.so4_inverse((m @ v)[None, :], ql[None, :], qr[None, :], variant)[0]
        np.testing.assert_allclose(back, v, atol=1e-14)


def test_single_quaternion_conjugation_is_so3_rotation():
    """RotaryQuant Appendix B: v -> q v conj(q) fixes Re(v) and rotates the
    imaginary part; textbook (Rodrigues): by angle 2*theta about axis u for
    q = (cos theta, sin theta * u).  This pins the conj on the right factor."""
    g = np.random.default_rng(4)
    for _ in range(20):
        theta = g.uniform(0, math.pi)
        u = g.standard_normal(3)
        u /= np.linalg.norm(u)
        q = np.concatenate([[math.cos(theta)], math.sin(theta) * u])
        v = g.standard_normal(4)
        out = O.so4_forward(v[None, :], q[None, :], q[None, :], O.FULL)[0]
        assert abs(out[0] - v[0]) < 1e-14
        a = 2 * theta
        w = v[1:]
        rod = w * math.cos(a) + np.cross(u, w) * math.sin(a) + u * np.dot(u, w) * (1 - math.cos(a))
        np.testing.assert_allclose(out[1:], rod, atol=1e-13)


def test_fast_is_left_isoclinic_and_full_with_identity_right():
    g = np.random.default_rng(5)
    for q in _rand_unit_quats(g, 20):
        m = _block_matrix(q, ONE, O.FAST)
        for v in g.standard_normal((5, 4)):
            # every vector is turned by the same angle: <v, Lv> = q_w |v|^2
            assert abs(v @ (m @ v) - q[0] * (v @ v)) < 1e-13
        np.testing.assert_allclose(m, _block_matrix(q, ONE, O.FULL), atol=1e-15)
        np.testing.assert_allclose(m, _block_matrix(q, _rand_unit_quats(g, 1)[0], O.FAST), atol=0)


def test_planar_is_the_complex_line_special_case():
    """IsoQuant names a 2-D special case of q_L v conj(q_R).  With both
    quaternions on the complex line span{1, i} the Hamilton products reduce
    to two independent plane rotations, by angle(q_L) - angle(q_R) on the
    block's first coordinate pair and angle(q_L) + angle(q_R) on the second
    (angles from atan2, independently of the product formulas)."""
    g = np.random.default_rng(8)
    ql, qr = _complex_line(g, 40), _complex_line(g, 40)
    v = g.standard_normal((40, 4))
    hamilton_full = O.so4_forward(v, ql, qr, O.FULL)
    np.testing.assert_allclose(O.planar_forward(v, ql, qr), hamilton_full, atol=1e-14)
    a = np.arctan2(ql[:, 1], ql[:, 0])
    b = np.arctan2(qr[:, 1], qr[:, 0])

    def rot(t, x, y):
        return np.cos(t) * x - np.sin(t) * y, np.sin(t) * x + np.cos(t) * y

    u01 = rot(a - b, v[:, 0], v[:, 1])
    u23 = rot(a + b, v[:, 2], v[:, 3])
    np.testing.assert_allclose(hamilton_full, np.stack([*u01, *u23], axis=1), atol=1e-13)
    # the planar inverse is the Full inverse with the same pair
    back = O.so4_inverse(O.planar_forward(v, ql, qr), ql, qr, O.PLANAR)
    np.testing.assert_allclose(back, v, atol=1e-14)
    # "lightweight": four multiply-adds per coordinate pair
    assert O.so4_fma_count(128, O.PLANAR) == 2 * 128


def test_single_quaternion_variant_leaves_a_quarter_unmixed():
    """RotaryQuant §4.6 Table 8, v1: v -> q v conj(q) spans only SO(3) and
    leaves one coordinate per block (25 % of all) unmixed; v2 (block SO(4)
    without the WHT) mixes only inside each block; v3 (WHT + SO(4)) mixes
    every coordinate into every other."""
    d = 128
    x = np.random.default_rng(9).standard_normal(d)
    y1 = O.rotate(x, O.make_params(d, O.SO3, seed=3)[0], O.SO3)
    # (|q|^2 = 1 to float32 rounding of the stored parameters)
    np.testing.assert_allclose(y1[0::4], x[0::4], rtol=1e-6)
    assert np.max(np.abs(y1[1::4] - x[1::4])) > 0.1
    # Jacobians: block-diagonal for v1 and v2, dense for v3
    for var in (O.SO3, O.BLOCK_SO4):
        r = O.rotate(np.eye(d), O.make_params(d, var, seed=3)[0], var).T
        mask = np.kron(np.eye(d // 4), np.ones((4, 4))) > 0
        assert np.all(r[~mask] == 0.0)
    r3 = O.rotate(np.eye(d), O.make_params(d, O.FULL, seed=3)[0], O.FULL).T
    assert np.count_nonzero(np.abs(r3) > 1e-12) > 0.99 * d * d


def test_rotation_fma_counts_match_pages():
    figs = _read_golden_pairs("page_figures.txt")
    assert O.so4_fma_count(128, O.FULL) == figs["isoquant_full_fmas_d128"]
    assert O.so4_fma_count(128, O.FAST) == figs["isoquant_fast_fmas_d128"]
    # RotaryQuant's 16 per block / 512 total is one product per block.
    assert O.so4_fma_count(128, O.FAST) == figs["so4_fmas_d128"] == 32 * figs["so4_fmas_per_block"]
    assert O.wht_op_count(128) + O.so4_fma_count(128, O.FAST) == figs["rotation_fmas_d128"]


# ---------------------------------------------------------------------------
# Composite rotation R = R_SO4 o (H_d / sqrt d)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("d", [128, 256])
@pytest.mark.parametrize("variant", O.VARIANTS)
def test_composite_rotation_orthogonal_and_inverse(d, variant):
    p32 = O.make_params(d, variant, seed=11)[0]
    # The stored parameters are float32, so their quaternions have unit norm
    # only to ~1e-7 and R is orthogonal to that level.
    r32 = O.rotate(np.eye(d), p32, variant).T
    np.testing.assert_allclose(r32.T @ r32, np.eye(d), atol=1e-6)
    # With exactly normalised float64 quaternions R is orthogonal to rounding.
    p = p32.astype(np.float64).reshape(d // 4, 2, 4)
    p = (p / np.linalg.norm(p, axis=-1, keepdims=True)).reshape(d // 4, 8)
    if variant == O.SO3:
        p[:, 4:] = p[:, :4]
    r = O.rotate(np.eye(d), p, variant).T          # column j = R e_j
    np.testing.assert_allclose(r.T @ r, np.eye(d), atol=1e-13)
    rinv = O.rotate_inverse(np.eye(d), p, variant).T
    np.testing.assert_allclose(rinv, r.T, atol=1e-13)
    g = np.random.default_rng(6)
    x, y = g.standard_normal((2, d))
    # RotaryQuant Appendix A: <Rx, Ry> = <x, y>
    assert abs(O.rotate(x, p, variant) @ O.rotate(y, p, variant) - x @ y) < 1e-11
    # Block structure: R e_j restricted to one block equals the block map of
    # the WHT column, independently rebuilt from the Sylvester matrix.
    h = _sylvester(d) / math.sqrt(d) if O.uses_wht(variant) else np.eye(d)
    blk = 5
    m = _block_matrix(p[blk, :4].astype(np.float64), p[blk, 4:].astype(np.float64), variant)
    np.testing.assert_allclose(r[4 * blk:4 * blk + 4, :], m @ h[4 * blk:4 * blk + 4, :], atol=1e-14)


# ---------------------------------------------------------------------------
# Parameter generator
# ---------------------------------------------------------------------------

def test_splitmix64_published_vector():
    with open(os.path.join(GOLDEN, "splitmix64_seed1234567.txt")) as f:
        lines = [ln.strip() for ln in f if ln.strip() and not ln.startswith("#")]
    seed = int(lines[0].split()[1])
    expect = [int(v) for v in lines[1:]]
    r = O.SplitMix64(seed)
    assert [r.next_u64() for _ in expect] == expect


def test_box_muller_moments():
    g = O.gaussian_stream(O.SplitMix64(99))
    x = np.array([next(g) for _ in range(200000)])
    assert abs(x.mean()) < 0.01
    assert abs(x.var() - 1.0) < 0.01
    assert abs(np.mean(x ** 4) - 3.0) < 0.06          # Gaussian kurtosis
    assert abs(np.mean(x[0::2] * x[1::2])) < 0.01     # cos/sin pair uncorrelated


def test_params_layout_and_draws():
    figs = _read_golden_pairs("page_figures.txt")
    full = O.make_params(128, O.FULL, seed=1, n_heads=3)
    fast = O.make_params(128, O.FAST, seed=1, n_heads=3)
    assert full.shape == (3, 32, 8) and full.dtype == np.float32
    assert full[0].size == figs["stored_params_per_head_d128"]
    assert 32 * 6 == figs["effective_dof_per_head_d128"]
    np.testing.assert_allclose(np.linalg.norm(full[..., :4], axis=-1), 1.0, atol=1e-6)
    np.testing.assert_allclose(np.linalg.norm(full[..., 4:], axis=-1), 1.0, atol=1e-6)
    np.testing.assert_array_equal(fast[..., :4], full[..., :4])
    np.testing.assert_array_equal(fast[..., 4:], np.tile([1, 0, 0, 0], (3, 32, 1)))
    assert not np.array_equal(full[0], full[1])
    # The stream is the one generator, drawn in order: head h continues it.
    one = O.make_params(128, O.FULL, seed=1, n_heads=1)
    np.testing.assert_array_equal(one[0], full[0])
    # The first q_L is the first four Box-Muller normals, normalised.
    g = O.gaussian_stream(O.SplitMix64(1))
    v = np.array([next(g) for _ in range(4)])
    np.testing.assert_array_equal(full[0, 0, :4], (v / np.linalg.norm(v)).astype(np.float32))
    # The variants consume the same eight normals per block.
    np.testing.assert_array_equal(O.make_params(128, O.BLOCK_SO4, seed=1, n_heads=3), full)
    so3 = O.make_params(128, O.SO3, seed=1, n_heads=3)
    np.testing.assert_array_equal(so3[..., :4], full[..., :4])
    np.testing.assert_array_equal(so3[..., 4:], full[..., :4])
    pl = O.make_params(128, O.PLANAR, seed=1, n_heads=3)
    np.testing.assert_array_equal(pl[..., 2:4], 0.0)
    np.testing.assert_array_equal(pl[..., 6:8], 0.0)
    np.testing.assert_allclose(np.hypot(pl[..., 0], pl[..., 1]), 1.0, atol=1e-6)
    w = np.array([next(g) for _ in range(4)])             # q_R's normals of block 0
    np.testing.assert_array_equal(pl[0, 0, :2], (v[:2] / np.linalg.norm(v[:2])).astype(np.float32))
    np.testing.assert_array_equal(pl[0, 0, 4:6], (w[:2] / np.linalg.norm(w[:2])).astype(np.float32))


def test_params_are_haar_distributed():
    p = O.make_params(512, O.FULL, seed=7, n_heads=16).reshape(-1, 8)
    q = np.concatenate([p[:, :4], p[:, 4:]]).astype(np.float64)
    # Uniform on S^3: each component has mean 0 and second moment 1/4.
    np.testing.assert_allclose(q.mean(axis=0), 0.0, atol=0.03)
    np.testing.assert_allclose((q * q).mean(axis=0), 0.25, atol=0.015)


# ---------------------------------------------------------------------------
# Lloyd-Max codebook
# ---------------------------------------------------------------------------

def _read_max_table():
    table = {}
    with open(os.path.join(GOLDEN, "lloyd_max_gaussian_max1960.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            parts = line.split()
            table[(int(parts[0]), parts[1])] = np.array([float(v) for v in parts[2:]])
    return table


def _phi(x):
    return math.exp(-0.5 * x * x) / math.sqrt(2 * math.pi)


def _distortion(c, t):
    edges = [-np.inf] + list(t) + [np.inf]
    total = 0.0
    for k in range(len(c)):
        val, _ = integrate.quad(lambda x: (x - c[k]) ** 2 * _phi(x), edges[k], edges[k + 1],
                                epsabs=1e-15, epsrel=1e-13, limit=200)
        total += val
    return total


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_lloyd_max_matches_max_1960(bits):
    table = _read_max_table()
    c, t = O.lloyd_max_gaussian(bits)
    half = len(c) // 2
    np.testing.assert_allclose(c[half:], table[(bits, "output")], atol=1.5e-3)
    np.testing.assert_allclose(t[half - 1:], table[(bits, "threshold")], atol=1.5e-3)
    mse = _distortion(c, t)
    assert abs(mse - table[(bits, "mse")][0]) < 2e-4 * max(1.0, table[(bits, "mse")][0] * 10)


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_lloyd_max_optimality_by_quadrature(bits):
    """Centroid condition checked by numerical integration, independent of
    the erf/erfc closed forms the oracle iterates with."""
    c, t = O.lloyd_max_gaussian(bits)
    edges = [-np.inf] + list(t) + [np.inf]
    for k in range(len(c)):
        num, _ = integrate.quad(lambda x: x * _phi(x), edges[k], edges[k + 1], epsabs=1e-16, epsrel=1e-14)
        den, _ = integrate.quad(_phi, edges[k], edges[k + 1], epsabs=1e-16, epsrel=1e-14)
        assert abs(num / den - c[k]) < 1e-12
    np.testing.assert_allclose(t, 0.5 * (c[:-1] + c[1:]), atol=0)
    np.testing.assert_array_equal(c, -c[::-1])
    assert np.all(np.diff(c) > 0)


def test_one_bit_closed_form_and_scaling():
    c, t = O.lloyd_max_gaussian(1)
    np.testing.assert_allclose(c, [-math.sqrt(2 / math.pi), math.sqrt(2 / math.pi)], rtol=1e-14)
    for d in (128, 256, 512):
        for b in (2, 3, 4):
            cd, td = O.make_codebook(d, b)
            c1, t1 = O.lloyd_max_gaussian(b)
            np.testing.assert_allclose(cd, c1 / math.sqrt(d), rtol=1e-14)
            np.testing.assert_allclose(td, t1 / math.sqrt(d), rtol=1e-14, atol=1e-300)


# ---------------------------------------------------------------------------
# Scalar quantiser and bit-pack
# ---------------------------------------------------------------------------

def _read_bitpack_golden():
    rows = []
    with open(os.path.join(GOLDEN, "bitpack_examples.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            b, codes, hexes = [p.strip() for p in line.split("|")]
            rows.append((int(b), [int(v) for v in codes.split()], [int(v, 16) for v in hexes.split()]))
    return rows


def test_bitpack_golden_examples():
    for bits, codes, expect in _read_bitpack_golden():
        got = O.bitpack(np.array([codes]), bits)[0]
        assert list(got) == expect
        assert list(O.bitunpack(np.array([expect], dtype=np.uint8), bits, len(codes))[0]) == codes


@pytest.mark.parametrize("bits", [2, 3, 4])
@pytest.mark.parametrize("d", [128, 256, 512])
def test_bitpack_roundtrip_and_size(bits, d):
    figs = _read_golden_pairs("page_figures.txt")
    assert O.packed_bytes(128, 3) == figs["bytes_per_vector_d128_b3"]
    assert abs(figs["fp16_bytes_per_vector_d128"] / O.packed_bytes(128, 3) - figs["compression_vs_fp16"]) < 0.05
    g = np.random.default_rng(bits * 1000 + d)
    codes = g.integers(0, 1 << bits, size=(7, d))
    packed = O.bitpack(codes, bits)
    assert packed.shape == (7, d * bits // 8)
    np.testing.assert_array_equal(O.bitunpack(packed, bits, d), codes)
    if bits != 3:
        # LSB-first as one little-endian integer per vector
        as_int = int.from_bytes(bytes(packed[0]), "little")
        assert as_int == sum(int(c) << (bits * i) for i, c in enumerate(codes[0]))
    else:
        # 32-code groups of three words: code 32k+8r+j in nibble j of word
        # 3k+r (low 3 bits); bit r of code 32k+24+j in bit 3 of that nibble
        words = np.frombuffer(bytes(packed[0]), dtype="<u4").astype(np.int64)
        for k in range(d // 32):
            for r in range(3):
                for j in range(8):
                    nib = (words[3 * k + r] >> (4 * j)) & 15
                    assert nib & 7 == codes[0, 32 * k + 8 * r + j]
                    assert nib >> 3 == (codes[0, 32 * k + 24 + j] >> r) & 1


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_threshold_count_is_nearest_centroid(bits):
    c, t = O.make_codebook(128, bits)
    g = np.random.default_rng(bits)
    y = g.standard_normal(20000) / math.sqrt(128) * 1.5
    codes = O.quantize_scalar(y, t)
    nearest = np.argmin(np.abs(y[:, None] - c[None, :]), axis=1)
    np.testing.assert_array_equal(codes, nearest)
    # exact ties resolve to the lower code
    np.testing.assert_array_equal(O.quantize_scalar(t, t), np.arange(len(t)))


# ---------------------------------------------------------------------------
# End-to-end quantise / dequantise
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("variant", O.VARIANTS)
@pytest.mark.parametrize("bits", [2, 3, 4])
def test_requantising_a_reconstruction_returns_its_codes(variant, bits):
    d = 128
    c, _ = O.make_codebook(d, bits)
    params = O.make_params(d, variant, seed=21)
    g = np.random.default_rng(22)
    # codes drawn with the Gaussian cell probabilities so ||c[codes]|| ~ 1
    probs = np.array([integrate.quad(_phi, a, b)[0] for a, b in
                      zip([-np.inf] + list(O.lloyd_max_gaussian(bits)[1]),
                          list(O.lloyd_max_gaussian(bits)[1]) + [np.inf])])
    codes = g.choice(len(c), size=(1, 2000, d), p=probs / probs.sum())
    norms_c = np.linalg.norm(c[codes], axis=-1)
    # Keep rows with ||c[codes]|| in [0.9, 1.1]: scaling any centroid of a
    # b <= 4 Gaussian Lloyd-Max codebook by a factor in [1/1.1, 1/0.9] keeps it
    # inside its own cell (Max 1960 table), so re-quantisation is exact.
    keep = (norms_c[0] > 0.9) & (norms_c[0] < 1.1)
    codes = codes[:, keep][:, :300]
    norms_c = norms_c[:, keep][:, :300]
    assert codes.shape[1] == 300
    s = g.lognormal(2.0, 0.5, (1, 300))
    x = O.rotate_inverse(c[codes], params[0], variant) * s[..., None]
    packed, norms = O.quantize(x, params, bits, variant)
    np.testing.assert_array_equal(O.bitunpack(packed, bits, d), codes)
    np.testing.assert_allclose(norms.astype(np.float64), s * norms_c, rtol=2 ** -11)
    # and dequantise gives s16 * R^T c exactly (closed form)
    xr = O.dequantize(packed, norms, params, bits, variant, d)
    expect = O.rotate_inverse(c[codes], params[0], variant) * norms.astype(np.float64)[..., None]
    np.testing.assert_allclose(xr, expect, atol=1e-13)


@pytest.mark.parametrize("variant", O.VARIANTS)
@pytest.mark.parametrize("bits", [2, 3, 4])
def test_stage1_mse_close_to_lloyd_distortion(bits, variant):
    """Unit vectors: per-coordinate rotated marginal ~ N(0, 1/d), so the mean
    squared reconstruction error is close to the Gaussian Lloyd-Max
    distortion (Max 1960), slightly below it (the exact marginal, a scaled
    Beta, has lighter tails).  An isotropic input stays isotropic under any
    rotation, so every variant lands in the same band."""
    table = _read_max_table()
    d = 128
    params = O.make_params(d, variant, seed=1)
    x = synth.unit_vectors(2000, d, seed=3, dtype=np.float64)
    packed, norms = O.quantize(x, params, bits, variant)
    xr = O.dequantize(packed, norms, params, bits, variant, d)
    mse = np.mean(np.sum((x - xr) ** 2, axis=-1))
    ref = table[(bits, "mse")][0]
    assert 0.85 * ref < mse < 1.05 * ref


def test_rotation_ablation_ordering_on_outlier_channels():
    """RotaryQuant §4.6 Table 8 on keys and values with outlier channels
    (Student-t, 4 channels x10, RoPE on K): the WHT-composed rotations
    (v3 Full, Fast, the 2-D case) spread the outliers and stay near the
    Lloyd-Max distortion; v2 (block SO(4), no WHT) keeps each outlier inside
    its block and v1 (one quaternion) also leaves a quarter of the
    coordinates unrotated, so their relative errors order v1 > v2 >> v3."""
    table = _read_max_table()
    d, bits = 128, 3
    k, v = synth.student_t_kv(1, 1000, d, seed=5, dtype=np.float64)
    for x in (k[0, 0], v[0, 0]):
        rel = {}
        for var in O.VARIANTS:
            p = O.make_params(d, var, seed=1)
            packed, norms = O.quantize(x[None], p, bits, var)
            xr = O.dequantize(packed, norms, p, bits, var, d)[0]
            rel[var] = np.mean(np.sum((x - xr) ** 2, -1) / np.sum(x * x, -1))
        ref = table[(bits, "mse")][0]
        for var in (O.FULL, O.FAST, O.PLANAR):
            assert 0.85 * ref < rel[var] < 1.05 * ref
        assert rel[O.SO3] > 1.1 * rel[O.BLOCK_SO4] > 4 * max(rel[O.FULL], rel[O.FAST], rel[O.PLANAR])


def test_zero_vector_and_tie_codes():
    d = 128
    params = O.make_params(d, O.FULL, seed=1)
    x = np.zeros((1, 2, d))
    x[0, 1, 0] = 3.0
    packed, norms = O.quantize(x, params, 3, O.FULL)
    np.testing.assert_array_equal(O.bitunpack(packed, 3, d)[0, 0], 3)  # L/2 - 1
    assert norms[0, 0] == 0 and norms[0, 1] == 3.0
    np.testing.assert_array_equal(O.dequantize(packed, norms, params, 3, O.FULL, d)[0, 0], 0.0)


def test_norm_is_float16_of_unrounded_norm():
    x = np.zeros((1, 1, 128))
    x[0, 0, :2] = [3.0, 4.0000001]
    _, norms = O.quantize(x, O.make_params(128, O.FULL, 1), 3, O.FULL)
    assert norms.dtype == np.float16 and norms[0, 0] == np.float16(math.hypot(3.0, 4.0000001))


# ---------------------------------------------------------------------------
# Decode attention
# ---------------------------------------------------------------------------

def _random_cache(g, b, hkv, tmax, d, bits):
    pk = g.integers(0, 256, size=(b, hkv, tmax, d * bits // 8), dtype=np.uint8)
    pv = g.integers(0, 256, size=(b, hkv, tmax, d * bits // 8), dtype=np.uint8)
    nk = g.lognormal(1.0, 0.3, (b, hkv, tmax)).astype(np.float16)
    nv = g.lognormal(1.0, 0.3, (b, hkv, tmax)).astype(np.float16)
    return pk, pv, nk, nv


@pytest.mark.parametrize("variant", [O.FULL, O.FAST])
@pytest.mark.parametrize("d,bits", [(128, 3), (256, 2), (128, 4)])
def test_compressed_space_attention_equals_ordinary(variant, d, bits):
    """RotaryQuant Appendix A: attention in the rotated domain with one
    inverse rotation equals ordinary attention over the reconstruction."""
    g = np.random.default_rng(31)
    bsz, hq, hkv, tmax = 3, 4, 2, 37
    pk, pv, nk, nv = _random_cache(g, bsz, hkv, tmax, d, bits)
    q = g.standard_normal((bsz, hq, d))
    lens = np.array([37, 0, 50])            # full, empty, clamped to Tmax
    pkk = O.make_params(d, variant, 1, hkv)
    pvv = O.make_params(d, variant, 2, hkv)
    a = O.decode_attention(q, pk, pv, nk, nv, lens, pkk, pvv, bits, variant, 1 / math.sqrt(d))
    b = O.decode_attention_reconstructed(q, pk, pv, nk, nv, lens, pkk, pvv, bits, variant, 1 / math.sqrt(d))
    np.testing.assert_allclose(a, b, atol=1e-12)
    assert np.all(a[1] == 0)
    # dense brute force: explicit R matrices and an explicit softmax
    c, _ = O.make_codebook(d, bits)
    for bb in (0, 2):
        for qh in range(hq):
            kvh = qh // (hq // hkv)
            rk = O.rotate(np.eye(d), pkk[kvh], variant).T
            rv = O.rotate(np.eye(d), pvv[kvh], variant).T
            kk = (c[O.bitunpack(pk[bb, kvh], bits, d)] * nk[bb, kvh, :, None].astype(float)) @ rk
            vv = (c[O.bitunpack(pv[bb, kvh], bits, d)] * nv[bb, kvh, :, None].astype(float)) @ rv
            z = kk @ q[bb, qh] / math.sqrt(d)
            w = np.exp(z - z.max())
            np.testing.assert_allclose(a[bb, qh], (w / w.sum()) @ vv, atol=1e-12)


def test_attention_special_cases():
    g = np.random.default_rng(41)
    d, bits, hkv, hq = 128, 3, 1, 2
    pk, pv, nk, nv = _random_cache(g, 1, hkv, 9, d, bits)
    pkk = O.make_params(d, O.FULL, 1, hkv)
    pvv = O.make_params(d, O.FULL, 2, hkv)
    vhat = O.dequantize(pv[0], nv[0], pvv, bits, O.FULL, d)[0]
    q = g.standard_normal((1, hq, d))
    # T = 1: the output is the one reconstructed value
    o1 = O.decode_attention(q, pk, pv, nk, nv, [1], pkk, pvv, bits, O.FULL, 0.1)
    np.testing.assert_allclose(o1[0, 0], vhat[0], atol=1e-12)
    # q = 0: uniform weights, the mean of the reconstructed values
    o0 = O.decode_attention(np.zeros_like(q), pk, pv, nk, nv, [9], pkk, pvv, bits, O.FULL, 0.1)
    np.testing.assert_allclose(o0[0, 1], vhat.mean(axis=0), atol=1e-12)
    # tokens past seq_len do not matter, even as NaN norms
    nk2, nv2 = nk.copy(), nv.copy()
    nk2[0, 0, 5:] = np.nan
    nv2[0, 0, 5:] = np.nan
    a = O.decode_attention(q, pk, pv, nk, nv, [5], pkk, pvv, bits, O.FULL, 0.1)
    b = O.decode_attention(q, pk, pv, nk2, nv2, [5], pkk, pvv, bits, O.FULL, 0.1)
    np.testing.assert_array_equal(a, b)
    # RotaryQuant §5 "Inverse rotation is mandatory": the rotated-domain
    # aggregate is not the output
    c, _ = O.make_codebook(d, bits)
    vt = c[O.bitunpack(pv[0, 0, :5], bits, d)] * nv[0, 0, :5, None].astype(float)
    kt = c[O.bitunpack(pk[0, 0, :5], bits, d)] * nk[0, 0, :5, None].astype(float)
    z = kt @ O.rotate(q[0, 0], pkk[0], O.FULL) * 0.1
    w = np.exp(z - z.max())
    o_rot = (w / w.sum()) @ vt
    np.testing.assert_allclose(O.rotate_inverse(o_rot, pvv[0], O.FULL), a[0, 0], atol=1e-12)
    assert np.max(np.abs(o_rot - a[0, 0])) > 0.1


@pytest.mark.parametrize("variant", [O.FULL, O.FAST])
def test_decode_append_token_by_token_equals_bulk_compression(variant):
    """RotaryQuant Figure 1 / Appendix D: compressing each decode-step entry
    on arrival gives the cache that compressing the whole sequence at once
    gives, at the positions the lengths name; rows already at Tmax stay as
    they were and are reported; negative lengths count as empty."""
    g = np.random.default_rng(61)
    bsz, hkv, tmax, d, bits, steps = 3, 2, 12, 128, 3, 5
    start = np.array([0, 4, -3])
    pk0, pv0, nk0, nv0 = _random_cache(g, bsz, hkv, tmax, d, bits)
    kseq = g.standard_normal((bsz, hkv, steps, d))
    vseq = g.standard_normal((bsz, hkv, steps, d)) * 3.0
    prk = O.make_params(d, variant, 1, hkv)
    prv = O.make_params(d, variant, 2, hkv)
    cache = (pk0, pv0, nk0, nv0, start)
    for s in range(steps):
        *cache, full = O.decode_append(kseq[:, :, s], vseq[:, :, s], *cache, prk, prv, bits, variant)
        assert full == []
    pk, pv, nk, nv, lens = cache
    np.testing.assert_array_equal(lens, np.maximum(start, 0) + steps)
    for b in range(bsz):
        t0 = max(start[b], 0)
        bk, bnk = O.quantize(kseq[b], prk, bits, variant)
        bv, bnv = O.quantize(vseq[b], prv, bits, variant)
        np.testing.assert_array_equal(pk[b, :, t0:t0 + steps], bk)
        np.testing.assert_array_equal(pv[b, :, t0:t0 + steps], bv)
        np.testing.assert_array_equal(nk[b, :, t0:t0 + steps].view(np.uint16), bnk.view(np.uint16))
        np.testing.assert_array_equal(nv[b, :, t0:t0 + steps].view(np.uint16), bnv.view(np.uint16))
        # everything outside the written span is untouched
        keep = np.ones(tmax, bool)
        keep[t0:t0 + steps] = False
        np.testing.assert_array_equal(pk[b][:, keep], pk0[b][:, keep])
        np.testing.assert_array_equal(nv[b][:, keep].view(np.uint16), nv0[b][:, keep].view(np.uint16))
    # a full row takes no token
    out = O.decode_append(kseq[:, :, 0], vseq[:, :, 0], pk, pv, nk, nv, np.array([tmax, 3, tmax + 5]),
                          prk, prv, bits, variant)
    assert out[5] == [0, 2]
    np.testing.assert_array_equal(out[4], [tmax, 4, tmax + 5])
    np.testing.assert_array_equal(out[0][0], pk[0])
    np.testing.assert_array_equal(out[0][2], pk[2])


def test_prefill_attention_is_causal_attention_over_the_reconstruction():
    """Chunked prefill: a dense causal softmax over the dequantised K/V with
    an explicit mask matrix (query t at position L - Tq + t sees tokens
    0..position) equals the oracle's compressed-space prefill; the last
    query equals a full-length decode; splitting the chunk in two changes
    nothing; queries before the cache start give zero rows."""
    g = np.random.default_rng(91)
    d, bits, hkv, hq, tmax, tq = 128, 3, 2, 4, 40, 9
    pk, pv, nk, nv = _random_cache(g, 2, hkv, tmax, d, bits)
    prk = O.make_params(d, O.FULL, 1, hkv)
    prv = O.make_params(d, O.FULL, 2, hkv)
    q = g.standard_normal((2, tq, hq, d))
    lens = np.array([33, 5])            # row 1: positions -4..4 (four empty queries)
    scale = 1 / math.sqrt(d)
    got = O.prefill_attention(q, pk, pv, nk, nv, lens, prk, prv, bits, O.FULL, scale)
    for b in range(2):
        for kvh in range(hkv):
            kh = O.dequantize(pk[b, kvh:kvh + 1], nk[b, kvh:kvh + 1], prk[kvh:kvh + 1], bits, O.FULL, d)[0]
            vh = O.dequantize(pv[b, kvh:kvh + 1], nv[b, kvh:kvh + 1], prv[kvh:kvh + 1], bits, O.FULL, d)[0]
            pos = lens[b] - tq + np.arange(tq)
            mask = np.arange(tmax)[None, :] <= pos[:, None]
            for hh in range(hq // hkv):
                qh = kvh * (hq // hkv) + hh
                z = q[b, :, qh] @ kh.T * scale
                z = np.where(mask, z, -np.inf)
                zmax = np.max(z, axis=1, keepdims=True)
                w = np.where(mask, np.exp(z - np.where(np.isfinite(zmax), zmax, 0)), 0.0)
                den = w.sum(axis=1, keepdims=True)
                o = np.where(den > 0, (w @ vh) / np.where(den > 0, den, 1), 0.0)
                np.testing.assert_allclose(got[b, :, qh], o, atol=1e-12)
    np.testing.assert_array_equal(got[1, :4], 0.0)
    last = O.decode_attention(q[:, -1], pk, pv, nk, nv, lens, prk, prv, bits, O.FULL, scale)
    np.testing.assert_allclose(got[:, -1], last, atol=1e-13)
    a = O.prefill_attention(q[:, :4], pk, pv, nk, nv, lens - 5, prk, prv, bits, O.FULL, scale)
    b2 = O.prefill_attention(q[:, 4:], pk, pv, nk, nv, lens, prk, prv, bits, O.FULL, scale)
    np.testing.assert_allclose(np.concatenate([a, b2], axis=1), got, atol=1e-13)


def test_split_k_combine_is_partition_independent():
    g = np.random.default_rng(51)
    t, d = 300, 16
    z = g.standard_normal(t) * 4
    v = g.standard_normal((t, d))
    w = np.exp(z - z.max())
    ref = (w / w.sum()) @ v
    for bounds in ([0, t], [0, 1, t], [0, 100, 100, 200, t], list(range(0, t + 1, 7)) + [t],
                   [0, 299, t]):
        bounds = sorted(set(bounds)) if bounds[-1] == t else bounds
        np.testing.assert_allclose(O.combine_partials(O.split_partials(z, v, bounds)), ref, atol=1e-13)
    # an empty split contributes nothing
    parts = O.split_partials(z, v, [0, 150, 150, t])
    assert parts[1][1] == 0.0
    np.testing.assert_allclose(O.combine_partials(parts), ref, atol=1e-13)


# ---------------------------------------------------------------------------
# Other figures on the pages
# ---------------------------------------------------------------------------

def test_page_figures_arithmetic():
    f = _read_golden_pairs("page_figures.txt")
    assert round(f["dense_rotation_fmas_d128"] / f["rotation_fmas_d128"], 1) == f["rotation_fma_reduction"]
    assert f["dense_rotation_params_d128"] / f["stored_params_per_head_d128"] == f["param_reduction"]
    assert f["dense_rotation_params_d128"] == 128 * 128
    # RotaryQuant eq. (5): packed QK + V accumulation is 2*T*d multiply-adds;
    # the inverse rotation (WHT + one product per block) runs once.
    inv = O.wht_op_count(128) + O.so4_fma_count(128, O.FAST)
    share = inv / (2 * 2048 * 128 + inv)
    assert share < f["inverse_rotation_share_bound_t2048_d128"]
    assert abs(share - 0.00268) < 1e-4
    transient = 2 * 28 * 8 * 128 * 2048 * 2
    assert transient == 234_881_024
    assert abs(transient / 1e6 - f["transient_prefill_bytes_mb"]) / f["transient_prefill_bytes_mb"] < 0.03
