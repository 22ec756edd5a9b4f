"""Pins of the RotorQuant comparator's oracle (``oracle.rotorquant``) against
facts it does not compute the same way: the Clifford algebra's defining
relations, closed forms of 3-D rotations, the cost figure printed on the
IsoQuant page, and IsoQuant's own reconstruction error on the same inputs."""

import math
import os

import numpy as np
import pytest

import oracle as O
from oracle import rotorquant as R
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _figures():
    rows = {}
    with open(os.path.join(GOLDEN, "page_figures.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            parts = [p.strip() for p in line.split("|")]
            rows[parts[0]] = float(parts[1])
    return rows


def _basis(i):
    e = np.zeros(8)
    e[i] = 1.0
    return e


def test_clifford_relations():
    """Cl(3,0): e_i e_i = 1, e_i e_j = -e_j e_i, (e_i e_j)^2 = -1,
    e1 e2 e3 squares to -1 and commutes with everything; the product is
    associative."""
    gp = R.geometric_product
    e1, e2, e3 = _basis(1), _basis(2), _basis(3)
    one = _basis(0)
    for e in (e1, e2, e3):
        np.testing.assert_array_equal(gp(e, e), one)
    for a, b in ((e1, e2), (e1, e3), (e2, e3)):
        np.testing.assert_array_equal(gp(a, b), -gp(b, a))
        np.testing.assert_array_equal(gp(gp(a, b), gp(a, b)), -one)
    np.testing.assert_array_equal(gp(e1, e2), _basis(4))
    np.testing.assert_array_equal(gp(e1, e3), _basis(5))
    np.testing.assert_array_equal(gp(e2, e3), _basis(6))
    i3 = gp(gp(e1, e2), e3)
    np.testing.assert_array_equal(i3, _basis(7))
    np.testing.assert_array_equal(gp(i3, i3), -one)
    g = np.random.default_rng(1)
    a, b, c = g.standard_normal((3, 8))
    np.testing.assert_allclose(gp(i3, a), gp(a, i3), atol=1e-14)
    np.testing.assert_allclose(gp(gp(a, b), c), gp(a, gp(b, c)), atol=1e-12)
    # reverse is an anti-automorphism: rev(ab) = rev(b) rev(a)
    np.testing.assert_allclose(R.reverse(gp(a, b)), gp(R.reverse(b), R.reverse(a)), atol=1e-12)


def test_sandwich_is_a_rotation_with_closed_form_angle_and_axis():
    """For a unit rotor R = s + p12 e12 + p13 e13 + p23 e23, v -> R v rev(R)
    is a proper rotation (orthogonal, det 1) by angle phi with
    cos(phi/2) = |s| (trace 4 s^2 - 1) about the axis dual to the bivector,
    (p23, -p13, p12); the counted evaluation equals the dense product and
    leaves no scalar, bivector or trivector part."""
    g = np.random.default_rng(2)
    r = g.standard_normal((30, 4))
    r /= np.linalg.norm(r, axis=1, keepdims=True)
    for rr in r:
        m = np.stack([R.sandwich(np.eye(3)[j], rr) for j in range(3)], axis=1)
        np.testing.assert_allclose(m.T @ m, np.eye(3), atol=1e-14)
        assert abs(np.linalg.det(m) - 1.0) < 1e-13
        assert abs(np.trace(m) - (4 * rr[0] ** 2 - 1)) < 1e-13
        axis = np.array([rr[3], -rr[2], rr[1]])
        np.testing.assert_allclose(m @ axis, axis, atol=1e-14)
        v = g.standard_normal(3)
        rm = R.rotor_multivector(rr)
        dense = R.geometric_product(R.geometric_product(rm, R.embed_vector(v)), R.reverse(rm))
        np.testing.assert_allclose(dense[[0, 4, 5, 6, 7]], 0.0, atol=1e-14)
        np.testing.assert_allclose(R.sandwich(v, rr), dense[1:4], atol=1e-14)
        np.testing.assert_allclose(R.sandwich_inverse(R.sandwich(v, rr), rr), v, atol=1e-14)


def test_rotation_cost_matches_the_page():
    """IsoQuant's abstract: about 2,408 FMAs for RotorQuant's forward rotation
    at d = 128 = 43 groups x (32 + 24)."""
    figs = _figures()
    assert R.n_groups(128) == 43
    assert R.rotation_fma_count(128) == figs["rotorquant_fmas_d128"]
    assert R.rotation_fma_count(256) == 86 * 56
    # against IsoQuant-Full's 1,024
    assert R.rotation_fma_count(128) / O.so4_fma_count(128, O.FULL) > 2.3


def test_rotors_layout_and_draws():
    rot = R.make_rotors(128, seed=5, n_heads=2)
    assert rot.shape == (2, 43, 4) and rot.dtype == np.float32
    np.testing.assert_allclose(np.linalg.norm(rot, axis=-1), 1.0, atol=1e-6)
    gs = O.gaussian_stream(O.SplitMix64(5))
    v = np.array([next(gs) for _ in range(4)])
    np.testing.assert_array_equal(rot[0, 0], (v / np.linalg.norm(v)).astype(np.float32))
    assert not np.array_equal(rot[0], rot[1])


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_bitstream_round_trip_and_size(bits):
    g = np.random.default_rng(3)
    for d in (128, 256, 512):
        n = 3 * R.n_groups(d)
        codes = g.integers(0, 1 << bits, size=(4, n))
        packed = R.bitpack(codes, bits)
        assert packed.shape[-1] == R.packed_bytes(d, bits) == 4 * math.ceil(n * bits / 32)
        np.testing.assert_array_equal(R.bitunpack(packed, bits, n), codes)
    # code i at bits [b i, b i + b): codes 1, 2, 3 at 3 bits -> 0b011_010_001
    p = R.bitpack(np.array([[1, 2, 3]]), 3)
    assert int(p[0, 0]) | (int(p[0, 1]) << 8) == 0b011010001


def test_padding_and_reconstruction():
    """The padded coordinate of the last group is rotated (and stored) like
    the others, and the reconstruction returns the d real coordinates:
    s16 * R^T c exactly, and x itself to within the quantiser's error."""
    d, bits = 128, 4
    rot = R.make_rotors(d, seed=7)
    x = synth.unit_vectors(50, d, seed=8, dtype=np.float64) * 3.0
    packed, norms, y = R.quantize(x, rot, bits, return_rotated=True)
    assert y.shape == (1, 50, 129)
    assert np.all(np.abs(y[0, :, 128]) > 0) or np.mean(np.abs(y[0, :, 128])) > 1e-3
    c, _ = O.make_codebook(d, bits)
    codes = R.bitunpack(packed, bits, 129)
    expect = R.rotate_inverse(c[codes], rot[0], d) * norms.astype(np.float64)[..., None]
    np.testing.assert_allclose(R.dequantize(packed, norms, rot, bits, d), expect, atol=1e-13)
    rel = np.mean(np.sum((R.dequantize(packed, norms, rot, bits, d) - x) ** 2, -1) / np.sum(x * x, -1))
    assert rel < 0.02


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_mse_comparable_to_isoquant(bits):
    """IsoQuant's abstract: comparable reconstruction MSE on normalised
    vectors; both sit at the Lloyd-Max distortion of N(0, 1/d)."""
    d = 128
    x = synth.unit_vectors(2000, d, seed=3, dtype=np.float64)
    rot = R.make_rotors(d, seed=1)
    pk, nk = R.quantize(x, rot, bits)
    rq = np.mean(np.sum((x - R.dequantize(pk, nk, rot, bits, d)) ** 2, -1))
    p = O.make_params(d, O.FULL, seed=1)
    pi, ni = O.quantize(x, p, bits, O.FULL)
    iq = np.mean(np.sum((x - O.dequantize(pi, ni, p, bits, O.FULL, d)) ** 2, -1))
    assert abs(rq - iq) < 0.03 * iq
