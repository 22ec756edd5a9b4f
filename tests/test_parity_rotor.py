"""Parity of the CUDA RotorQuant comparator with its float64 oracle
(``oracle.rotorquant``) through the C ABI, on the stage-1 sweep's inputs."""

import numpy as np
import pytest

import oracle as O
from oracle import rotorquant as R
import synth
from isoq_testlib import CODE_BAND, DEQ_REL, check_norms, f16_half_ulp

torch = pytest.importorskip("torch")
import compressed_space_attention_b200 as isoq  # noqa: E402

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _t(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def _check_rotor_codes(gpu_packed, oracle_packed, oracle_y, bits, d):
    """Codes bit-exact except coordinates within CODE_BAND of a threshold,
    where the two sides may pick adjacent codes."""
    n = 3 * R.n_groups(d)
    _, thresholds = O.make_codebook(d, bits)
    gc = R.bitunpack(gpu_packed, bits, n)
    oc = R.bitunpack(oracle_packed, bits, n)
    mism = gc != oc
    k = int(mism.sum())
    if k:
        y = np.asarray(oracle_y)[mism]
        dist = np.min(np.abs(y[:, None] - np.asarray(thresholds)[None, :]), axis=1)
        assert np.all(dist < CODE_BAND), f"{k} mismatches, worst boundary distance {dist.max():.3g}"
        assert np.all(np.abs(gc[mism] - oc[mism]) == 1)
    # the bits past the 3G codes (padding of the last word) are zero
    bits_all = np.unpackbits(np.asarray(gpu_packed, dtype=np.uint8), axis=-1, bitorder="little")
    assert not bits_all[..., n * bits:].any()
    return k


def test_host_sizes_and_params():
    assert isoq.isoq_rotor_groups(128) == 43 and isoq.isoq_rotor_groups(512) == 171
    assert isoq.isoq_rotor_packed_bytes(128, 3) == R.packed_bytes(128, 3) == 52
    assert isoq.isoq_rotor_packed_bytes(128, 5) == 0
    got = isoq.isoq_rotor_make_params(256, seed=9, n_heads=2)
    ref = R.make_rotors(256, seed=9, n_heads=2)
    diff = np.abs(got.view(np.int32).astype(np.int64) - ref.view(np.int32).astype(np.int64))
    assert got.shape == ref.shape and diff.max() <= 1


@pytest.mark.parametrize("dtype", [np.float16, np.float32])
@pytest.mark.parametrize("bits", [2, 3, 4])
@pytest.mark.parametrize("d", [128, 256, 512])
def test_rotor_quantize_parity(d, bits, dtype):
    """4,099 normalised N(0, I_d) vectors per setting (a ragged tail, an odd
    count for the two-vector warps at d = 128)."""
    seed = 500 + d + 10 * bits + (dtype == np.float32)
    x = synth.unit_vectors(4099, d, seed=seed, dtype=dtype)
    rot = R.make_rotors(d, seed=seed)
    gc, gn = isoq.isoq_rotor_quantize(_t(x), _t(rot), bits)
    torch.cuda.synchronize()
    oc, on, y = R.quantize(x.astype(np.float64), rot, bits, return_rotated=True)
    assert _check_rotor_codes(gc.cpu().numpy(), oc, y, bits, d) <= 20
    check_norms(gn.cpu().numpy(), on, x.astype(np.float64))


@pytest.mark.parametrize("out_dtype", [np.float32, np.float16])
@pytest.mark.parametrize("d,bits", [(128, 3), (256, 2), (512, 4)])
def test_rotor_dequantize_parity(d, bits, out_dtype):
    """Dequantise the oracle's own codes of outlier-channel values (two
    heads) on the GPU: within 1e-6 of each vector's norm."""
    rot = R.make_rotors(d, seed=61, n_heads=2)
    x = synth.student_t_kv(2, 555, d, seed=62, dtype=np.float32)[1][0]
    oc, on = R.quantize(x.astype(np.float64), rot, bits)
    ref = R.dequantize(oc, on, rot, bits, d)
    tdt = torch.float16 if out_dtype == np.float16 else torch.float32
    got = isoq.isoq_rotor_dequantize(_t(oc), _t(on), _t(rot), d, bits, out_dtype=tdt)
    torch.cuda.synchronize()
    got = got.cpu().numpy().astype(np.float64)
    tol = DEQ_REL * on.astype(np.float64)[..., None]
    if out_dtype == np.float16:
        tol = tol + f16_half_ulp(ref)
    assert np.all(np.abs(got - ref) <= tol), float(np.max(np.abs(got - ref) - tol))


def test_rotor_round_trip_mse_matches_oracle_and_isoquant():
    """GPU round trip of 20,000 unit vectors at d = 128: the reconstruction
    error equals the oracle's and is comparable to IsoQuant's (the IsoQuant
    page's 'comparable reconstruction MSE')."""
    d, n = 128, 20000
    x = synth.unit_vectors(n, d, seed=71, dtype=np.float32)
    rot = R.make_rotors(d, seed=72)
    p = O.make_params(d, O.FULL, seed=72)
    for bits in (2, 3, 4):
        gc, gn = isoq.isoq_rotor_quantize(_t(x), _t(rot), bits)
        rec = isoq.isoq_rotor_dequantize(gc, gn, _t(rot), d, bits).cpu().numpy()
        gpu = float(np.mean(np.sum((rec - x) ** 2, -1)))
        oc, on = R.quantize(x.astype(np.float64), rot, bits)
        ref = float(np.mean(np.sum((R.dequantize(oc, on, rot, bits, d) - x) ** 2, -1)))
        assert abs(gpu - ref) <= 1e-3 * ref
        ic, inorm = isoq.isoq_quantize(_t(x), _t(p), bits, isoq.ISOQ_FULL)
        irec = isoq.isoq_dequantize(ic, inorm, _t(p), d, bits, isoq.ISOQ_FULL).cpu().numpy()
        iso = float(np.mean(np.sum((irec - x) ** 2, -1)))
        assert abs(gpu - iso) < 0.03 * iso


def test_rotor_multi_head_strided_and_empty():
    """Two heads read from a token-major buffer [T][H][d] (strided rows), and
    an empty call that writes nothing."""
    d, bits, t, h = 256, 3, 1001, 2
    g = np.random.default_rng(81)
    xt = g.standard_normal((t, h, d)).astype(np.float16)
    rot = R.make_rotors(d, seed=82, n_heads=h)
    xdev = _t(xt).permute(1, 0, 2)                     # [H][T][d] view, row stride h*d
    gc, gn = isoq.isoq_rotor_quantize(xdev, _t(rot), bits)
    torch.cuda.synchronize()
    oc, on, y = R.quantize(np.transpose(xt, (1, 0, 2)).astype(np.float64), rot, bits, return_rotated=True)
    assert _check_rotor_codes(gc.cpu().numpy(), oc, y, bits, d) <= 10
    empty = torch.empty((1, 0, d), dtype=torch.float16, device=DEV)
    c0, n0 = isoq.isoq_rotor_quantize(empty, _t(rot[:1]), bits)
    assert c0.numel() == 0 and n0.numel() == 0
