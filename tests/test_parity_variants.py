"""Parity of the rotation variants (IsoQuant's 2-D special case and the
RotaryQuant §4.6 ablation designs v1 and v2) between the CUDA compressor and
the float64 oracle, and the ablation's error ordering measured on the GPU."""

import math

import numpy as np
import pytest

import oracle as O
import synth
from isoq_testlib import DEQ_REL, check_attention, check_codes, check_norms, f16_half_ulp

torch = pytest.importorskip("torch")
import compressed_space_attention_b200 as isoq  # noqa: E402

pytestmark = pytest.mark.gpu

DEV = "cuda"
NEW_VARIANTS = [O.PLANAR, O.BLOCK_SO4, O.SO3]


def _t(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def _gpu_quantize(x, params, bits, variant):
    codes, norms = isoq.isoq_quantize(_t(x), _t(params), bits, variant)
    torch.cuda.synchronize()
    assert isoq.isoq_check_device_error() == 0
    return codes.cpu().numpy(), norms.cpu().numpy()


@pytest.mark.parametrize("variant", NEW_VARIANTS)
@pytest.mark.parametrize("dtype", [np.float16, np.float32])
@pytest.mark.parametrize("d,bits", [(128, 3), (256, 2), (512, 4), (128, 4), (256, 3)])
def test_variant_quantize_parity(variant, dtype, d, bits):
    """4,099 normalised N(0, I_d) vectors (several tiles and a ragged tail)
    per setting: codes bit-exact outside the boundary band, norms exact."""
    seed = 1000 + 10 * variant + d // 128 + bits
    x = synth.unit_vectors(4099, d, seed=seed, dtype=dtype)
    params = O.make_params(d, variant, seed=seed)
    gc, gn = _gpu_quantize(x, params, bits, variant)
    oc, on, y = O.quantize(x.astype(np.float64), params, bits, variant, return_rotated=True)
    assert check_codes(gc, oc, y, bits, d) <= 20
    check_norms(gn, on, x.astype(np.float64))


@pytest.mark.parametrize("variant", NEW_VARIANTS)
@pytest.mark.parametrize("out_dtype", [np.float32, np.float16])
@pytest.mark.parametrize("d,bits", [(128, 3), (512, 2)])
def test_variant_dequantize_parity(variant, out_dtype, d, bits):
    """Dequantise the oracle's own codes and norms of outlier-channel values
    (two heads) on the GPU."""
    params = O.make_params(d, variant, seed=31, n_heads=2)
    x = synth.student_t_kv(2, 777, d, seed=32, dtype=np.float32)[1][0]
    oc, on = O.quantize(x.astype(np.float64), params, bits, variant)
    ref = O.dequantize(oc, on, params, bits, variant, d)
    tdt = torch.float16 if out_dtype == np.float16 else torch.float32
    got = isoq.isoq_dequantize(_t(oc), _t(on), _t(params), d, bits, variant, out_dtype=tdt)
    torch.cuda.synchronize()
    got = got.cpu().numpy().astype(np.float64)
    tol = DEQ_REL * on.astype(np.float64)[..., None]
    if out_dtype == np.float16:
        tol = tol + f16_half_ulp(ref)
    assert np.all(np.abs(got - ref) <= tol), float(np.max(np.abs(got - ref) - tol))


def test_ablation_error_ordering_on_gpu():
    """RotaryQuant §4.6 Table 8 measured through the CUDA round trip on the
    prefill generator's keys (Student-t, 4 outlier channels x10, RoPE): the
    relative reconstruction error of every variant equals the oracle's, and
    orders v1 (SO3) > v2 (BLOCK_SO4) >> v3 (Full, Fast, 2-D)."""
    d, bits, n = 128, 3, 8192
    k, _ = synth.student_t_kv(1, n, d, seed=41)
    x = k[0]                                                 # [1][n][d] float16
    x64 = x.astype(np.float64)
    rel = {}
    for var in O.VARIANTS:
        params = O.make_params(d, var, seed=42)
        gc, gn = _gpu_quantize(x, params, bits, var)
        rec = isoq.isoq_dequantize(_t(gc), _t(gn), _t(params), d, bits, var, out_dtype=torch.float32)
        g = rec.cpu().numpy().astype(np.float64)
        gpu_rel = float(np.mean(np.sum((g - x64) ** 2, -1) / np.sum(x64 * x64, -1)))
        oc, on = O.quantize(x64, params, bits, var)
        o = O.dequantize(oc, on, params, bits, var, d)
        ref_rel = float(np.mean(np.sum((o - x64) ** 2, -1) / np.sum(x64 * x64, -1)))
        assert abs(gpu_rel - ref_rel) <= 2e-3 * ref_rel
        rel[var] = gpu_rel
    best = max(rel[O.FULL], rel[O.FAST], rel[O.PLANAR])
    assert rel[O.SO3] > 1.1 * rel[O.BLOCK_SO4] > 4 * best


@pytest.mark.parametrize("d,hq,hkv", [(128, 8, 2), (256, 16, 8)])
def test_planar_decode_matches_oracle(d, hq, hkv):
    """Decode attention with the 2-D special case's parameters (the decode
    applies the Full block map, which those parameters make two plane
    rotations): batch 2 x 1,000 tokens of oracle-compressed K/V."""
    b, t, bits = 2, 1000, 3
    k, v = synth.student_t_kv(hkv, t, d, seed=51, batch=b)
    prk = O.make_params(d, O.PLANAR, seed=52, n_heads=hkv)
    prv = O.make_params(d, O.PLANAR, seed=53, n_heads=hkv)
    pk, nk = O.quantize(k.reshape(b * hkv, t, d).astype(np.float64), np.tile(prk, (b, 1, 1)), bits, O.PLANAR)
    pv, nv = O.quantize(v.reshape(b * hkv, t, d).astype(np.float64), np.tile(prv, (b, 1, 1)), bits, O.PLANAR)
    pb = d * bits // 8
    pk, pv = pk.reshape(b, hkv, t, pb), pv.reshape(b, hkv, t, pb)
    nk, nv = nk.reshape(b, hkv, t), nv.reshape(b, hkv, t)
    q = synth.queries(b, hq, d, seed=54)
    lens = np.array([t, 613], dtype=np.int32)
    scale = 1 / math.sqrt(d)
    ref = O.decode_attention(q, pk, pv, nk, nv, lens, prk, prv, bits, O.PLANAR, scale)
    got = isoq.isoq_decode_attention(_t(q), _t(pk), _t(pv), _t(nk), _t(nv), _t(lens), _t(prk), _t(prv),
                                     bits=bits, variant=isoq.ISOQ_PLANAR, scale=scale)
    torch.cuda.synchronize()
    assert isoq.isoq_check_device_error() == 0
    check_attention(got.cpu().numpy(), ref, np.float16)
