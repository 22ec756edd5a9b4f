"""Parity of the CUDA compressor (isoq_quantize / isoq_dequantize) with the
float64 oracle on the same seeded inputs, through the C ABI."""

import numpy as np
import pytest

import oracle as O
import synth
from isoq_testlib import DEQ_REL, check_codes, check_norms, f16_half_ulp

torch = pytest.importorskip("torch")
import compressed_space_attention_b200 as isoq  # noqa: E402

pytestmark = pytest.mark.gpu

DEV = "cuda"
NP2TORCH = {np.float16: torch.float16, np.float32: torch.float32}


def _gpu_quantize(x, params, bits, variant):
    xt = torch.from_numpy(np.ascontiguousarray(x)).to(DEV)
    pt = torch.from_numpy(params).to(DEV)
    codes, norms = isoq.isoq_quantize(xt, pt, bits, variant)
    torch.cuda.synchronize()
    assert isoq.isoq_check_device_error() == 0
    return codes.cpu().numpy(), norms.cpu().numpy()


def _compare_quantize(x, params, bits, variant):
    gc, gn = _gpu_quantize(x, params, bits, variant)
    x64 = np.asarray(x, dtype=np.float64)
    oc, on, y = O.quantize(x64, params, bits, variant, return_rotated=True)
    d = x.shape[-1]
    n_code = check_codes(gc, oc, y, bits, d)
    n_norm = check_norms(gn, on, x64)
    return n_code, n_norm, (gc, gn, oc, on)


def test_tiny_fp32_keys_and_values():
    """One head, d=128, IsoQuant-Full, 3-bit, float32; 4,096 K and 4,096 V."""
    k, v, _ = synth.tiny_kv(seed=0)
    params = O.make_params(128, O.FULL, seed=1)
    for x in (k, v):
        n_code, n_norm, _ = _compare_quantize(x, params, 3, O.FULL)
        assert n_code <= 10 and n_norm <= 2


@pytest.mark.parametrize("variant", [O.FULL, O.FAST])
@pytest.mark.parametrize("dtype", [np.float16, np.float32])
@pytest.mark.parametrize("bits", [2, 3, 4])
@pytest.mark.parametrize("d", [128, 256, 512])
def test_stage1_sweep_settings(d, bits, dtype, variant):
    """Every (d, bits, dtype, variant) setting of the stage-1 sweep on 4,099
    normalised N(0, I_d) vectors (a ragged tail past several tiles)."""
    idx = [128, 256, 512].index(d) * 12 + [2, 3, 4].index(bits) * 4 + \
        [np.float16, np.float32].index(dtype) * 2 + variant
    x = synth.unit_vectors(4099, d, seed=idx, dtype=dtype)
    params = O.make_params(d, variant, seed=100 + idx)
    n_code, n_norm, _ = _compare_quantize(x, params, bits, variant)
    assert n_code <= 20


def test_stage1_full_size_sampled():
    """N = 2^20 unit vectors, d=128, 3-bit, float16, Full (the benchmark's
    quantize launch); 4,096 sampled vectors checked against the oracle."""
    n, d = 1 << 20, 128
    x = synth.unit_vectors(n, d, seed=7, dtype=np.float16)
    params = O.make_params(d, O.FULL, seed=1)
    gc, gn = _gpu_quantize(x, params, 3, O.FULL)
    sample = np.sort(synth.rng(8).choice(n, size=4096, replace=False))
    xs = x[:, sample]
    oc, on, y = O.quantize(xs.astype(np.float64), params, 3, O.FULL, return_rotated=True)
    assert check_codes(gc[:, sample], oc, y, 3, d) <= 10
    check_norms(gn[:, sample], on, xs.astype(np.float64))


def test_prefill_compression_full(prefill_kv):
    """4 KV heads x 32,768 tokens x 128, float16 Student-t with outliers and
    RoPE on K, 3-bit Full with separate K and V rotations: every vector."""
    for name in ("k", "v"):
        x = prefill_kv[name]
        params = prefill_kv["params_" + name]
        oc, on, y = prefill_kv["oracle_" + name]
        gc, gn = _gpu_quantize(x, params, 3, O.FULL)
        n_code = check_codes(gc, oc, y, 3, 128)
        n_norm = check_norms(gn, on, x.astype(np.float64))
        assert n_code <= 50 and n_norm <= 20


def test_edge_cases_sizes_zeros_magnitudes():
    d = 128
    params = O.make_params(d, O.FULL, seed=5, n_heads=2)
    for n in (1, 2, 63, 64, 65, 129):
        x = synth.unit_vectors(n, d, seed=n, dtype=np.float16, n_heads=2).astype(np.float32)
        x[0, 0] = 0.0                      # a zero vector
        x[1, -1] *= 3.0e4                  # large magnitude
        if n > 2:
            x[0, 1] *= 1.0e-3              # small magnitude
        x = x.astype(np.float16)
        n_code, _, (gc, gn, oc, on) = _compare_quantize(x, params, 3, O.FULL)
        assert n_code <= 2
        np.testing.assert_array_equal(O.bitunpack(gc[0, :1], 3, d), 3)
        assert gn[0, 0] == 0


@pytest.mark.parametrize("d,dtype", [(128, np.float16), (128, np.float32), (256, np.float16)])
@pytest.mark.parametrize("bits", [2, 3, 4])
@pytest.mark.parametrize("variant", [O.FULL, O.FAST])
def test_zero_vectors_get_the_middle_negative_code(d, dtype, bits, variant):
    """A zero vector has y = 0, so code = #{k : 0 > t_k} = L/2 - 1 at every
    coordinate (RotaryQuant Algorithm 1 with the threshold rule; the oracle's
    reading for a zero norm), and a zero norm: on every kernel path, next to
    ordinary vectors in the same tile."""
    params = O.make_params(d, variant, seed=3)
    x = synth.unit_vectors(200, d, seed=d + bits, dtype=dtype)
    for j in (0, 37, 128, 199):
        x[0, j] = 0
    gc, gn = _gpu_quantize(x, params, bits, variant)
    codes = O.bitunpack(gc, bits, d)
    for j in (0, 37, 128, 199):
        np.testing.assert_array_equal(codes[0, j], (1 << bits) // 2 - 1)
        assert gn[0, j] == 0
    oc, on, y = O.quantize(x.astype(np.float64), params, bits, variant, return_rotated=True)
    assert check_codes(gc, oc, y, bits, d) <= 2


def test_empty_is_noop():
    x = torch.zeros((2, 0, 128), dtype=torch.float16, device=DEV)
    p = torch.from_numpy(O.make_params(128, O.FULL, 1, 2)).to(DEV)
    codes, norms = isoq.isoq_quantize(x, p, 3, O.FULL)
    assert codes.shape == (2, 0, 48) and norms.shape == (2, 0)


@pytest.mark.parametrize("d,dtype", [(128, np.float16), (512, np.float16), (512, np.float32)])
def test_token_major_input_into_larger_cache(d, dtype):
    """x in token-major [T][Hkv][d] layout written into a [Hkv][Tmax] cache at
    an offset: strided input and out_head_stride > n_vec (at d = 512 the rows
    are staged through a 4-D tensor map of 128-byte chunks)."""
    hkv, t, tmax, off = 3, 200, 512, 40
    xt = synth.unit_vectors(t * hkv, d, seed=9, dtype=dtype).reshape(t, hkv, d)
    params = O.make_params(d, O.FULL, seed=6, n_heads=hkv)
    x_dev = torch.from_numpy(xt).to(DEV)
    view = x_dev.permute(1, 0, 2)                     # [Hkv][T][d], strides (d, Hkv*d, 1)
    cache_codes = torch.full((hkv, tmax, d * 3 // 8), 0xAB, dtype=torch.uint8, device=DEV)
    cache_norms = torch.full((hkv, tmax), 7.0, dtype=torch.float16, device=DEV)
    isoq.isoq_quantize(view, torch.from_numpy(params).to(DEV), 3, O.FULL,
                       codes=cache_codes[:, off:], norms=cache_norms[:, off:], out_head_stride=tmax)
    torch.cuda.synchronize()
    gc = cache_codes.cpu().numpy()
    gn = cache_norms.cpu().numpy()
    x64 = np.transpose(xt, (1, 0, 2)).astype(np.float64)
    oc, on, y = O.quantize(x64, params, 3, O.FULL, return_rotated=True)
    assert check_codes(gc[:, off:off + t], oc, y, 3, d) <= 2
    check_norms(gn[:, off:off + t], on, x64)
    assert np.all(gc[:, :off] == 0xAB) and np.all(gc[:, off + t:] == 0xAB)
    assert np.all(gn[:, :off] == 7.0) and np.all(gn[:, off + t:] == 7.0)


@pytest.mark.parametrize("out_dtype", [np.float32, np.float16])
@pytest.mark.parametrize("d,bits,variant", [(128, 3, O.FULL), (256, 2, O.FAST), (512, 4, O.FULL),
                                            (128, 4, O.FAST), (256, 3, O.FULL)])
def test_dequantize_parity(d, bits, variant, out_dtype):
    """Dequantise the oracle's own codes and norms on the GPU."""
    n = 1000
    params = O.make_params(d, variant, seed=11, n_heads=2)
    x = synth.student_t_kv(2, n, d, seed=12, dtype=np.float32)[1][0]
    oc, on = O.quantize(x.astype(np.float64), params, bits, variant)
    ref = O.dequantize(oc, on, params, bits, variant, d)
    got = isoq.isoq_dequantize(torch.from_numpy(oc).to(DEV), torch.from_numpy(on).to(DEV),
                               torch.from_numpy(params).to(DEV), d, bits, variant,
                               out_dtype=NP2TORCH[out_dtype])
    torch.cuda.synchronize()
    got = got.cpu().numpy().astype(np.float64)
    s = on.astype(np.float64)[..., None]
    tol = DEQ_REL * s
    if out_dtype == np.float16:
        tol = tol + f16_half_ulp(ref)
    assert np.all(np.abs(got - ref) <= tol), float(np.max(np.abs(got - ref) - tol))


@pytest.mark.parametrize("bits", [2, 3])
@pytest.mark.parametrize("variant", [O.FULL, O.FAST])
def test_dequantize_tensor_core_strided_heads(variant, bits):
    """The tensor-core dequantizer (d = 128, 2 and 3 bits, float16 out) on five heads
    of 20,000 vectors whose codes sit in a longer per-head buffer, written into
    a strided window of a larger output: the values match the oracle, the
    rows and columns around the window keep their sentinel, and CTAs whose
    tiles span two heads rebuild the rotation between them."""
    d, H, n, pad_v, pad_d = 128, 5, 20000, 24, 8
    params = O.make_params(d, variant, seed=41, n_heads=H)
    x = synth.unit_vectors(H * n, d, seed=42, dtype=np.float32).reshape(H, n, d)
    oc, on = O.quantize(x.astype(np.float64), params, bits, variant)
    ref = O.dequantize(oc, on, params, bits, variant, d)
    pb = oc.shape[-1]
    codes_big = torch.zeros((H, n + 20, pb), dtype=torch.uint8, device=DEV)
    norms_big = torch.zeros((H, n + 20), dtype=torch.float16, device=DEV)
    codes_big[:, :n] = torch.from_numpy(oc).to(DEV)
    norms_big[:, :n] = torch.from_numpy(on).to(DEV)
    sentinel = 3.25
    out_big = torch.full((H, n + 2 * pad_v, d + pad_d), sentinel, dtype=torch.float16, device=DEV)
    out = out_big[:, pad_v:pad_v + n, :d]
    isoq.isoq_dequantize(codes_big[:, :n], norms_big[:, :n], torch.from_numpy(params).to(DEV), d, bits, variant,
                         out=out, in_head_stride=n + 20)
    torch.cuda.synchronize()
    assert isoq.isoq_check_device_error() == 0
    big = out_big.cpu().numpy()
    got = big[:, pad_v:pad_v + n, :d].astype(np.float64)
    tol = DEQ_REL * on.astype(np.float64)[..., None] + f16_half_ulp(ref)
    assert np.all(np.abs(got - ref) <= tol), float(np.max(np.abs(got - ref) - tol))
    assert np.all(big[:, :pad_v] == sentinel) and np.all(big[:, pad_v + n:] == sentinel)
    assert np.all(big[:, :, d:] == sentinel)


def test_stage1_round_trip_mse_matches_oracle():
    """GPU quantize then GPU dequantize of unit vectors: the reconstruction
    MSE equals the oracle's (same codes up to boundary flips)."""
    d, n = 128, 20000
    x = synth.unit_vectors(n, d, seed=21, dtype=np.float32)
    params = O.make_params(d, O.FULL, seed=1)
    for bits in (2, 3, 4):
        gc, gn = _gpu_quantize(x, params, bits, O.FULL)
        rec = isoq.isoq_dequantize(torch.from_numpy(gc).to(DEV), torch.from_numpy(gn).to(DEV),
                                   torch.from_numpy(params).to(DEV), d, bits, O.FULL)
        gpu_mse = float(np.mean(np.sum((rec.cpu().numpy() - x) ** 2, axis=-1)))
        oc, on = O.quantize(x.astype(np.float64), params, bits, O.FULL)
        ref_mse = float(np.mean(np.sum((O.dequantize(oc, on, params, bits, O.FULL, d) - x) ** 2, axis=-1)))
        assert abs(gpu_mse - ref_mse) <= 1e-3 * ref_mse


def test_no_device_error_pending():
    assert isoq.isoq_check_device_error() == 0
