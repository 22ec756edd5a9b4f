"""Parity of the CUDA decode-step append (and the append-then-attend step)
with the float64 oracle.  The caches start as the oracle's own compression
or seeded random bytes; the new tokens' codes and norms written by the GPU
are compared with ``oracle.decode_append``, and the attention of a step is
compared with ``oracle.decode_attention`` over the cache the GPU wrote."""

import math

import numpy as np
import pytest

import oracle as O
import synth
from isoq_testlib import check_attention, check_codes, check_norms

torch = pytest.importorskip("torch")
import compressed_space_attention_b200 as isoq  # noqa: E402

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _t(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def _random_cache(g, b, hkv, tmax, d, bits):
    pb = d * bits // 8
    pk = g.integers(0, 256, size=(b, hkv, tmax, pb), dtype=np.uint8)
    pv = g.integers(0, 256, size=(b, hkv, tmax, pb), dtype=np.uint8)
    nk = g.lognormal(2.5, 0.3, (b, hkv, tmax)).astype(np.float16)
    nv = g.lognormal(1.0, 0.3, (b, hkv, tmax)).astype(np.float16)
    return pk, pv, nk, nv


def _check_written(gpu, ref_cache, kn, vn, lens0, prk, prv, bits, variant, d):
    """Codes and norms of the positions the append wrote, against the oracle;
    every other byte of the cache unchanged."""
    gpk, gpv, gnk, gnv = gpu
    pk0, pv0, nk0, nv0 = ref_cache
    rpk, rpv, rnk, rnv, _, full = O.decode_append(kn, vn, pk0, pv0, nk0, nv0, lens0, prk, prv, bits, variant)
    mism = 0
    for b in range(kn.shape[0]):
        if b in full:
            continue
        t = max(int(lens0[b]), 0)
        for which, x, params, gp, rp, gn, rn in ((0, kn, prk, gpk, rpk, gnk, rnk), (1, vn, prv, gpv, rpv, gnv, rnv)):
            _, _, y = O.quantize(np.asarray(x[b], np.float64)[:, None, :], params, bits, variant,
                                 return_rotated=True)
            mism += check_codes(gp[b, :, t], rp[b, :, t], y[:, 0], bits, d)
            check_norms(gn[b, :, t], rn[b, :, t], np.asarray(x[b], np.float64))
            # the rest of this row, and of every other row, is as before
            gp2, rp2 = gp[b].copy(), rp[b].copy()
            gp2[:, t] = 0
            rp2[:, t] = 0
            np.testing.assert_array_equal(gp2, rp2)
    for b in full:
        np.testing.assert_array_equal(gpk[b], pk0[b])
        np.testing.assert_array_equal(gnv[b].view(np.uint16), nv0[b].view(np.uint16))
    return mism


@pytest.mark.parametrize("variant", [isoq.ISOQ_FULL, isoq.ISOQ_FAST])
@pytest.mark.parametrize("dtype", [np.float16, np.float32])
@pytest.mark.parametrize("d,bits", [(128, 3), (256, 3), (512, 3), (128, 2), (256, 4)])
def test_append_matches_oracle(variant, dtype, d, bits):
    """B=3 rows at lengths 0, 5 and -2 (counts as empty), Hkv=2, Tmax=16:
    the new K/V (Student-t with outlier channels) land at the right
    positions with the oracle's codes and norms; lengths advance by one."""
    g = np.random.default_rng(100 + d + bits)
    b, hkv, tmax = 3, 2, 16
    cache = _random_cache(g, b, hkv, tmax, d, bits)
    k, v = synth.student_t_kv(hkv, 1, d, seed=d + bits, batch=b, dtype=dtype)
    kn, vn = k[:, :, 0], v[:, :, 0]
    prk = O.make_params(d, variant, seed=1, n_heads=hkv)
    prv = O.make_params(d, variant, seed=2, n_heads=hkv)
    lens0 = np.array([0, 5, -2], dtype=np.int32)
    dev = [_t(a) for a in cache]
    lens = _t(lens0)
    isoq.isoq_decode_append(_t(kn), _t(vn), *dev, lens, _t(prk), _t(prv), bits=bits, variant=variant)
    torch.cuda.synchronize()
    assert isoq.isoq_check_device_error() == 0
    np.testing.assert_array_equal(lens.cpu().numpy(), [1, 6, 1])
    gpu = [a.cpu().numpy() for a in dev]
    mism = _check_written(gpu, cache, kn, vn, lens0, prk, prv, bits, variant, d)
    assert mism <= 2


def test_append_full_row_is_reported_and_left_unchanged():
    """A row already holding Tmax tokens takes no token: its cache and length
    stay as they were, the other rows are written, and the device error
    check reports ISOQ_ERR_INVALID_ARG once (then clears)."""
    g = np.random.default_rng(7)
    b, hkv, tmax, d, bits = 3, 4, 8, 128, 3
    cache = _random_cache(g, b, hkv, tmax, d, bits)
    k, v = synth.student_t_kv(hkv, 1, d, seed=3, batch=b)
    kn, vn = k[:, :, 0], v[:, :, 0]
    prk = O.make_params(d, isoq.ISOQ_FULL, seed=1, n_heads=hkv)
    prv = O.make_params(d, isoq.ISOQ_FULL, seed=2, n_heads=hkv)
    lens0 = np.array([tmax, 7, tmax + 3], dtype=np.int32)
    dev = [_t(a) for a in cache]
    lens = _t(lens0)
    isoq.isoq_decode_append(_t(kn), _t(vn), *dev, lens, _t(prk), _t(prv), bits=bits, variant=isoq.ISOQ_FULL)
    assert isoq.isoq_check_device_error() == isoq.ISOQ_ERR_INVALID_ARG
    assert isoq.isoq_check_device_error() == 0
    np.testing.assert_array_equal(lens.cpu().numpy(), [tmax, 8, tmax + 3])
    gpu = [a.cpu().numpy() for a in dev]
    _check_written(gpu, cache, kn, vn, lens0, prk, prv, bits, isoq.ISOQ_FULL, d)


@pytest.mark.parametrize("d,hq,hkv", [(128, 32, 4), (256, 16, 8), (128, 8, 8)])
def test_decode_steps_match_oracle(d, hq, hkv):
    """Four decode steps of isoq_decode_step on a ragged batch (lengths
    uniform in [300, 700], Tmax 704): after each step the new entries match
    the oracle's compression, and the attention output matches the oracle's
    decode over the cache the GPU holds (T + 1 tokens)."""
    b, tmax, bits, steps = 4, 704, 3, 4
    k, v = synth.student_t_kv(hkv, tmax, d, seed=11, batch=b)
    prk = O.make_params(d, O.FULL, seed=1, n_heads=hkv)
    prv = O.make_params(d, O.FULL, seed=2, n_heads=hkv)
    pk, nk = O.quantize(k.reshape(b * hkv, tmax, d).astype(np.float64), np.tile(prk, (b, 1, 1)), bits, O.FULL)
    pv, nv = O.quantize(v.reshape(b * hkv, tmax, d).astype(np.float64), np.tile(prv, (b, 1, 1)), bits, O.FULL)
    pb = d * bits // 8
    cache = [pk.reshape(b, hkv, tmax, pb), pv.reshape(b, hkv, tmax, pb), nk.reshape(b, hkv, tmax),
             nv.reshape(b, hkv, tmax)]
    lens_np = synth.ragged_lengths(b, 300, 700, seed=12)
    dev = [_t(a) for a in cache]
    lens = _t(lens_np)
    ws = torch.empty(isoq.isoq_decode_workspace_size(b, hq, hkv, tmax, d), dtype=torch.uint8, device=DEV)
    out = torch.empty((b, hq, d), dtype=torch.float16, device=DEV)
    tpk, tpv = _t(prk), _t(prv)
    for s in range(steps):
        kn, vn = synth.student_t_kv(hkv, 1, d, seed=20 + s, batch=b)
        kn, vn = kn[:, :, 0], vn[:, :, 0]
        q = synth.queries(b, hq, d, seed=30 + s)
        before = [a.cpu().numpy() for a in dev]
        got = isoq.isoq_decode_step(_t(q), _t(kn), _t(vn), *dev, lens, tpk, tpv, bits=bits,
                                    variant=isoq.ISOQ_FULL, out=out, workspace=ws)
        torch.cuda.synchronize()
        assert isoq.isoq_check_device_error() == 0
        lens_np = lens_np + 1
        np.testing.assert_array_equal(lens.cpu().numpy(), lens_np)
        gpu = [a.cpu().numpy() for a in dev]
        _check_written(gpu, before, kn, vn, lens_np - 1, prk, prv, bits, O.FULL, d)
        ref = O.decode_attention(q, *gpu, lens_np, prk, prv, bits, O.FULL, 1 / math.sqrt(d))
        check_attention(got.cpu().numpy(), ref, np.float16)


def test_step_rejects_bad_attention_arguments_before_writing():
    """isoq_decode_step validates the attention half first: a call with Hq
    not a multiple of Hkv returns an error and leaves cache and lengths as
    they were."""
    g = np.random.default_rng(5)
    b, hkv, tmax, d, bits = 2, 2, 16, 128, 3
    cache = _random_cache(g, b, hkv, tmax, d, bits)
    dev = [_t(a) for a in cache]
    lens = _t(np.array([3, 4], dtype=np.int32))
    prk = _t(O.make_params(d, O.FULL, seed=1, n_heads=hkv))
    kn = torch.randn((b, hkv, d), device=DEV, dtype=torch.float16)
    q = torch.randn((b, 3, d), device=DEV, dtype=torch.float16)           # 3 % 2 != 0
    ws = torch.empty(1 << 20, dtype=torch.uint8, device=DEV)
    out = torch.empty((b, 3, d), dtype=torch.float16, device=DEV)
    st = isoq.lib().isoq_decode_step(
        q.data_ptr(), kn.data_ptr(), kn.data_ptr(), isoq.ISOQ_F16, *(a.data_ptr() for a in dev),
        lens.data_ptr(), b, 3, hkv, tmax, d, bits, isoq.ISOQ_FULL, prk.data_ptr(), prk.data_ptr(),
        0.1, out.data_ptr(), ws.data_ptr(), ws.numel(), None)
    assert st == isoq.ISOQ_ERR_INVALID_ARG
    torch.cuda.synchronize()
    np.testing.assert_array_equal(lens.cpu().numpy(), [3, 4])
    for a, ref in zip(dev, cache):
        np.testing.assert_array_equal(a.cpu().numpy().view(np.uint8), ref.view(np.uint8))


def test_append_full_size_sampled():
    """The long-context cache shape (batch 32 x Tmax 65,536, d=256, Hkv 8,
    3-bit Full) with every row at Tmax - 1 but one empty row and one full
    row: the append writes position Tmax - 1 (the highest address of each
    row), sampled rows are compared with the oracle, and the full row is
    reported."""
    b, hkv, tmax, d, bits = 32, 8, 65536, 256, 3
    pb = d * bits // 8
    torch.cuda.empty_cache()
    pk = torch.zeros((b, hkv, tmax, pb), dtype=torch.uint8, device=DEV)
    pv = torch.zeros_like(pk)
    nk = torch.zeros((b, hkv, tmax), dtype=torch.float16, device=DEV)
    nv = torch.zeros_like(nk)
    lens0 = np.full(b, tmax - 1, dtype=np.int32)
    lens0[5], lens0[17] = 0, tmax
    lens = _t(lens0)
    k, v = synth.student_t_kv(hkv, 1, d, seed=41, batch=b)
    kn, vn = k[:, :, 0], v[:, :, 0]
    prk = O.make_params(d, O.FULL, seed=1, n_heads=hkv)
    prv = O.make_params(d, O.FULL, seed=2, n_heads=hkv)
    isoq.isoq_decode_append(_t(kn), _t(vn), pk, pv, nk, nv, lens, _t(prk), _t(prv), bits=bits,
                            variant=isoq.ISOQ_FULL)
    assert isoq.isoq_check_device_error() == isoq.ISOQ_ERR_INVALID_ARG
    got_lens = lens.cpu().numpy()
    exp = np.minimum(np.maximum(lens0, 0) + 1, tmax)
    np.testing.assert_array_equal(got_lens, exp)
    for bb in (0, 5, 17, 31):
        t = max(int(lens0[bb]), 0)
        if lens0[bb] >= tmax:
            assert int(pk[bb].count_nonzero()) == 0 and int(nk[bb].count_nonzero()) == 0
            continue
        rpk, rnk = O.quantize(np.asarray(kn[bb], np.float64)[:, None, :], prk, bits, O.FULL)
        rpv, rnv = O.quantize(np.asarray(vn[bb], np.float64)[:, None, :], prv, bits, O.FULL)
        _, _, yk = O.quantize(np.asarray(kn[bb], np.float64)[:, None, :], prk, bits, O.FULL, return_rotated=True)
        _, _, yv = O.quantize(np.asarray(vn[bb], np.float64)[:, None, :], prv, bits, O.FULL, return_rotated=True)
        check_codes(pk[bb, :, t].cpu().numpy(), rpk[:, 0], yk[:, 0], bits, d)
        check_codes(pv[bb, :, t].cpu().numpy(), rpv[:, 0], yv[:, 0], bits, d)
        check_norms(nk[bb, :, t].cpu().numpy(), rnk[:, 0], np.asarray(kn[bb], np.float64))
        check_norms(nv[bb, :, t].cpu().numpy(), rnv[:, 0], np.asarray(vn[bb], np.float64))
        # only that one position of the row was written
        assert int(pk[bb].count_nonzero()) == int(pk[bb, :, t].count_nonzero())
    del pk, pv, nk, nv
    torch.cuda.empty_cache()
