"""Parity of the CUDA chunked-prefill attention (isoq_prefill_attention)
with the float64 oracle's causal prefill, on caches the oracle compressed."""

import math

import numpy as np
import pytest

import oracle as O
import synth
from isoq_testlib import check_attention

torch = pytest.importorskip("torch")
import compressed_space_attention_b200 as isoq  # noqa: E402

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _t(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def _cache(b, hkv, tmax, d, seed, variant=O.FULL):
    k, v = synth.student_t_kv(hkv, tmax, d, seed=seed, batch=b)
    prk = O.make_params(d, variant, seed=seed + 1, n_heads=hkv)
    prv = O.make_params(d, variant, seed=seed + 2, n_heads=hkv)
    pk, nk = O.quantize(k.reshape(b * hkv, tmax, d).astype(np.float64), np.tile(prk, (b, 1, 1)), 3, variant)
    pv, nv = O.quantize(v.reshape(b * hkv, tmax, d).astype(np.float64), np.tile(prv, (b, 1, 1)), 3, variant)
    pb = d * 3 // 8
    return (pk.reshape(b, hkv, tmax, pb), pv.reshape(b, hkv, tmax, pb), nk.reshape(b, hkv, tmax),
            nv.reshape(b, hkv, tmax), prk, prv)


def _run(q, cache, lens, variant=O.FULL):
    pk, pv, nk, nv, prk, prv = cache
    out = isoq.isoq_prefill_attention(_t(q), _t(pk), _t(pv), _t(nk), _t(nv), _t(np.asarray(lens, np.int32)),
                                      _t(prk), _t(prv), bits=3, variant=variant)
    torch.cuda.synchronize()
    assert isoq.isoq_check_device_error() == 0
    return out.cpu().numpy()


@pytest.mark.parametrize("d,hq,hkv", [(128, 32, 4), (256, 16, 8), (128, 4, 4), (128, 16, 4)])
def test_prefill_matches_oracle(d, hq, hkv):
    """Chunks of 70 queries at the end of caches of 300 and 45 tokens (the
    second starts 25 positions before the cache: zero rows), several query
    tiles with a ragged last one, several K/V tiles with a partial last one."""
    b, tmax, tq = 2, 320, 70
    cache = _cache(b, hkv, tmax, d, seed=d + hq)
    q = synth.queries(b * tq, hq, d, seed=hq).reshape(b, tq, hq, d)
    lens = [300, 45]
    ref = O.prefill_attention(q, *cache[:4], lens, cache[4], cache[5], 3, O.FULL, 1 / math.sqrt(d))
    got = _run(q, cache, lens)
    assert np.all(got[1, :25] == 0)
    check_attention(got, ref, np.float16)


def test_prefill_fast_and_planar_variants():
    d, hq, hkv, b, tmax, tq = 128, 8, 2, 1, 200, 64
    for variant in (O.FAST, O.PLANAR):
        cache = _cache(b, hkv, tmax, d, seed=30 + variant, variant=variant)
        q = synth.queries(tq, hq, d, seed=31).reshape(b, tq, hq, d)
        lens = [190]
        ref = O.prefill_attention(q, *cache[:4], lens, cache[4], cache[5], 3, variant, 1 / math.sqrt(d))
        check_attention(_run(q, cache, lens, variant), ref, np.float16)


def test_prefill_long_context_sampled():
    """A chunk of 256 queries at the end of a 16,384-token context (d=256,
    GQA 16/8): sampled query rows against the oracle, and the last query
    against the decode kernel's output for the full length."""
    b, hq, hkv, tmax, d, tq = 1, 16, 8, 16384, 256, 256
    torch.cuda.empty_cache()
    k, v = synth.student_t_kv_torch(b, hkv, tmax, d, seed=41, device=DEV)
    prk = O.make_params(d, O.FULL, seed=42, n_heads=hkv)
    prv = O.make_params(d, O.FULL, seed=43, n_heads=hkv)
    pk, nk = isoq.isoq_quantize(k.view(-1, tmax, d), _t(prk), 3, isoq.ISOQ_FULL)
    pv, nv = isoq.isoq_quantize(v.view(-1, tmax, d), _t(prv), 3, isoq.ISOQ_FULL)
    pk, pv = pk.view(b, hkv, tmax, -1), pv.view(b, hkv, tmax, -1)
    nk, nv = nk.view(b, hkv, tmax), nv.view(b, hkv, tmax)
    del k, v
    q = synth.queries(tq, hq, d, seed=44).reshape(b, tq, hq, d)
    lens = np.array([tmax], dtype=np.int32)
    got = isoq.isoq_prefill_attention(_t(q), pk, pv, nk, nv, _t(lens), _t(prk), _t(prv), bits=3,
                                      variant=isoq.ISOQ_FULL).cpu().numpy()
    pk_h, pv_h, nk_h, nv_h = (x.cpu().numpy() for x in (pk, pv, nk, nv))
    for t in (0, 97, 255):
        pos = tmax - tq + t
        ref = O.decode_attention(q[:, t], pk_h, pv_h, nk_h, nv_h, [pos + 1], prk, prv, 3, O.FULL, 1 / math.sqrt(d))
        check_attention(got[:, t], ref, np.float16)
    # the last query sees the whole cache: the decode kernel on the same
    # cache meets the same bar against the same oracle row
    dec = isoq.isoq_decode_attention(_t(q[:, -1]), pk, pv, nk, nv, _t(lens), _t(prk), _t(prv), bits=3,
                                     variant=isoq.ISOQ_FULL).cpu().numpy()
    check_attention(dec, ref, np.float16)


def test_prefill_host_validation():
    lib = isoq.lib()
    call = lambda **kw: lib.isoq_prefill_attention(*[kw.get(k, v) for k, v in (
        ("q", 256), ("dtype", isoq.ISOQ_F16), ("pk", 256), ("pv", 256), ("nk", 256), ("nv", 256),
        ("sl", 256), ("B", 1), ("Tq", 4), ("Hq", 8), ("Hkv", 2), ("Tmax", 64), ("d", 128), ("bits", 3),
        ("variant", 0), ("prk", 256), ("prv", 256), ("scale", 0.1), ("out", 256), ("stream", None))])
    assert call(d=512) == isoq.ISOQ_ERR_UNSUPPORTED
    assert call(bits=4) == isoq.ISOQ_ERR_UNSUPPORTED
    assert call(dtype=isoq.ISOQ_F32) == isoq.ISOQ_ERR_UNSUPPORTED
    assert call(Hq=6, Hkv=2) == isoq.ISOQ_ERR_UNSUPPORTED        # G = 3
    assert call(Hq=7) == isoq.ISOQ_ERR_INVALID_ARG
    assert call(variant=isoq.ISOQ_SO3) == isoq.ISOQ_ERR_UNSUPPORTED
    assert call(q=None) == isoq.ISOQ_ERR_INVALID_ARG
    assert call(pk=256 + 8) == isoq.ISOQ_ERR_UNSUPPORTED
    assert call(scale=float("nan")) == isoq.ISOQ_ERR_INVALID_ARG
    assert call(Tq=0) == isoq.ISOQ_OK
