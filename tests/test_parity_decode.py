"""Parity of the CUDA compressed-space decode attention with the float64
oracle.  Packed K/V fed to the GPU are always the oracle's own compression
(or seeded random bytes), so both sides score the same codes."""

import math

import numpy as np
import pytest

import oracle as O
import synth
from isoq_testlib import check_attention, check_codes

torch = pytest.importorskip("torch")
import compressed_space_attention_b200 as isoq  # noqa: E402

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _t(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def _gpu_decode(q, pk, pv, nk, nv, lens, prk, prv, bits, variant, scale, split_calls=False):
    args = [_t(q), _t(pk), _t(pv), _t(nk), _t(nv), _t(np.asarray(lens, dtype=np.int32)), _t(prk), _t(prv)]
    out = isoq.isoq_decode_attention(*args, bits=bits, variant=variant, scale=scale)
    torch.cuda.synchronize()
    assert isoq.isoq_check_device_error() == 0
    return out.cpu().numpy()


def _random_cache(seed, b, hkv, tmax, d, bits):
    g = synth.rng(seed)
    pb = d * bits // 8
    pk = g.integers(0, 256, size=(b, hkv, tmax, pb), dtype=np.uint8)
    pv = g.integers(0, 256, size=(b, hkv, tmax, pb), dtype=np.uint8)
    nk = g.lognormal(2.5, 0.3, (b, hkv, tmax)).astype(np.float16)
    nv = g.lognormal(1.0, 0.3, (b, hkv, tmax)).astype(np.float16)
    return pk, pv, nk, nv


def test_tiny_fp32_decode():
    """One head, d=128, Full, 3-bit, float32: 4,096 tokens, one N(0,1) query,
    scale 1/sqrt(128); float32 output within 1e-5."""
    k, v, q = synth.tiny_kv(seed=0)
    params = O.make_params(128, O.FULL, seed=1)
    pk, nk = O.quantize(k.astype(np.float64), params, 3, O.FULL)
    pv, nv = O.quantize(v.astype(np.float64), params, 3, O.FULL)
    pk, pv, nk, nv = pk[None], pv[None], nk[None], nv[None]
    lens = [4096]
    ref = O.decode_attention(q, pk, pv, nk, nv, lens, params, params, 3, O.FULL, 1 / math.sqrt(128))
    got = _gpu_decode(q, pk, pv, nk, nv, lens, params, params, 3, O.FULL, 1 / math.sqrt(128))
    assert got.dtype == np.float32
    check_attention(got, ref, np.float32)
    # and the same as ordinary attention over the oracle's reconstruction
    ref_b = O.decode_attention_reconstructed(q, pk, pv, nk, nv, lens, params, params, 3, O.FULL,
                                             1 / math.sqrt(128))
    check_attention(got, ref_b, np.float32)


def test_decode_batch1_context32768_gqa32_4(prefill_kv):
    """GQA 32/4, d=128, float16 queries, batch 1 x context 32,768 over the
    prefill workload's oracle-compressed K/V: every output element."""
    pk, nk = prefill_kv["oracle_k"][0][None], prefill_kv["oracle_k"][1][None]
    pv, nv = prefill_kv["oracle_v"][0][None], prefill_kv["oracle_v"][1][None]
    q = synth.queries(1, 32, 128, seed=4)
    prk, prv = prefill_kv["params_k"], prefill_kv["params_v"]
    lens = [32768]
    ref = O.decode_attention(q, pk, pv, nk, nv, lens, prk, prv, 3, O.FULL, 1 / math.sqrt(128))
    got = _gpu_decode(q, pk, pv, nk, nv, lens, prk, prv, 3, O.FULL, 1 / math.sqrt(128))
    check_attention(got, ref, np.float16)


def test_decode_batch16_ragged_lengths():
    """Batch 16 x context 8,192 with lengths uniform in [4096, 8192]."""
    b, hkv, hq, tmax, d = 16, 4, 32, 8192, 128
    k, v = synth.student_t_kv(hkv, tmax, d, seed=5, batch=b)
    prk = O.make_params(d, O.FULL, seed=1, n_heads=hkv)
    prv = O.make_params(d, O.FULL, seed=2, n_heads=hkv)
    lens = synth.ragged_lengths(b, 4096, 8192, seed=0)
    pk, nk = O.quantize(k.reshape(b * hkv, tmax, d).astype(np.float64), np.tile(prk, (b, 1, 1)), 3, O.FULL)
    pv, nv = O.quantize(v.reshape(b * hkv, tmax, d).astype(np.float64), np.tile(prv, (b, 1, 1)), 3, O.FULL)
    pk, pv = pk.reshape(b, hkv, tmax, 48), pv.reshape(b, hkv, tmax, 48)
    nk, nv = nk.reshape(b, hkv, tmax), nv.reshape(b, hkv, tmax)
    q = synth.queries(b, hq, d, seed=6)
    ref = O.decode_attention(q, pk, pv, nk, nv, lens, prk, prv, 3, O.FULL, 1 / math.sqrt(d))
    got = _gpu_decode(q, pk, pv, nk, nv, lens, prk, prv, 3, O.FULL, 1 / math.sqrt(d))
    check_attention(got, ref, np.float16)


def test_long_context_shape_small():
    """d=256, GQA 16/8, 3-bit Full, batch 2 x 2,048 tokens: every element."""
    b, hkv, hq, t, d = 2, 8, 16, 2048, 256
    k, v = synth.student_t_kv(hkv, t, d, seed=7, batch=b)
    prk = O.make_params(d, O.FULL, seed=1, n_heads=hkv)
    prv = O.make_params(d, O.FULL, seed=2, n_heads=hkv)
    pk, nk = O.quantize(k.reshape(b * hkv, t, d).astype(np.float64), np.tile(prk, (b, 1, 1)), 3, O.FULL)
    pv, nv = O.quantize(v.reshape(b * hkv, t, d).astype(np.float64), np.tile(prv, (b, 1, 1)), 3, O.FULL)
    pk, pv = pk.reshape(b, hkv, t, 96), pv.reshape(b, hkv, t, 96)
    nk, nv = nk.reshape(b, hkv, t), nv.reshape(b, hkv, t)
    q = synth.queries(b, hq, d, seed=8)
    lens = [t, t]
    ref = O.decode_attention(q, pk, pv, nk, nv, lens, prk, prv, 3, O.FULL, 1 / math.sqrt(d))
    got = _gpu_decode(q, pk, pv, nk, nv, lens, prk, prv, 3, O.FULL, 1 / math.sqrt(d))
    check_attention(got, ref, np.float16)


def test_long_context_full_size_sampled():
    """The benchmark's launch: batch 32 x 65,536 tokens, d=256, GQA 16/8.
    K/V are drawn on the device and compressed by the CUDA path; 16 sampled
    (b, kvh) rows (the four corners of the grid and 12 seeded others) are
    also compressed by the oracle (codes compared), their oracle codes are
    written into the cache, and the decode outputs of those rows' query
    heads are compared with the oracle."""
    b, hkv, hq, t, d = 32, 8, 16, 65536, 256
    torch.cuda.empty_cache()
    k, v = synth.student_t_kv_torch(b, hkv, t, d, seed=9, device=DEV)
    prk = O.make_params(d, O.FULL, seed=1, n_heads=hkv)
    prv = O.make_params(d, O.FULL, seed=2, n_heads=hkv)
    pk, nk = isoq.isoq_quantize(k.view(b * hkv, t, d), _t(np.tile(prk, (b, 1, 1))), 3, O.FULL)
    pv, nv = isoq.isoq_quantize(v.view(b * hkv, t, d), _t(np.tile(prv, (b, 1, 1))), 3, O.FULL)
    pk, pv = pk.view(b, hkv, t, 96), pv.view(b, hkv, t, 96)
    nk, nv = nk.view(b, hkv, t), nv.view(b, hkv, t)
    pick = synth.rng(90).choice(b * hkv, size=16, replace=False)
    samples = [(0, 0), (0, hkv - 1), (b - 1, 0), (b - 1, hkv - 1)]
    samples += [(int(i) // hkv, int(i) % hkv) for i in pick if (int(i) // hkv, int(i) % hkv) not in samples][:12]
    rows = {}
    for (bb, kvh) in samples:
        for name, x, codes, norms, par in (("k", k, pk, nk, prk), ("v", v, pv, nv, prv)):
            xs = x[bb, kvh].cpu().numpy().astype(np.float64)[None]
            oc, on, y = O.quantize(xs, par[kvh:kvh + 1], 3, O.FULL, return_rotated=True)
            check_codes(codes[bb, kvh].cpu().numpy()[None], oc, y, 3, d)
            codes[bb, kvh].copy_(_t(oc[0]))
            norms[bb, kvh].copy_(_t(on[0]))
            rows[(bb, kvh, name)] = (oc[0], on[0])
    del k, v
    q = synth.queries_torch(b, hq, d, seed=10, device=DEV)
    lens = torch.full((b,), t, dtype=torch.int32, device=DEV)
    out = isoq.isoq_decode_attention(q, pk, pv, nk, nv, lens, _t(prk), _t(prv), 3, O.FULL)
    torch.cuda.synchronize()
    out = out.cpu().numpy()
    qn = q.cpu().numpy()
    g = hq // hkv
    for (bb, kvh) in samples:
        ck, nk0 = rows[(bb, kvh, "k")]
        cv, nv0 = rows[(bb, kvh, "v")]
        heads = list(range(kvh * g, kvh * g + g))
        ref = O.decode_attention(qn[bb:bb + 1, heads], ck[None, None], cv[None, None],
                                 nk0[None, None], nv0[None, None], [t], prk[kvh:kvh + 1],
                                 prv[kvh:kvh + 1], 3, O.FULL, 1 / math.sqrt(d))
        check_attention(out[bb, heads], ref[0], np.float16)


@pytest.mark.parametrize("case", [
    # (dtype, d, bits, variant, B, Hq, Hkv, Tmax, lens)  -- path exercised
    (np.float16, 128, 3, O.FULL, 3, 8, 2, 136, [0, 1, 500]),       # tensor-core; empty, 1, clamp
    (np.float16, 256, 3, O.FAST, 2, 16, 2, 264, [264, 77]),        # tensor-core, Fast, G=8
    (np.float16, 128, 3, O.FULL, 2, 4, 4, 1001, [1001, 640]),      # generic: Tmax % 8 != 0, G=1
    (np.float16, 128, 2, O.FULL, 2, 8, 2, 300, [300, 33]),         # generic: 2-bit
    (np.float16, 256, 4, O.FAST, 1, 32, 2, 200, [199]),            # generic: 4-bit, G=16
    (np.float16, 512, 3, O.FULL, 1, 4, 2, 128, [128]),             # generic: d=512
    (np.float32, 256, 3, O.FULL, 2, 6, 3, 96, [96, 95]),           # float32 generic
    (np.float32, 512, 2, O.FAST, 1, 2, 1, 70, [70]),               # float32 generic
])
def test_decode_edge_cases(case):
    dt, d, bits, variant, b, hq, hkv, tmax, lens = case
    pk, pv, nk, nv = _random_cache(sum(map(ord, repr(case))) % 1000, b, hkv, tmax, d, bits)
    q = synth.queries(b, hq, d, seed=13, dtype=dt)
    prk = O.make_params(d, variant, seed=1, n_heads=hkv)
    prv = O.make_params(d, variant, seed=2, n_heads=hkv)
    # norms past each sequence's end are NaN: they must not reach the output
    for i, ln in enumerate(lens):
        nk[i, :, min(max(ln, 0), tmax):] = np.nan
        nv[i, :, min(max(ln, 0), tmax):] = np.nan
    ref = O.decode_attention(q, pk, pv, nk, nv, lens, prk, prv, bits, variant, 1 / math.sqrt(d))
    got = _gpu_decode(q, pk, pv, nk, nv, lens, prk, prv, bits, variant, 1 / math.sqrt(d))
    assert got.dtype == dt
    check_attention(got, ref, dt)
    for i, ln in enumerate(lens):
        if ln <= 0:
            assert np.all(got[i] == 0)


def test_split_and_combine_calls_equal_fused_call():
    b, hq, hkv, tmax, d = 2, 8, 2, 4096, 128
    pk, pv, nk, nv = _random_cache(3, b, hkv, tmax, d, 3)
    q = synth.queries(b, hq, d, seed=14)
    prk = _t(O.make_params(d, O.FULL, seed=1, n_heads=hkv))
    prv = _t(O.make_params(d, O.FULL, seed=2, n_heads=hkv))
    args = [_t(q), _t(pk), _t(pv), _t(nk), _t(nv), _t(np.array([4096, 3000], np.int32))]
    fused = isoq.isoq_decode_attention(*args, prk, prv, 3, O.FULL)
    ws = torch.empty(isoq.isoq_decode_workspace_size(b, hq, hkv, tmax, d), dtype=torch.uint8, device=DEV)
    isoq.isoq_decode_split(*args, prk, 3, O.FULL, ws)
    out = torch.empty_like(fused)
    isoq.isoq_decode_combine(out, args[5], b, hq, hkv, tmax, d, O.FULL, prv, ws)
    torch.cuda.synchronize()
    assert torch.equal(out, fused)


def test_scale_argument_is_used():
    b, hq, hkv, tmax, d = 1, 2, 1, 256, 128
    pk, pv, nk, nv = _random_cache(4, b, hkv, tmax, d, 3)
    q = synth.queries(b, hq, d, seed=15)
    prk = O.make_params(d, O.FULL, seed=1)
    prv = O.make_params(d, O.FULL, seed=2)
    for scale in (0.0, 0.02, 0.3):
        ref = O.decode_attention(q, pk, pv, nk, nv, [256], prk, prv, 3, O.FULL, scale)
        got = _gpu_decode(q, pk, pv, nk, nv, [256], prk, prv, 3, O.FULL, scale)
        check_attention(got, ref, np.float16)


@pytest.mark.parametrize("d,hq,hkv", [(128, 32, 4), (256, 16, 8)])
def test_attention_sink_with_small_value_norm(d, hq, hkv):
    """One dominant token (its score 12 nats above every other) whose V norm
    is 40 times below the others', as attention sinks often are, among 700
    tokens: the other tokens' small weights must still be accumulated to the
    float16 tolerance, not rounded away against the sink's scale."""
    b, t, bits = 2, 700, 3
    k, v = synth.student_t_kv(hkv, t, d, seed=71, batch=b)
    prk = O.make_params(d, O.FULL, seed=1, n_heads=hkv)
    prv = O.make_params(d, O.FULL, seed=2, n_heads=hkv)
    pk, nk = O.quantize(k.reshape(b * hkv, t, d).astype(np.float64), np.tile(prk, (b, 1, 1)), bits, O.FULL)
    pv, nv = O.quantize(v.reshape(b * hkv, t, d).astype(np.float64), np.tile(prv, (b, 1, 1)), bits, O.FULL)
    pb = d * bits // 8
    pk, pv = pk.reshape(b, hkv, t, pb), pv.reshape(b, hkv, t, pb)
    nk, nv = nk.reshape(b, hkv, t), nv.reshape(b, hkv, t)
    sink = [3, 450]
    scale = 1 / math.sqrt(d)
    q = np.empty((b, hq, d), dtype=np.float16)
    for bb in range(b):
        nv[bb, :, sink[bb]] = (nv[bb, :, sink[bb]].astype(np.float64) / 40).astype(np.float16)
        for kvh in range(hkv):
            khat = O.dequantize(pk[bb, kvh:kvh + 1], nk[bb, kvh:kvh + 1], prk[kvh:kvh + 1], bits, O.FULL, d)[0]
            k0 = khat[sink[bb]]
            others = np.delete(khat, sink[bb], axis=0) @ k0
            alpha = 12.0 / (scale * (k0 @ k0 - others.max()))
            for g in range(hq // hkv):
                q[bb, kvh * (hq // hkv) + g] = (alpha * (1.0 + 0.05 * g) * k0).astype(np.float16)
    lens = [t, t]
    ref = O.decode_attention(q, pk, pv, nk, nv, lens, prk, prv, bits, O.FULL, scale)
    got = _gpu_decode(q, pk, pv, nk, nv, lens, prk, prv, bits, O.FULL, scale)
    check_attention(got, ref, np.float16)
