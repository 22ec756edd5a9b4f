"""The C-ABI library on the host: it loads, exports every entry point the
header declares, and its host-only functions (parameter generator, codebook,
split policy, argument validation) behave as specified.  No device work."""

import numpy as np
import pytest

import oracle as O
from isoq_testlib import header_functions

import compressed_space_attention_b200 as isoq
from compressed_space_attention_b200 import binding


def test_library_exports_every_header_function():
    lib = isoq.lib()
    declared = header_functions()
    assert len(declared) >= 15
    for name in declared:
        assert hasattr(lib, name), f"{name} declared in isoq.h but not exported"
    bound = {n for n, _, _ in binding.SIGNATURES}
    assert set(declared) == bound, "binding and header disagree"
    assert isoq.isoq_abi_version() == 1


def test_sizes():
    assert isoq.isoq_params_size(128) == 256
    assert isoq.isoq_params_size(256) == 512
    assert isoq.isoq_params_size(100) < 0
    assert isoq.isoq_packed_bytes(128, 3) == 48
    assert isoq.isoq_packed_bytes(256, 3) == 96
    assert isoq.isoq_packed_bytes(512, 4) == 256
    assert isoq.isoq_packed_bytes(128, 5) == 0


@pytest.mark.parametrize("variant", [isoq.ISOQ_FULL, isoq.ISOQ_FAST, isoq.ISOQ_PLANAR,
                                     isoq.ISOQ_BLOCK_SO4, isoq.ISOQ_SO3])
@pytest.mark.parametrize("d", [128, 256, 512])
def test_make_params_matches_oracle(variant, d):
    got = isoq.isoq_make_params(d, variant, seed=1234, n_heads=3)
    ref = O.make_params(d, variant, seed=1234, n_heads=3)
    assert got.shape == ref.shape
    # Same published generator on both sides; allow one float32 ulp for a
    # last-bit difference in the host libm.
    diff = np.abs(got.view(np.int32).astype(np.int64) - ref.view(np.int32).astype(np.int64))
    assert diff.max() <= 1
    assert (diff == 0).mean() > 0.99


@pytest.mark.parametrize("bits", [2, 3, 4])
@pytest.mark.parametrize("d", [128, 256, 512])
def test_make_codebook_matches_oracle(bits, d):
    c, t = isoq.isoq_make_codebook(d, bits)
    rc, rt = O.make_codebook(d, bits)
    np.testing.assert_allclose(c, rc, rtol=0, atol=1e-14 / np.sqrt(d))
    np.testing.assert_allclose(t, rt, rtol=0, atol=1e-14 / np.sqrt(d))
    assert t[len(t) // 2] == 0.0
    np.testing.assert_array_equal(c, -c[::-1])


def test_split_policy_and_workspace():
    for (B, hkv, tmax, d) in [(1, 4, 32768, 128), (16, 4, 8192, 128), (32, 8, 65536, 256),
                              (1, 1, 4096, 128), (3, 2, 1, 512), (2, 2, 1001, 128)]:
        n = isoq.isoq_decode_num_splits(B, hkv, tmax, d)
        assert n >= 1
        hq = 2 * hkv
        ws = isoq.isoq_decode_workspace_size(B, hq, hkv, tmax, d)
        # partial states, then the prepared queries of the int8 path (include/isoq.h)
        r256 = lambda x: (x + 255) // 256 * 256
        assert ws == r256(B * hq * n * (d + 2) * 4) + r256(B * hkv * (24 * d + 32))
    assert isoq.isoq_decode_workspace_size(1, 3, 2, 100, 128) == 0  # Hq % Hkv != 0


def _wave_model_chunk(B, hkv, tmax):
    """The split policy restated: the chunk in {4096, ..., 512} minimising
    the busiest SM's phases of up to 4 CTAs, (k + 0.7)(min(c, Tmax) + 160)
    each, ties to the larger chunk."""
    best, best_cost = None, None
    for c in (4096, 3072, 2048, 1536, 1024, 768, 512):
        n_ctas = B * hkv * -(-tmax // c)
        m, cost = -(-n_ctas // 148), 0.0
        while m > 0:
            k = min(m, 4)
            cost += k + 0.7
            m -= k
        cost *= min(c, tmax) + 160
        if best_cost is None or cost < best_cost - 1e-9:
            best, best_cost = c, cost
    return best


def test_split_policy_matches_its_model():
    rng = np.random.default_rng(5)
    for _ in range(300):
        B, hkv = int(rng.integers(1, 65)), int(rng.choice([1, 2, 4, 8, 16]))
        tmax = int(rng.integers(1, 300000))
        n = isoq.isoq_decode_num_splits(B, hkv, tmax, 128)
        assert n == -(-tmax // _wave_model_chunk(B, hkv, tmax)), (B, hkv, tmax, n)


def test_split_policy_wave_model():
    """The chunk is one of 512 .. 4096 tokens; on measured decode shapes it is
    the one the timed chunk sweep found fastest or within 7 % of it (batch 32
    x 8 KV heads: 1K context 512 tokens, 4K 1024, 8K 2048, 32K and 64K 4096;
    64K context at batch 4 x 8 KV heads: 2048)."""
    expect = {(32, 8, 1024): 2, (32, 8, 4096): 4, (32, 8, 8192): 4,
              (32, 8, 32768): 8, (32, 8, 65536): 16, (4, 8, 65536): 32}
    for (B, hkv, tmax), n in expect.items():
        assert isoq.isoq_decode_num_splits(B, hkv, tmax, 256) == n, (B, hkv, tmax)
    for B, hkv, tmax in [(1, 1, 100), (7, 3, 5000), (64, 8, 131072), (2, 16, 300000)]:
        n = isoq.isoq_decode_num_splits(B, hkv, tmax, 128)
        assert -(-tmax // 4096) <= n <= max(1, -(-tmax // 512)), (B, hkv, tmax, n)


def _call_quantize(**kw):
    args = dict(x=1, dtype=isoq.ISOQ_F16, n_heads=1, n_vec=10, d=128, bits=3,
                variant=isoq.ISOQ_FULL, hs=1280, vs=128, params=16, codes=16, norms=16,
                ohs=10, stream=None)
    args.update(kw)
    return isoq.lib().isoq_quantize(args["x"], args["dtype"], args["n_heads"], args["n_vec"],
                                    args["d"], args["bits"], args["variant"], args["hs"],
                                    args["vs"], args["params"], args["codes"], args["norms"],
                                    args["ohs"], args["stream"])


def test_quantize_validation_happens_on_host():
    # Every case fails validation before any CUDA call, so no GPU is needed.
    assert _call_quantize(d=100) == isoq.ISOQ_ERR_UNSUPPORTED
    assert _call_quantize(bits=5) == isoq.ISOQ_ERR_UNSUPPORTED
    assert _call_quantize(variant=7) == isoq.ISOQ_ERR_UNSUPPORTED
    assert _call_quantize(variant=5) == isoq.ISOQ_ERR_UNSUPPORTED
    assert _call_quantize(variant=-1) == isoq.ISOQ_ERR_UNSUPPORTED
    assert _call_quantize(dtype=9) == isoq.ISOQ_ERR_UNSUPPORTED
    assert _call_quantize(n_vec=-1) == isoq.ISOQ_ERR_INVALID_ARG
    assert _call_quantize(x=None, n_vec=10) == isoq.ISOQ_ERR_INVALID_ARG
    assert _call_quantize(vs=64) == isoq.ISOQ_ERR_INVALID_ARG
    assert _call_quantize(ohs=5) == isoq.ISOQ_ERR_INVALID_ARG
    assert _call_quantize(x=0x1002) == isoq.ISOQ_ERR_UNSUPPORTED      # misaligned
    assert _call_quantize(vs=132) == isoq.ISOQ_ERR_UNSUPPORTED        # 264-byte rows
    assert _call_quantize(n_vec=0) == isoq.ISOQ_OK                    # empty is a no-op
    assert "stride" in isoq.last_error() or isoq.last_error() == ""


def test_decode_validation_happens_on_host():
    lib = isoq.lib()
    ws = isoq.isoq_decode_workspace_size(1, 8, 2, 64, 128)

    def call(**kw):
        a = dict(q=256, dtype=isoq.ISOQ_F16, pk=256, pv=256, nk=256, nv=256, sl=256, B=1, Hq=8,
                 Hkv=2, Tmax=64, d=128, bits=3, variant=0, prk=256, prv=256, scale=0.088,
                 out=256, ws=4096, wsb=ws)
        a.update(kw)
        return lib.isoq_decode_attention(a["q"], a["dtype"], a["pk"], a["pv"], a["nk"], a["nv"],
                                         a["sl"], a["B"], a["Hq"], a["Hkv"], a["Tmax"], a["d"],
                                         a["bits"], a["variant"], a["prk"], a["prv"], a["scale"],
                                         a["out"], a["ws"], a["wsb"], None)

    assert call(Hq=7) == isoq.ISOQ_ERR_INVALID_ARG
    assert call(Hq=64, Hkv=2, wsb=1 << 30) == isoq.ISOQ_ERR_UNSUPPORTED   # group 32 > 16
    assert call(d=64) == isoq.ISOQ_ERR_UNSUPPORTED
    assert call(bits=1) == isoq.ISOQ_ERR_UNSUPPORTED
    assert call(wsb=ws - 1) == isoq.ISOQ_ERR_INVALID_ARG
    assert call(ws=4096 + 16) == isoq.ISOQ_ERR_INVALID_ARG               # not 256-aligned
    assert call(q=None) == isoq.ISOQ_ERR_INVALID_ARG
    assert call(B=0) == isoq.ISOQ_ERR_INVALID_ARG
    assert call(scale=float("nan")) == isoq.ISOQ_ERR_INVALID_ARG
    assert call(out=None) == isoq.ISOQ_ERR_INVALID_ARG
    # the ablation's no-WHT variants are stage-1 only
    assert call(variant=isoq.ISOQ_BLOCK_SO4) == isoq.ISOQ_ERR_UNSUPPORTED
    assert call(variant=isoq.ISOQ_SO3) == isoq.ISOQ_ERR_UNSUPPORTED
    assert call(variant=5) == isoq.ISOQ_ERR_UNSUPPORTED


def test_status_strings():
    for s in (0, -1, -2, -3, -4):
        assert isoq.status_string(s)
    assert isoq.status_string(-99) == "unknown status"


def test_binding_rejects_cpu_tensors():
    torch = pytest.importorskip("torch")
    x = torch.zeros((1, 4, 128), dtype=torch.float16)
    p = torch.zeros((1, 32, 8))
    with pytest.raises(ValueError, match="CUDA"):
        isoq.isoq_quantize(x, p, 3, isoq.ISOQ_FULL)


def test_append_and_step_validation_happens_on_host():
    lib = isoq.lib()
    ws = isoq.isoq_decode_workspace_size(1, 8, 2, 64, 128)

    def append(**kw):
        a = dict(k=256, v=256, dtype=isoq.ISOQ_F16, pk=256, pv=256, nk=256, nv=256, sl=256, B=1,
                 Hkv=2, Tmax=64, d=128, bits=3, variant=0, prk=256, prv=256)
        a.update(kw)
        return lib.isoq_decode_append(a["k"], a["v"], a["dtype"], a["pk"], a["pv"], a["nk"], a["nv"],
                                      a["sl"], a["B"], a["Hkv"], a["Tmax"], a["d"], a["bits"],
                                      a["variant"], a["prk"], a["prv"], None)

    assert append(d=96) == isoq.ISOQ_ERR_UNSUPPORTED
    assert append(bits=5) == isoq.ISOQ_ERR_UNSUPPORTED
    assert append(variant=3) == isoq.ISOQ_ERR_UNSUPPORTED
    assert append(dtype=7) == isoq.ISOQ_ERR_UNSUPPORTED
    assert append(B=0) == isoq.ISOQ_ERR_INVALID_ARG
    assert append(Tmax=0) == isoq.ISOQ_ERR_INVALID_ARG
    assert append(Tmax=1 << 31) == isoq.ISOQ_ERR_INVALID_ARG
    assert append(k=None) == isoq.ISOQ_ERR_INVALID_ARG
    assert append(sl=None) == isoq.ISOQ_ERR_INVALID_ARG
    assert append(prv=None) == isoq.ISOQ_ERR_INVALID_ARG
    assert append(k=256 + 8) == isoq.ISOQ_ERR_UNSUPPORTED               # misaligned
    assert append(sl=256 + 2) == isoq.ISOQ_ERR_UNSUPPORTED

    def step(**kw):
        a = dict(q=256, k=256, v=256, dtype=isoq.ISOQ_F16, pk=256, pv=256, nk=256, nv=256, sl=256,
                 B=1, Hq=8, Hkv=2, Tmax=64, d=128, bits=3, variant=0, prk=256, prv=256, scale=0.088,
                 out=256, ws=4096, wsb=ws)
        a.update(kw)
        return lib.isoq_decode_step(a["q"], a["k"], a["v"], a["dtype"], a["pk"], a["pv"], a["nk"],
                                    a["nv"], a["sl"], a["B"], a["Hq"], a["Hkv"], a["Tmax"], a["d"],
                                    a["bits"], a["variant"], a["prk"], a["prv"], a["scale"], a["out"],
                                    a["ws"], a["wsb"], None)

    # each of these is an attention-half error, caught before the append
    assert step(Hq=7) == isoq.ISOQ_ERR_INVALID_ARG
    assert step(wsb=ws - 1) == isoq.ISOQ_ERR_INVALID_ARG
    assert step(q=None) == isoq.ISOQ_ERR_INVALID_ARG
    assert step(out=None) == isoq.ISOQ_ERR_INVALID_ARG
    assert step(scale=float("inf")) == isoq.ISOQ_ERR_INVALID_ARG
    assert step(out=256 + 4) == isoq.ISOQ_ERR_UNSUPPORTED
    # and the append half's own checks
    assert step(k=None) == isoq.ISOQ_ERR_INVALID_ARG
    assert step(bits=1) == isoq.ISOQ_ERR_UNSUPPORTED


def test_selftest_limit_is_validated_on_the_host():
    """Out-of-range limits are rejected before any launch (no GPU needed)."""
    lib = isoq.lib()
    assert lib.isoq_selftest_wait_timeout(0, None) == isoq.ISOQ_ERR_INVALID_ARG
    assert lib.isoq_selftest_wait_timeout(2_000_000_000, None) == isoq.ISOQ_ERR_INVALID_ARG


def test_prefill_validation_happens_on_host():
    """Every rejected shape or pointer returns before any launch; an empty
    chunk (Tq = 0) is a no-op (the fake pointers are never touched)."""
    lib = isoq.lib()

    def call(**kw):
        a = dict(q=256, dtype=isoq.ISOQ_F16, pk=256, pv=256, nk=256, nv=256, sl=256, B=1, Tq=16,
                 Hq=8, Hkv=2, Tmax=64, d=128, bits=3, variant=0, prk=256, prv=256, scale=0.088,
                 out=256)
        a.update(kw)
        return lib.isoq_prefill_attention(a["q"], a["dtype"], a["pk"], a["pv"], a["nk"], a["nv"],
                                          a["sl"], a["B"], a["Tq"], a["Hq"], a["Hkv"], a["Tmax"],
                                          a["d"], a["bits"], a["variant"], a["prk"], a["prv"],
                                          a["scale"], a["out"], None)

    assert call(d=512) == isoq.ISOQ_ERR_UNSUPPORTED
    assert call(bits=2) == isoq.ISOQ_ERR_UNSUPPORTED
    assert call(variant=isoq.ISOQ_SO3) == isoq.ISOQ_ERR_UNSUPPORTED
    assert call(dtype=isoq.ISOQ_F32) == isoq.ISOQ_ERR_UNSUPPORTED
    assert call(B=0) == isoq.ISOQ_ERR_INVALID_ARG
    assert call(Tq=-1) == isoq.ISOQ_ERR_INVALID_ARG
    assert call(Hq=7) == isoq.ISOQ_ERR_INVALID_ARG                  # Hq % Hkv != 0
    assert call(Hq=32, Hkv=2) == isoq.ISOQ_ERR_UNSUPPORTED          # G = 16
    assert call(Hq=6, Hkv=2) == isoq.ISOQ_ERR_UNSUPPORTED           # G = 3
    assert call(Tmax=60) == isoq.ISOQ_ERR_UNSUPPORTED               # Tmax % 8 != 0
    assert call(q=None) == isoq.ISOQ_ERR_INVALID_ARG
    assert call(prv=None) == isoq.ISOQ_ERR_INVALID_ARG
    assert call(pk=256 + 8) == isoq.ISOQ_ERR_UNSUPPORTED            # misaligned
    assert call(scale=float("nan")) == isoq.ISOQ_ERR_INVALID_ARG
    assert call(Tq=0) == isoq.ISOQ_OK


def test_rotor_validation_happens_on_host():
    lib = isoq.lib()

    def quant(**kw):
        a = dict(x=256, dtype=isoq.ISOQ_F16, nh=1, nv=10, d=128, bits=3, hs=1280, vs=128, rot=256,
                 codes=256, norms=256, ohs=10)
        a.update(kw)
        return lib.isoq_rotor_quantize(a["x"], a["dtype"], a["nh"], a["nv"], a["d"], a["bits"], a["hs"],
                                       a["vs"], a["rot"], a["codes"], a["norms"], a["ohs"], None)

    assert quant(d=96) == isoq.ISOQ_ERR_UNSUPPORTED
    assert quant(bits=5) == isoq.ISOQ_ERR_UNSUPPORTED
    assert quant(dtype=9) == isoq.ISOQ_ERR_UNSUPPORTED
    assert quant(nv=-1) == isoq.ISOQ_ERR_INVALID_ARG
    assert quant(nv=0) == isoq.ISOQ_OK                                # empty: no launch
    assert quant(x=None) == isoq.ISOQ_ERR_INVALID_ARG
    assert quant(vs=64) == isoq.ISOQ_ERR_INVALID_ARG                  # rows overlap
    assert quant(ohs=5) == isoq.ISOQ_ERR_INVALID_ARG                  # output rows overlap
    assert quant(x=256 + 8) == isoq.ISOQ_ERR_UNSUPPORTED              # misaligned
    assert isoq.isoq_rotor_groups(128) == 43 and isoq.isoq_rotor_groups(100) < 0



@pytest.mark.parametrize("fn", ["isoq_dequantize", "isoq_rotor_dequantize"])
def test_dequantize_validation_happens_on_host(fn):
    lib = isoq.lib()
    rotor = fn == "isoq_rotor_dequantize"

    def call(**kw):
        a = dict(codes=256, norms=256, nh=1, nv=10, d=128, bits=3, variant=isoq.ISOQ_FULL, ihs=10,
                 par=256, out=256, dtype=isoq.ISOQ_F16, hs=1280, vs=128)
        a.update(kw)
        if rotor:
            return lib.isoq_rotor_dequantize(a["codes"], a["norms"], a["nh"], a["nv"], a["d"], a["bits"],
                                             a["ihs"], a["par"], a["out"], a["dtype"], a["hs"], a["vs"], None)
        return lib.isoq_dequantize(a["codes"], a["norms"], a["nh"], a["nv"], a["d"], a["bits"],
                                   a["variant"], a["ihs"], a["par"], a["out"], a["dtype"], a["hs"],
                                   a["vs"], None)

    assert call(d=64) == isoq.ISOQ_ERR_UNSUPPORTED
    assert call(bits=1) == isoq.ISOQ_ERR_UNSUPPORTED
    assert call(dtype=5) == isoq.ISOQ_ERR_UNSUPPORTED
    if not rotor:
        assert call(variant=9) == isoq.ISOQ_ERR_UNSUPPORTED
    assert call(nv=-1) == isoq.ISOQ_ERR_INVALID_ARG
    assert call(nv=0) == isoq.ISOQ_OK                                 # empty: no launch
    assert call(out=None) == isoq.ISOQ_ERR_INVALID_ARG
    assert call(ihs=5) == isoq.ISOQ_ERR_INVALID_ARG                   # input rows overlap
    assert call(vs=64) == isoq.ISOQ_ERR_INVALID_ARG                   # output rows overlap
    assert call(out=256 + 4) == isoq.ISOQ_ERR_UNSUPPORTED             # misaligned
    assert call(vs=132) == isoq.ISOQ_ERR_UNSUPPORTED                  # 264-byte rows
