"""isoq_decode_attention_static: decode attention for callers that cannot
allocate device memory (for example a host program whose device memory is
owned by another framework's allocator, or a plugin handed only its inputs
and outputs).  Its split-K scratch is a fixed array inside the library.

The test calls the entry point through the C ABI with raw device pointers,
several times in a row on different inputs (the last one with lengths that
leave most splits empty, right after a long call), and checks each output
against the regular isoq_decode_attention (caller-provided workspace) on the
same input, within the attention tolerance of the parity tests.  This file is named so
that pytest collects it last.
"""

import ctypes
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


def _case(seed, b, hq, hkv, tmax, d, dtype):
    g = synth.rng(seed)
    pb = d * 3 // 8
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(DEV)  # noqa: E731
    return dict(
        q=t(synth.queries(b, hq, d, seed=seed + 1, dtype=dtype)),
        pk=t(g.integers(0, 256, size=(b, hkv, tmax, pb), dtype=np.uint8)),
        pv=t(g.integers(0, 256, size=(b, hkv, tmax, pb), dtype=np.uint8)),
        nk=t(g.lognormal(2.5, 0.3, (b, hkv, tmax)).astype(np.float16)),
        nv=t(g.lognormal(1.0, 0.3, (b, hkv, tmax)).astype(np.float16)),
        lens=t(g.integers(1, tmax + 1, size=b).astype(np.int32)),
        prk=t(O.make_params(d, O.FULL, seed=seed + 2, n_heads=hkv)),
        prv=t(O.make_params(d, O.FULL, seed=seed + 3, n_heads=hkv)),
        shape=(b, hq, hkv, tmax, d),
    )


def _static_call(c, out, dtype_code):
    b, hq, hkv, tmax, d = c["shape"]
    lib = isoq.lib()
    return lib.isoq_decode_attention_static(
        c["q"].data_ptr(), dtype_code, c["pk"].data_ptr(), c["pv"].data_ptr(),
        c["nk"].data_ptr(), c["nv"].data_ptr(), c["lens"].data_ptr(), b, hq, hkv, tmax, d, 3,
        isoq.ISOQ_FULL, c["prk"].data_ptr(), c["prv"].data_ptr(), ctypes.c_float(1 / math.sqrt(d)),
        out.data_ptr(), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_static_workspace_matches_allocating_entry_point_twice():
    long_case = _case(11, 4, 16, 8, 4096, 256, np.float16)
    # the same shapes with lengths that leave most splits empty, right after
    # the long call filled the array with partial states
    short_case = dict(long_case, lens=torch.tensor([1, 37, 0, 300], dtype=torch.int32, device=DEV))
    cases = [(long_case, isoq.ISOQ_F16, np.float16),
             (_case(12, 3, 8, 2, 1000, 128, np.float32), isoq.ISOQ_F32, np.float32),
             (long_case, isoq.ISOQ_F16, np.float16),
             (short_case, isoq.ISOQ_F16, np.float16)]
    for c, code, dt in cases:
        b, hq, hkv, tmax, d = c["shape"]
        ref = isoq.isoq_decode_attention(c["q"], c["pk"], c["pv"], c["nk"], c["nv"], c["lens"],
                                         c["prk"], c["prv"], 3, isoq.ISOQ_FULL)
        out = torch.empty_like(ref)
        torch.cuda.synchronize()
        before = (torch.cuda.memory_allocated(), torch.cuda.memory_reserved())
        assert _static_call(c, out, code) == isoq.ISOQ_OK, isoq.last_error()
        torch.cuda.synchronize()
        # nothing went through torch's allocator either
        assert (torch.cuda.memory_allocated(), torch.cuda.memory_reserved()) == before
        check_attention(out.cpu().numpy(), ref.cpu().numpy(), dt)
    assert isoq.isoq_check_device_error() == 0


def test_rejects_shapes_beyond_the_builtin_workspace():
    cap = isoq.lib().isoq_decode_static_workspace_bytes()
    assert cap == 16 << 20
    b, hq, hkv, tmax, d = 64, 64, 8, 65536, 512
    assert isoq.isoq_decode_workspace_size(b, hq, hkv, tmax, d) > cap
    dummy = torch.empty(256, dtype=torch.uint8, device=DEV)
    p = dummy.data_ptr()
    st = isoq.lib().isoq_decode_attention_static(p, isoq.ISOQ_F16, p, p, p, p, p, b, hq, hkv, tmax,
                                                 d, 3, isoq.ISOQ_FULL, p, p, ctypes.c_float(0.04),
                                                 p, None)
    assert st == isoq.ISOQ_ERR_UNSUPPORTED
    assert "workspace" in isoq.last_error()
