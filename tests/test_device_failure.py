"""Failure detection on the GPU without a fault: a device wait that nothing
ends gives up after its limit, records a timeout in the device error word,
and the host reads ISOQ_ERR_TIMEOUT; the context stays usable."""

import numpy as np
import pytest

import oracle as O
import synth

torch = pytest.importorskip("torch")
import compressed_space_attention_b200 as isoq  # noqa: E402

pytestmark = pytest.mark.gpu

DEV = "cuda"


def test_bounded_wait_gives_up_and_is_reported():
    assert isoq.isoq_check_device_error() == isoq.ISOQ_OK
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    isoq.isoq_selftest_wait_timeout(50_000_000)          # 50 ms
    t1.record()
    torch.cuda.synchronize()
    assert t0.elapsed_time(t1) >= 45.0                   # it waited for its limit
    assert isoq.isoq_check_device_error() == isoq.ISOQ_ERR_TIMEOUT
    assert isoq.isoq_check_device_error() == isoq.ISOQ_OK  # read and cleared

    # The context is still usable: a compression right after it is exact.
    x = synth.unit_vectors(1000, 128, seed=31, dtype=np.float16)
    params = O.make_params(128, O.FULL, seed=1)
    codes, norms = isoq.isoq_quantize(torch.from_numpy(x).to(DEV), torch.from_numpy(params).to(DEV), 3, O.FULL)
    torch.cuda.synchronize()
    assert isoq.isoq_check_device_error() == isoq.ISOQ_OK
    oc, on = O.quantize(x.astype(np.float64), params, 3, O.FULL)
    assert np.mean(codes.cpu().numpy() == oc) > 0.999
