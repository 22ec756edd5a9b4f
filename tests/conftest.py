import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")


import numpy as np  # noqa: E402
import pytest  # noqa: E402


@pytest.fixture(scope="session")
def prefill_kv():
    """Prefill-compression workload: 4 KV heads x 32,768 tokens x d=128,
    float16 Student-t (nu=4) with outlier channels and RoPE on K, plus the
    oracle's compression of it (K rotation seed 1, V rotation seed 2)."""
    import oracle as O
    import synth

    k, v = synth.student_t_kv(n_heads=4, t=32768, d=128, seed=3)
    k, v = k[0], v[0]
    pk_params = O.make_params(128, O.FULL, seed=1, n_heads=4)
    pv_params = O.make_params(128, O.FULL, seed=2, n_heads=4)
    ok = O.quantize(k.astype(np.float64), pk_params, 3, O.FULL, return_rotated=True)
    ov = O.quantize(v.astype(np.float64), pv_params, 3, O.FULL, return_rotated=True)
    return dict(k=k, v=v, params_k=pk_params, params_v=pv_params, oracle_k=ok, oracle_v=ov)
