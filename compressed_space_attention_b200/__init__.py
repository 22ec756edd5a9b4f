"""IsoQuant KV compression and compressed-space decode attention for B200.

The product is the CUDA library ``libisoq.so`` (C ABI in ``include/isoq.h``);
this package holds its sources (``csrc/``), the build step (``build.py``) and
a thin ctypes binding (``binding.py``) whose functions carry the C names.
"""

from .binding import (  # noqa: F401
    ISOQ_ERR_CUDA,
    ISOQ_ERR_INVALID_ARG,
    ISOQ_ERR_TIMEOUT,
    ISOQ_ERR_UNSUPPORTED,
    ISOQ_F16,
    ISOQ_F32,
    ISOQ_BLOCK_SO4,
    ISOQ_FAST,
    ISOQ_FULL,
    ISOQ_OK,
    ISOQ_PLANAR,
    ISOQ_SO3,
    IsoqError,
    isoq_abi_version,
    isoq_check_device_error,
    isoq_selftest_wait_timeout,
    isoq_decode_append,
    isoq_decode_attention,
    isoq_decode_combine,
    isoq_decode_num_splits,
    isoq_decode_split,
    isoq_decode_step,
    isoq_decode_workspace_size,
    isoq_dequantize,
    isoq_make_codebook,
    isoq_make_params,
    isoq_packed_bytes,
    isoq_params_size,
    isoq_prefill_attention,
    isoq_quantize,
    isoq_rotor_dequantize,
    isoq_rotor_groups,
    isoq_rotor_make_params,
    isoq_rotor_packed_bytes,
    isoq_rotor_quantize,
    last_error,
    lib,
    status_string,
)
