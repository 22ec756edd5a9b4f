"""Float64 CPU oracle for IsoQuant compression and compressed-space attention.

TEST INFRASTRUCTURE ONLY: imported by the tests, the package smoke check and
the benchmark's CPU-baseline leg, never by the product path.  It shares no
code with the CUDA library.  See ``oracle.isoquant`` for the sources and the
readings it follows.
"""

from .isoquant import (  # noqa: F401
    BLOCK_SO4,
    FAST,
    PLANAR,
    SO3,
    VARIANTS,
    FULL,
    SplitMix64,
    bitpack,
    bitunpack,
    combine_partials,
    decode_append,
    decode_attention,
    decode_attention_reconstructed,
    dequantize,
    gaussian_stream,
    hamilton,
    lloyd_max_gaussian,
    make_codebook,
    make_params,
    packed_bytes,
    planar_forward,
    prefill_attention,
    qconj,
    quantize,
    quantize_scalar,
    rotate,
    rotate_inverse,
    so4_fma_count,
    so4_forward,
    so4_inverse,
    split_partials,
    uses_wht,
    wht,
    wht_op_count,
)
