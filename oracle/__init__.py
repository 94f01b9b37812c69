"""fp64 CPU oracle for hybrid-masked GQA attention with q/k RMSNorm and interleaved mRoPE.

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import, call or execute this
package: only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` use it. It shares no code with the CUDA path (no kernels, headers, tables or
helpers); both sides only share the seeded input generator in ``workloads``.

See ``oracle/reference.py`` for the functions and the passages they follow.
"""
from .reference import (  # noqa: F401
    CAUSAL,
    FULL_SEQUENCE,
    FULL_IN_SEGMENT,
    GEN_IMAGE,
    TILE_SKIP,
    TILE_PARTIAL,
    TILE_FULL,
    ROPE_MROPE_INTERLEAVED,
    ROPE_2D_ALTERNATING,
    ROPE_2D_HALVES,
    bf16_to_f64,
    rms_norm,
    mrope_inv_freq,
    mrope_axis_of_frequency,
    mrope_angles,
    rope_rotate_half,
    prologue,
    dense_mask,
    masked_gqa_attention,
    attention_rows,
    forward,
    unmasked_pairs,
    tile_classes,
    qkv_projection,
    layer_forward,
    layer_rows,
)
