"""B200-native (sm_100a) hybrid-masked GQA attention for unified text+pixel sequences.

The compute lives in ``libhgx_attn.so`` (C ABI, ``include/hgx_attn.h``); this package is a
thin ctypes binding with the same names. There is no fallback: if the library is missing
or the GPU is not an sm_100a part, every call raises.
"""
from .binding import (  # noqa: F401
    HGX_OK,
    HGX_ERR_INVALID_ARG,
    HGX_ERR_UNSUPPORTED,
    HGX_ERR_OOM,
    HGX_ERR_CUDA,
    HGX_ERR_TIMEOUT,
    HGX_SEG_CAUSAL,
    HGX_SEG_FULL_SEQUENCE,
    HGX_SEG_FULL_IN_SEGMENT,
    HGX_SEG_GEN_IMAGE,
    HGX_TILE_SKIP,
    HGX_TILE_PARTIAL,
    HGX_TILE_FULL,
    HGX_DEBUG_CHECKED,
    HGX_DEBUG_STALL_TEST,
    HGX_DEBUG_FAIL_ALLOC,
    HGX_DEBUG_SPLIT_TEST,
    HGX_ROPE_MROPE_INTERLEAVED,
    HGX_ROPE_2D_ALTERNATING,
    HGX_ROPE_2D_HALVES,
    HgxError,
    AttnConfig,
    Attention,
    lib,
    library_path,
    row_limits,
    visible_pairs,
    schedule,
    classify,
)
