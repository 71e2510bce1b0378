"""B200 (sm_100a) MLA decoding over a paged latent KV cache.

The compute path lives in libmla_b200.so (C ABI, include/mla.h); this package
is its Python binding (argument marshalling) plus buffer plumbing.
"""
from ._capi import (  # noqa: F401
    MLA_DEBUG_SKIP_COMBINE, MLA_DEBUG_WITHHOLD_SCORES, MLA_DEVICE_STATUS_BOUNDS, MLA_DEVICE_STATUS_TIMEOUT, MLA_ERR_CUDA,
    MLA_ERR_DEVICE_BOUNDS, MLA_ERR_DEVICE_TIMEOUT, MLA_ERR_INVALID_ARG, MLA_ERR_UNSUPPORTED,
    MLA_ERR_WORKSPACE_TOO_SMALL, MLA_KV_BF16, MLA_KV_FP8_E4M3, MLA_KV_NVFP4, MLA_MAX_ROWS, MLA_OK, MLA_TILE_MD_INTS,
    LIB_PATH, MLAError, MlaDecodeArgs, lib, make_args, mla_clear_device_status, mla_combine,
    mla_combine_sink, mla_decode_geometry, mla_out_rope_fp8, mla_q_norm_rope, mla_decode_paged, mla_decode_sparse, mla_get_metadata, mla_get_metadata_host, mla_get_num_sm_parts,
    mla_query_device_status, mla_status_string, mla_workspace_size)
from .runner import DecodeRunner  # noqa: F401
