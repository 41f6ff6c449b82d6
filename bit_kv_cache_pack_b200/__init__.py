"""OmniKVQuant 2-bit KV-cache write and fused decode attention for B200 (sm_100a).

The compute lives in libomnikv.so (hand-written CUDA behind the C ABI of
include/omnikv.h); this package is its thin Python binding plus PyTorch
allocation helpers.
"""
from ._abi import (OMNIKV_DEVERR_CAPACITY, OMNIKV_ERR_CAPACITY, OMNIKV_ERR_CUDA,  # noqa: F401
                   OMNIKV_META_FP16, OMNIKV_META_MXFP4, OMNIKV_META_TURBO, omnikv_record_bytes_meta,
                   OMNIKV_ERR_INVALID_ARG, OMNIKV_ERR_UNSUPPORTED, OMNIKV_OK, OmniKVCache,
                   OmniKVConfig, OmniKVError, load, omnikv_abi_version, omnikv_combine,
                   omnikv_append_decode, omnikv_calibrate_bases, omnikv_calibrate_workspace_bytes,
                   omnikv_combine_step, omnikv_decode_attention, omnikv_decode_static,
                   omnikv_decode_step, omnikv_step_splits, omnikv_default_splits, omnikv_dense_decode_bf16,
                   omnikv_dense_partials_bytes, omnikv_partials_bytes,
                   omnikv_record_bytes, omnikv_stream_decode, omnikv_stream_write_cache,
                   omnikv_test_decode_pending, omnikv_write_cache,
                   omnikv_write_cache_rotations, status_string)
from .layer import KVCache, LayerConstants, partials_tensor, stream_rings  # noqa: F401
