"""MTLA hot path on B200: Python binding of the C ABI in ``include/mtla.h``.

Multi-head Temporal Latent Attention keeps a KV cache compressed in feature
width (MLA-style latents plus decoupled-RoPE keys) and in time (a sigmoid
hyper-network merges every s adjacent steps).  Every step of the hot path runs
in the CUDA library ``libmtla.so``; this package only marshals arguments
(torch tensors -> device pointers, the current CUDA stream) and turns error
statuses into exceptions.  Importing it fails if the library is not built.
"""
from ._abi import (  # noqa: F401
    DECODE_STATIC_SCRATCH_BYTES,
    DEVERR_CAPACITY,
    DEVERR_EMPTY,
    DEVERR_PE_RANGE,
    DEVERR_TIMEOUT,
    LIB_PATH,
    MTLA_BF16,
    MAX_NEW_TOKENS,
    MTLA_F32,
    PROJ_IN,
    PROJ_OUT,
    TRAIN_ATTN_BWD,
    TRAIN_KV_BWD,
    TRAIN_MERGE_BWD,
    WS_DECODE,
    MtlaError,
    dims,
    exported_symbols,
    lib,
    mtla_cache_length,
    mtla_debug_stride_mask,
    mtla_decode_attn,
    mtla_decode_attn_multi,
    mtla_decode_multi_workspace_bytes,
    mtla_decode_attn_static,
    mtla_merge_append,
    mtla_prefill_kv,
    mtla_prefill_masked_attn,
    mtla_prefill_unabsorbed_attn,
    mtla_project_in,
    mtla_project_out,
    mtla_project_workspace_bytes,
    mtla_status_string,
    mtla_train_attn_bwd,
    mtla_train_attn_fwd,
    mtla_train_kv_bwd,
    mtla_train_merge_bwd,
    mtla_train_workspace_bytes,
    mtla_workspace_bytes,
)
