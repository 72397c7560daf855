"""B200 (sm_100a) locality-constrained block-sparse causal attention.

FlashVSR's LCSA attention core as a C-ABI CUDA library (liblcsa.so, declared
in include/lcsa.h) with a thin PyTorch binding: block pooling, block
selection (causal + locality window + top-K), tcgen05 sparse attention and
the streaming KV-cache append.
"""
from .api import (  # noqa: F401
    HostPipeline,
    KVCache,
    LcsaError,
    NativePipeline,
    SelectParams,
    StreamingStep,
    WINDOW_PRESERVE,
    WINDOW_PRESERVE_TOKENS,
    WINDOW_TRUNCATE,
    WINDOW_TRUNCATE_TOKENS,
    attn_workspace,
    debug_exp2_poly,
    debug_set_wait_limit_ns,
    debug_stalled_wait,
    ingest_chunk,
    kv_append,
    last_device_error,
    pool_qk,
    segment_blocks,
    select_blocks,
    select_blocks_noalloc,
    select_kmax,
    select_workspace_bytes,
    sparse_attn_bwd,
    sparse_attn_bwd_workspace_bytes,
    sparse_attn_fwd,
    tensor_desc,
)
from .build import LIB_PATH  # noqa: F401
from .partition import rank_slices, rank_units  # noqa: F401
