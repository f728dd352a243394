"""paged_kv_cache_407_b200: the decode hot path of a paged KV cache on B200.

The compute lives in ``libpkv.so`` (C ABI, ``include/pkv.h``); this package is
its thin binding plus host-side byte accounting.
"""

from .binding import (  # noqa: F401
    DEV_BAD_BLOCK,
    DEV_BAD_LEN,
    DEV_BAD_SLOT,
    DEV_TIMEOUT,
    CHECK_LIB_PATH,
    ERR_ALIAS,
    LIB_PATH,
    PREFILL_WORKSPACE_BYTES,
    PkvError,
    PreparedCall,
    cache_desc,
    check_library,
    copy_blocks,
    fp8_cache_desc,
    library,
    merge_attention_states,
    paged_attention_decode,
    paged_attention_decode_lse,
    paged_prefill,
    paged_attention_decode_fp8,
    partition_size,
    reshape_and_cache,
    reshape_and_cache_fp8,
    state_buffer,
    state_views,
    use_check_build,
    version,
    workspace_size,
)
