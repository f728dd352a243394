"""Oracle package: TEST INFRASTRUCTURE ONLY (see ``oracle.paged_kv``).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` import this package.  The CUDA library and its Python binding do
not, and this package imports nothing from them.
"""

from .paged_kv import (  # noqa: F401
    BF16,
    F16,
    append_token,
    attend,
    copy_blocks,
    decode_bits,
    decode_sequence,
    e4m3_decode,
    e4m3_encode,
    encode_bits,
    free_request,
    kv_head_of,
    lse_combine,
    materialize,
    materialize_fp8,
    paged_attention_decode,
    paged_attention_decode_fp8,
    partial_state,
    quantize_e4m3,
    reshape_and_cache,
    reshape_and_cache_fp8,
    slot_location,
)
from .prefill import paged_prefill  # noqa: F401,E402
