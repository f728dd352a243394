"""Thin Python binding of libpkv (``include/pkv.h``) over torch tensors.

Argument marshalling only: every step of the hot path runs in the CUDA
kernels of ``libpkv.so``.  There is no fallback: if the library is missing or
the device is not a B200 the calls raise.
"""

from __future__ import annotations

import ctypes
import os

import torch

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG_DIR, "libpkv.so")
CHECK_LIB_PATH = os.path.join(PKG_DIR, "libpkv_check.so")

# pkv_status
OK = 0
STATUS_NAMES = {
    0: "PKV_OK", 1: "PKV_ERR_NULL_POINTER", 2: "PKV_ERR_BAD_DTYPE", 3: "PKV_ERR_BAD_SHAPE",
    4: "PKV_ERR_MISALIGNED", 5: "PKV_ERR_WORKSPACE", 6: "PKV_ERR_BAD_PARTITION",
    7: "PKV_ERR_TOO_LARGE", 8: "PKV_ERR_CUDA", 9: "PKV_ERR_DEVICE",
    10: "PKV_ERR_NO_BLOCKS", 11: "PKV_ERR_BAD_SEQUENCE", 12: "PKV_ERR_ALIAS",
}
ERR_TOO_LARGE = 7
ERR_NO_BLOCKS = 10
ERR_BAD_SEQUENCE = 11
ERR_ALIAS = 12
# device-side flags
DEV_BAD_BLOCK = 0x1
DEV_BAD_SLOT = 0x2
DEV_BAD_LEN = 0x4
DEV_TIMEOUT = 0x8

PKV_F16 = 0
PKV_BF16 = 1
PKV_FP8_E4M3 = 2
_DTYPES = {torch.float16: PKV_F16, torch.bfloat16: PKV_BF16}
_FP8_DTYPES = (torch.uint8, torch.float8_e4m3fn)

# Every function declared in include/*.h, with (restype, argtypes).
_c_void_p, _i32, _i64, _f32, _size_t = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t


class CacheDesc(ctypes.Structure):
    """``pkv_cache_desc``."""

    _fields_ = [
        ("num_blocks", ctypes.c_int32),
        ("block_size", ctypes.c_int32),
        ("num_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("dtype", ctypes.c_int),
    ]


SIGNATURES = {
    "pkv_reshape_and_cache": (ctypes.c_int, [_c_void_p, _c_void_p, _i64, _i64, _c_void_p, _c_void_p,
                                             CacheDesc, _c_void_p, _i32, _c_void_p, _c_void_p]),
    "pkv_paged_attention_workspace_size": (_size_t, [_i32, _i32, _i32, _i32, _i32, _i32, _i32]),
    "pkv_paged_attention_partition_size": (_i32, [_i32, _i32, _i32, _i32, _i32]),
    "pkv_paged_attention_decode": (ctypes.c_int, [_c_void_p, _c_void_p, _c_void_p, _c_void_p, CacheDesc,
                                                  _c_void_p, _i32, _c_void_p, _i32, _i32, _i32, _f32,
                                                  _i32, _c_void_p, _size_t, _c_void_p, _c_void_p]),
    "pkv_paged_attention_decode_noalloc": (ctypes.c_int, [_c_void_p, _c_void_p, _c_void_p, _c_void_p,
                                                          CacheDesc, _c_void_p, _i32, _c_void_p, _i32,
                                                          _i32, _i32, _f32, _i32, _c_void_p, _c_void_p]),
    "pkv_copy_blocks": (ctypes.c_int, [_c_void_p, _c_void_p, CacheDesc, _c_void_p, _i32, _c_void_p,
                                       _c_void_p]),
    "pkv_reshape_and_cache_fp8": (ctypes.c_int, [_c_void_p, _c_void_p, _i64, _i64, ctypes.c_int, _c_void_p,
                                                 _c_void_p, CacheDesc, _c_void_p, _i32, _f32, _f32,
                                                 _c_void_p, _c_void_p]),
    "pkv_paged_attention_decode_fp8": (ctypes.c_int, [_c_void_p, _c_void_p, ctypes.c_int, _c_void_p, _c_void_p,
                                                      CacheDesc, _c_void_p, _i32, _c_void_p, _i32, _i32, _i32,
                                                      _f32, _f32, _f32, _i32, _c_void_p, _size_t, _c_void_p,
                                                      _c_void_p]),
    "pkv_paged_attention_decode_lse": (ctypes.c_int, [_c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_void_p,
                                                      CacheDesc, _c_void_p, _i32, _c_void_p, _i32, _i32, _i32,
                                                      _f32, _i32, _c_void_p, _size_t, _c_void_p, _c_void_p]),
    "pkv_merge_attention_states": (ctypes.c_int, [_c_void_p, ctypes.c_int, _c_void_p, _i64, _i32, _i32, _i32,
                                                  _c_void_p]),
    "pkv_paged_prefill": (ctypes.c_int, [_c_void_p, _c_void_p, _c_void_p, _c_void_p, CacheDesc, _c_void_p, _i32,
                                         _c_void_p, _c_void_p, _i32, _i32, _i32, _i32, _f32, _c_void_p,
                                         ctypes.c_size_t, _c_void_p, _c_void_p]),
    "pkv_test_decode_withheld_load": (ctypes.c_int, [_c_void_p, _c_void_p, _c_void_p, _c_void_p, CacheDesc,
                                                     _c_void_p, _i32, _c_void_p, _i32, _i32, _i32, _f32, _i32,
                                                     _c_void_p, _size_t, _i32, ctypes.c_uint32, _c_void_p,
                                                     _c_void_p]),
    "pkv_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    # include/pkv_block_manager.h (host only)
    "pkv_bm_create": (ctypes.c_int, [_i32, _i32, _i32, ctypes.POINTER(_c_void_p)]),
    "pkv_bm_destroy": (None, [_c_void_p]),
    "pkv_bm_num_free_blocks": (_i32, [_c_void_p]),
    "pkv_bm_num_sequences": (_i32, [_c_void_p]),
    "pkv_bm_ref_count": (_i32, [_c_void_p, _i32]),
    "pkv_bm_context_len": (_i32, [_c_void_p, _i64]),
    "pkv_bm_add_sequence": (ctypes.c_int, [_c_void_p, _i64, _i32, _c_void_p]),
    "pkv_bm_fork": (ctypes.c_int, [_c_void_p, _i64, _i64]),
    "pkv_bm_free_sequence": (ctypes.c_int, [_c_void_p, _i64]),
    "pkv_bm_blocks_needed": (_i32, [_c_void_p, _c_void_p, _i32]),
    "pkv_bm_append": (ctypes.c_int, [_c_void_p, _c_void_p, _i32, _c_void_p, _c_void_p, _i32,
                                     ctypes.POINTER(_i32)]),
    "pkv_bm_block_tables": (ctypes.c_int, [_c_void_p, _c_void_p, _i32, _c_void_p, _i32, _c_void_p]),
    "pkv_bm_free_list": (ctypes.c_int, [_c_void_p, _c_void_p, _i32, ctypes.POINTER(_i32)]),
    "pkv_version": (_i32, []),
    "pkv_check_build": (_i32, []),
}

_lib = None
_check_lib = None


class PkvError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        name = STATUS_NAMES.get(status, str(status))
        text = library().pkv_status_string(status).decode()
        super().__init__(f"{where}: {name} ({text})")


def load(path: str) -> ctypes.CDLL:
    """Open one build of the library and give every entry point its C
    signature.  Raises if the file is missing."""
    if not os.path.exists(path):
        flag = " --check" if path == CHECK_LIB_PATH else ""
        raise RuntimeError(f"{path} is missing: build it with `python -m paged_kv_cache_407_b200.build{flag}`")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


def library() -> ctypes.CDLL:
    """The build every binding call goes through: libpkv.so, loaded on first
    use, unless use_check_build() chose the check build first.  Raises if it
    has not been built."""
    global _lib
    if _lib is None:
        _lib = load(LIB_PATH)
    return _lib


def check_library() -> ctypes.CDLL:
    """The check build libpkv_check.so (PKV_CHECK: the cache write and the
    block copy also verify that no slot / copy destination repeats,
    synchronising the stream; see include/pkv.h), loaded once, beside
    whichever build library() serves.  Its calls take the same C arguments."""
    global _check_lib
    if _check_lib is None:
        _check_lib = load(CHECK_LIB_PATH)
    return _check_lib


def use_check_build() -> None:
    """Route every later binding call to the check build.  Call it before the
    first library call of the process; raises if libpkv.so is already in use."""
    global _lib
    if _lib is not None and _lib is not check_library():
        raise RuntimeError("libpkv.so is already in use: call use_check_build() before the first library call")
    _lib = check_library()


def _check(status: int, where: str) -> None:
    if status != OK:
        raise PkvError(status, where)


class PreparedCall:
    """One library call whose arguments were checked and marshalled once
    (``prepare=True`` on the calls that accept it): calling it issues the C
    call again with the same tensors, scalars and stream, and raises on a
    non-zero status as the plain call does.  It keeps the tensors it refers
    to alive.  For loops that repeat a call on fixed buffers, where the
    per-call argument checks would cost more host time than the launch."""

    __slots__ = ("_fn", "_argv", "_where", "_keep", "result")

    def __init__(self, fn, argv, where, keep, result):
        self._fn, self._argv, self._where, self._keep, self.result = fn, argv, where, keep, result

    def __call__(self):
        st = self._fn(*self._argv)
        if st != OK:
            raise PkvError(st, self._where)
        return self.result


def _invoke(fn, argv, where, prepare, keep=(), result=None):
    if prepare:
        return PreparedCall(fn, tuple(argv), where, keep, result)
    _check(fn(*argv), where)
    return result


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream, device) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream)


def cache_desc(k_cache: torch.Tensor) -> CacheDesc:
    """Descriptor of a ``[num_blocks, num_kv_heads, block_size, head_dim]`` pool."""
    if k_cache.dim() != 4 or not k_cache.is_contiguous():
        raise ValueError("cache must be a contiguous [num_blocks, num_kv_heads, block_size, head_dim] tensor")
    if k_cache.dtype not in _DTYPES:
        raise TypeError(f"cache dtype must be float16 or bfloat16, got {k_cache.dtype}")
    N, Hkv, B, D = k_cache.shape
    return CacheDesc(N, B, Hkv, D, _DTYPES[k_cache.dtype])


def _same_pool(k_cache, v_cache):
    if v_cache.shape != k_cache.shape or v_cache.dtype != k_cache.dtype or not v_cache.is_contiguous():
        raise ValueError("k_cache and v_cache must have the same shape, dtype and layout")


def reshape_and_cache(key, value, k_cache, v_cache, slot_mapping, d_status=None, stream=None, prepare=False):
    """Write new tokens ``key/value [T, Hkv, D]`` into the slots ``slot_mapping [T]`` (int64)."""
    desc = cache_desc(k_cache)
    _same_pool(k_cache, v_cache)
    T = key.shape[0]
    for t in (key, value):
        if t.dim() != 3 or t.shape[1:] != k_cache.shape[1:2] + k_cache.shape[3:4] or t.dtype != k_cache.dtype:
            raise ValueError("key/value must be [T, num_kv_heads, head_dim] in the cache dtype")
        if t.stride(2) != 1 or t.stride(1) != t.shape[2]:
            raise ValueError("key/value heads and dims must be contiguous within a token")
    if slot_mapping.dtype != torch.int64 or slot_mapping.numel() != T or not slot_mapping.is_contiguous():
        raise ValueError("slot_mapping must be a contiguous int64 tensor with one entry per token")
    return _invoke(library().pkv_reshape_and_cache,
                   (_ptr(key), _ptr(value), key.stride(0), value.stride(0), _ptr(k_cache), _ptr(v_cache), desc,
                    _ptr(slot_mapping), T, _ptr(d_status), _stream(stream, k_cache.device)),
                   "pkv_reshape_and_cache", prepare, (key, value, k_cache, v_cache, slot_mapping, d_status))


def _workspace(workspace, S, Hq, desc, D, max_context_len, partition_size, device):
    """The caller's workspace and its size in bytes, or, when the caller gave
    none and one is needed, a fresh torch allocation (the library itself
    never allocates)."""
    if workspace is not None:
        return workspace, workspace.numel() * workspace.element_size()
    need = workspace_size(S, Hq, desc.num_kv_heads, D, desc.block_size, max_context_len, partition_size)
    if need == 0:
        return None, 0
    return torch.empty(need, dtype=torch.uint8, device=device), need


def workspace_size(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, max_context_len,
                   partition_size=0) -> int:
    return int(library().pkv_paged_attention_workspace_size(
        num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, max_context_len, partition_size))


def partition_size(num_seqs, num_kv_heads, block_size, max_context_len, partition_size=0) -> int:
    return int(library().pkv_paged_attention_partition_size(
        num_seqs, num_kv_heads, block_size, max_context_len, partition_size))


def paged_attention_decode(out, query, k_cache, v_cache, block_tables, context_lens, max_context_len,
                           scale, partition_size=0, workspace=None, d_status=None, stream=None, prepare=False):
    """Decode attention: ``out [S, Hq, D] = attention(query [S, Hq, D], paged K/V)``.

    ``workspace``: a device tensor of at least ``workspace_size(...)`` bytes;
    when None and one is needed it is allocated with torch (the library
    itself never allocates).
    """
    desc = cache_desc(k_cache)
    _same_pool(k_cache, v_cache)
    S, Hq, D = query.shape
    if out.shape != query.shape or out.dtype != k_cache.dtype or query.dtype != k_cache.dtype:
        raise ValueError("query/out must be [S, Hq, head_dim] in the cache dtype")
    if not (query.is_contiguous() and out.is_contiguous()):
        raise ValueError("query/out must be contiguous")
    if block_tables.dtype != torch.int32 or block_tables.dim() != 2 or block_tables.shape[0] != S \
            or not block_tables.is_contiguous():
        raise ValueError("block_tables must be a contiguous int32 [S, max_blocks_per_seq] tensor")
    if context_lens.dtype != torch.int32 or context_lens.numel() != S or not context_lens.is_contiguous():
        raise ValueError("context_lens must be a contiguous int32 [S] tensor")
    workspace, ws_bytes = _workspace(workspace, S, Hq, desc, D, max_context_len, partition_size, query.device)
    return _invoke(library().pkv_paged_attention_decode,
                   (_ptr(out), _ptr(query), _ptr(k_cache), _ptr(v_cache), desc, _ptr(block_tables),
                    block_tables.shape[1], _ptr(context_lens), S, Hq, int(max_context_len), float(scale),
                    int(partition_size), _ptr(workspace), ws_bytes, _ptr(d_status), _stream(stream, query.device)),
                   "pkv_paged_attention_decode", prepare,
                   (out, query, k_cache, v_cache, block_tables, context_lens, workspace, d_status), out)


def paged_attention_decode_lse(out, lse, query, k_cache, v_cache, block_tables, context_lens, max_context_len,
                               scale, partition_size=0, workspace=None, d_status=None, stream=None):
    """Decode attention over the tokens the tables describe, returned as an
    attention state: ``out`` fp32 ``[S, Hq, D]`` (normalised) and ``lse`` fp32
    ``[S, Hq]`` (natural log of the softmax denominator, -inf for no tokens).
    ``out`` and ``lse`` may be views of one packed buffer (``state_buffer``)."""
    desc = cache_desc(k_cache)
    _same_pool(k_cache, v_cache)
    S, Hq, D = query.shape
    if query.dtype != k_cache.dtype or not query.is_contiguous():
        raise ValueError("query must be a contiguous [S, Hq, head_dim] tensor in the cache dtype")
    if out.dtype != torch.float32 or tuple(out.shape) != (S, Hq, D) or not out.is_contiguous():
        raise ValueError("out must be a contiguous float32 [S, Hq, head_dim] tensor")
    if lse.dtype != torch.float32 or lse.numel() != S * Hq or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous float32 [S, Hq] tensor")
    if block_tables.dtype != torch.int32 or block_tables.dim() != 2 or block_tables.shape[0] != S \
            or not block_tables.is_contiguous():
        raise ValueError("block_tables must be a contiguous int32 [S, max_blocks_per_seq] tensor")
    if context_lens.dtype != torch.int32 or context_lens.numel() != S or not context_lens.is_contiguous():
        raise ValueError("context_lens must be a contiguous int32 [S] tensor")
    workspace, ws_bytes = _workspace(workspace, S, Hq, desc, D, max_context_len, partition_size, query.device)
    st = library().pkv_paged_attention_decode_lse(
        _ptr(out), _ptr(lse), _ptr(query), _ptr(k_cache), _ptr(v_cache), desc, _ptr(block_tables),
        block_tables.shape[1], _ptr(context_lens), S, Hq, int(max_context_len), float(scale),
        int(partition_size), _ptr(workspace), ws_bytes, _ptr(d_status), _stream(stream, query.device))
    _check(st, "pkv_paged_attention_decode_lse")
    return out, lse


def state_buffer(num_rows: int, head_dim: int, num_states: int = 1, device="cuda") -> torch.Tensor:
    """fp32 ``[num_states, num_rows * (head_dim + 1)]``: per state, the rows'
    outputs followed by their log-sum-exps (the layout the merge reads)."""
    return torch.empty((num_states, num_rows * (head_dim + 1)), dtype=torch.float32, device=device)


def state_views(state: torch.Tensor, num_seqs: int, num_q_heads: int, head_dim: int):
    """(out ``[S, Hq, D]``, lse ``[S, Hq]``) views of one state of a state buffer."""
    rows = num_seqs * num_q_heads
    return (state[: rows * head_dim].view(num_seqs, num_q_heads, head_dim),
            state[rows * head_dim: rows * (head_dim + 1)].view(num_seqs, num_q_heads))


def merge_attention_states(out, states, stream=None):
    """Merge ``states`` (``[R, rows * (D + 1)]`` fp32, see ``state_buffer``)
    into ``out`` (fp16/bf16 ``[..., D]`` with ``rows`` rows)."""
    if out.dtype not in _DTYPES or not out.is_contiguous():
        raise ValueError("out must be a contiguous fp16/bf16 tensor")
    D = out.shape[-1]
    rows = out.numel() // D
    if states.dtype != torch.float32 or states.dim() != 2 or states.shape[1] < rows * (D + 1) \
            or not states.is_contiguous():
        raise ValueError("states must be a contiguous float32 [R, rows * (head_dim + 1)] tensor")
    st = library().pkv_merge_attention_states(_ptr(out), _DTYPES[out.dtype], _ptr(states), states.shape[1],
                                              states.shape[0], rows, D, _stream(stream, out.device))
    _check(st, "pkv_merge_attention_states")
    return out


def paged_prefill(out, query, k_cache, v_cache, block_tables, query_start, context_lens, max_query_len, scale,
                  d_status=None, stream=None, prepare=False, dynamic=True, workspace=None):
    """Causal attention of chunks of new tokens over their sequences' paged
    K/V: ``query``/``out`` ``[T, Hq, 128]``; sequence s owns rows
    ``query_start[s] .. query_start[s+1]`` (its last tokens, already written
    to the cache); ``context_lens`` counts them.

    ``dynamic``: the CTAs take the work items from a counter in ``workspace``
    (a device tensor of at least PREFILL_WORKSPACE_BYTES; allocated with
    torch when None), which keeps them evenly loaded when the chunks differ
    in length; False: a fixed assignment (no workspace).  Same outputs."""
    desc = cache_desc(k_cache)
    _same_pool(k_cache, v_cache)
    T, Hq, D = query.shape
    if out.shape != query.shape or out.dtype != k_cache.dtype or query.dtype != k_cache.dtype:
        raise ValueError("query/out must be [T, Hq, head_dim] in the cache dtype")
    if not (query.is_contiguous() and out.is_contiguous()):
        raise ValueError("query/out must be contiguous")
    S = context_lens.numel()
    if block_tables.dtype != torch.int32 or block_tables.dim() != 2 or block_tables.shape[0] != S \
            or not block_tables.is_contiguous():
        raise ValueError("block_tables must be a contiguous int32 [S, max_blocks_per_seq] tensor")
    for t, n in ((query_start, S + 1), (context_lens, S)):
        if t.dtype != torch.int32 or t.numel() != n or not t.is_contiguous():
            raise ValueError("query_start / context_lens must be contiguous int32 [S + 1] / [S] tensors")
    if dynamic and workspace is None:
        workspace = torch.empty(PREFILL_WORKSPACE_BYTES, dtype=torch.uint8, device=query.device)
    if not dynamic:
        workspace = None
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    return _invoke(library().pkv_paged_prefill,
                   (_ptr(out), _ptr(query), _ptr(k_cache), _ptr(v_cache), desc, _ptr(block_tables),
                    block_tables.shape[1], _ptr(query_start), _ptr(context_lens), S, T, int(max_query_len), Hq,
                    float(scale), _ptr(workspace), ws_bytes, _ptr(d_status), _stream(stream, query.device)),
                   "pkv_paged_prefill", prepare,
                   (out, query, k_cache, v_cache, block_tables, query_start, context_lens, d_status, workspace), out)


def test_decode_withheld_load(out, query, k_cache, v_cache, block_tables, context_lens, max_context_len, scale,
                              withheld_block, wait_limit_us, partition_size=0, workspace=None, d_status=None,
                              stream=None):
    """Fault injection for tests: ``paged_attention_decode`` with the load of
    logical block ``withheld_block`` of sequence 0, kv head 0 withheld and every
    wait limited to ``wait_limit_us``; the kernel must end with the timeout bit
    in ``d_status``."""
    desc = cache_desc(k_cache)
    _same_pool(k_cache, v_cache)
    S, Hq, D = query.shape
    if out.shape != query.shape or out.dtype != k_cache.dtype or query.dtype != k_cache.dtype:
        raise ValueError("query/out must be [S, Hq, head_dim] in the cache dtype")
    workspace, ws_bytes = _workspace(workspace, S, Hq, desc, D, max_context_len, partition_size, query.device)
    st = library().pkv_test_decode_withheld_load(
        _ptr(out), _ptr(query), _ptr(k_cache), _ptr(v_cache), desc, _ptr(block_tables), block_tables.shape[1],
        _ptr(context_lens), S, Hq, int(max_context_len), float(scale), int(partition_size), _ptr(workspace),
        ws_bytes, int(withheld_block), int(wait_limit_us), _ptr(d_status), _stream(stream, query.device))
    _check(st, "pkv_test_decode_withheld_load")
    return out


# Workspace of pkv_paged_prefill's dynamic item order (PKV_PREFILL_WORKSPACE_BYTES).
PREFILL_WORKSPACE_BYTES = 16

# Capacity of the library's built-in split-K scratch (PKV_NOALLOC_SCRATCH_BYTES).
NOALLOC_SCRATCH_BYTES = 32 * 1024 * 1024


def paged_attention_decode_noalloc(out, query, k_cache, v_cache, block_tables, context_lens,
                                   max_context_len, scale, partition_size=0, d_status=None, stream=None):
    """Decode attention that allocates nothing, neither here nor in the library.

    For callers that cannot allocate device memory (their memory is all
    reserved up front, or they cannot afford cudaMalloc's device-wide
    synchronisation): the split-K scratch is the library's built-in buffer of
    ``NOALLOC_SCRATCH_BYTES`` per device.  Sizes that need more raise
    ``PkvError`` (PKV_ERR_TOO_LARGE); calls that overlap on the GPU race on
    the shared buffer.  Same arguments and result as ``paged_attention_decode``
    without ``workspace``.
    """
    desc = cache_desc(k_cache)
    _same_pool(k_cache, v_cache)
    S, Hq, D = query.shape
    if out.shape != query.shape or out.dtype != k_cache.dtype or query.dtype != k_cache.dtype:
        raise ValueError("query/out must be [S, Hq, head_dim] in the cache dtype")
    if not (query.is_contiguous() and out.is_contiguous()):
        raise ValueError("query/out must be contiguous")
    if block_tables.dtype != torch.int32 or block_tables.dim() != 2 or block_tables.shape[0] != S \
            or not block_tables.is_contiguous():
        raise ValueError("block_tables must be a contiguous int32 [S, max_blocks_per_seq] tensor")
    if context_lens.dtype != torch.int32 or context_lens.numel() != S or not context_lens.is_contiguous():
        raise ValueError("context_lens must be a contiguous int32 [S] tensor")
    st = library().pkv_paged_attention_decode_noalloc(
        _ptr(out), _ptr(query), _ptr(k_cache), _ptr(v_cache), desc, _ptr(block_tables),
        block_tables.shape[1], _ptr(context_lens), S, Hq, int(max_context_len), float(scale),
        int(partition_size), _ptr(d_status), _stream(stream, query.device))
    if st == ERR_TOO_LARGE:
        need = workspace_size(S, Hq, desc.num_kv_heads, D, desc.block_size, max_context_len, partition_size)
        if need > NOALLOC_SCRATCH_BYTES:
            raise PkvError(st, f"pkv_paged_attention_decode_noalloc: these sizes need {need} bytes of split-K "
                               f"scratch, more than the built-in {NOALLOC_SCRATCH_BYTES}")
    _check(st, "pkv_paged_attention_decode_noalloc")
    return out


def fp8_cache_desc(k_cache: torch.Tensor, v_cache: torch.Tensor) -> CacheDesc:
    """Descriptor of 8-bit pools: K ``[N, Hkv, B, D]``, V ``[N, Hkv, D, B]`` of
    E4M3 codes (``torch.uint8`` or ``torch.float8_e4m3fn``)."""
    if k_cache.dtype not in _FP8_DTYPES or v_cache.dtype not in _FP8_DTYPES:
        raise TypeError("8-bit pools must be torch.uint8 or torch.float8_e4m3fn")
    if k_cache.dim() != 4 or not (k_cache.is_contiguous() and v_cache.is_contiguous()):
        raise ValueError("8-bit pools must be contiguous 4-d tensors")
    N, Hkv, B, D = k_cache.shape
    if tuple(v_cache.shape) != (N, Hkv, D, B):
        raise ValueError("v_cache must be [num_blocks, num_kv_heads, head_dim, block_size]")
    return CacheDesc(N, B, Hkv, D, PKV_FP8_E4M3)


def reshape_and_cache_fp8(key, value, k_cache, v_cache, slot_mapping, k_scale, v_scale, d_status=None,
                          stream=None, prepare=False):
    """Quantising write of new tokens ``key/value [T, Hkv, D]`` (fp16/bf16) into
    8-bit pools: codes e4m3(x / scale)."""
    desc = fp8_cache_desc(k_cache, v_cache)
    T = key.shape[0]
    for t in (key, value):
        if t.dim() != 3 or tuple(t.shape[1:]) != (desc.num_kv_heads, desc.head_dim) or t.dtype not in _DTYPES:
            raise ValueError("key/value must be fp16/bf16 [T, num_kv_heads, head_dim]")
        if t.stride(2) != 1 or t.stride(1) != t.shape[2]:
            raise ValueError("key/value heads and dims must be contiguous within a token")
    if value.dtype != key.dtype:
        raise ValueError("key and value must have the same dtype")
    if slot_mapping.dtype != torch.int64 or slot_mapping.numel() != T or not slot_mapping.is_contiguous():
        raise ValueError("slot_mapping must be a contiguous int64 tensor with one entry per token")
    return _invoke(library().pkv_reshape_and_cache_fp8,
                   (_ptr(key), _ptr(value), key.stride(0), value.stride(0), _DTYPES[key.dtype], _ptr(k_cache),
                    _ptr(v_cache), desc, _ptr(slot_mapping), T, float(k_scale), float(v_scale), _ptr(d_status),
                    _stream(stream, k_cache.device)),
                   "pkv_reshape_and_cache_fp8", prepare, (key, value, k_cache, v_cache, slot_mapping, d_status))


def paged_attention_decode_fp8(out, query, k_cache, v_cache, block_tables, context_lens, max_context_len,
                               scale, k_scale, v_scale, partition_size=0, workspace=None, d_status=None,
                               stream=None, prepare=False):
    """Decode attention over 8-bit pools (K, V read back as code * scale);
    query/out fp16 or bf16 ``[S, Hq, D]``."""
    desc = fp8_cache_desc(k_cache, v_cache)
    S, Hq, D = query.shape
    if query.dtype not in _DTYPES or out.dtype != query.dtype or out.shape != query.shape:
        raise ValueError("query/out must be fp16/bf16 [S, Hq, head_dim] of one dtype")
    if not (query.is_contiguous() and out.is_contiguous()):
        raise ValueError("query/out must be contiguous")
    if block_tables.dtype != torch.int32 or block_tables.dim() != 2 or block_tables.shape[0] != S \
            or not block_tables.is_contiguous():
        raise ValueError("block_tables must be a contiguous int32 [S, max_blocks_per_seq] tensor")
    if context_lens.dtype != torch.int32 or context_lens.numel() != S or not context_lens.is_contiguous():
        raise ValueError("context_lens must be a contiguous int32 [S] tensor")
    workspace, ws_bytes = _workspace(workspace, S, Hq, desc, D, max_context_len, partition_size, query.device)
    return _invoke(library().pkv_paged_attention_decode_fp8,
                   (_ptr(out), _ptr(query), _DTYPES[query.dtype], _ptr(k_cache), _ptr(v_cache), desc,
                    _ptr(block_tables), block_tables.shape[1], _ptr(context_lens), S, Hq, int(max_context_len),
                    float(scale), float(k_scale), float(v_scale), int(partition_size), _ptr(workspace), ws_bytes,
                    _ptr(d_status), _stream(stream, query.device)),
                   "pkv_paged_attention_decode_fp8", prepare,
                   (out, query, k_cache, v_cache, block_tables, context_lens, workspace, d_status), out)


def copy_blocks(k_cache, v_cache, block_pairs, d_status=None, stream=None, prepare=False):
    """Copy-on-write: block ``pairs[i, 1]`` of both pools becomes a copy of
    ``pairs[i, 0]`` (fp16/bf16 pools, or 8-bit pools)."""
    if k_cache.dtype in _FP8_DTYPES:
        desc = fp8_cache_desc(k_cache, v_cache)
    else:
        desc = cache_desc(k_cache)
        _same_pool(k_cache, v_cache)
    if block_pairs.dtype != torch.int64 or block_pairs.dim() != 2 or block_pairs.shape[1] != 2 \
            or not block_pairs.is_contiguous():
        raise ValueError("block_pairs must be a contiguous int64 [num_pairs, 2] tensor")
    return _invoke(library().pkv_copy_blocks,
                   (_ptr(k_cache), _ptr(v_cache), desc, _ptr(block_pairs), block_pairs.shape[0], _ptr(d_status),
                    _stream(stream, k_cache.device)),
                   "pkv_copy_blocks", prepare, (k_cache, v_cache, block_pairs, d_status))


def version() -> int:
    return int(library().pkv_version())
