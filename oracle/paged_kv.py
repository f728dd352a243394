"""Oracle for paged-KV decode: plain, slow, float64, CPU only.

TEST INFRASTRUCTURE ONLY.  Imported by ``tests/``, by ``__graft_entry__.smoke()``
and by the CPU-baseline leg of ``bench.py``; the library path never imports it,
and it imports nothing from the CUDA package.  Every result the CUDA kernels
produce is checked against these functions.

Sources (web pages describing vLLM's PagedAttention):

* [LSHU] lshu.cn/news/11644, vLLM architecture analysis, section
  "核心创新：PagedAttention 的设计逻辑": sub-sections "方案：页式内存管理"
  (fixed 16-token blocks, per-request Block Table, the append rule, the kernel
  reading scattered blocks through the table as one logical sequence),
  "收益分析" (blocks returned to the free pool when a request finishes) and
  "内存共享" (shared prefix blocks are read-only; a divergence is handled by
  copy-on-write).
* [ZZM] zzmblog.top, "vLLM使用指南", section "核心原理 / Transformer推理与KV缓存":
  a decode step computes only the current token's K, V, appends them to the
  cache and then computes attention.
* Scaled dot-product attention with a softmax over the context is the textbook
  definition; the pages name attention but do not print the formula.

Numerics: fp16/bf16 inputs are decoded exactly to float64; all arithmetic is
float64.  Nothing here is blocked, fused, partitioned or reordered.
"""

from __future__ import annotations

import numpy as np

F16 = "f16"
BF16 = "bf16"


# ---------------------------------------------------------------------------
# Storage formats
# ---------------------------------------------------------------------------

def decode_bits(bits: np.ndarray, dtype: str) -> np.ndarray:
    """Exact float64 value of fp16 / bf16 bit patterns."""
    bits = np.asarray(bits, dtype=np.uint16)
    if dtype == F16:
        return bits.view(np.float16).astype(np.float64)
    if dtype == BF16:
        return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    raise ValueError(dtype)


def encode_bits(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round float64 values to the nearest fp16 / bf16 (ties to even).

    Used only to report how far the exact result is from its own storage
    rounding (the floor any fp16/bf16 output can reach).
    """
    x = np.asarray(x, dtype=np.float64)
    if dtype == F16:
        return x.astype(np.float16).view(np.uint16)
    if dtype == BF16:
        # 8 significant bits: x = m * 2**e with 0.5 <= |m| < 1.
        m, e = np.frexp(x)
        r = np.ldexp(np.rint(np.ldexp(m, 8)), e - 8)  # exact in float32
        return (r.astype(np.float32).view(np.uint32) >> np.uint32(16)).astype(np.uint16)
    raise ValueError(dtype)


# ---------------------------------------------------------------------------
# Block table and slots ([LSHU] 方案：页式内存管理)
# ---------------------------------------------------------------------------

def slot_location(slot: int, block_size: int) -> tuple[int, int]:
    """A slot number names (physical block, position inside the block)."""
    return int(slot) // block_size, int(slot) % block_size


def append_token(table: list, length: int, free_pool: list, block_size: int) -> int:
    """The append rule: a request that grows by one token puts it in its last
    block if that block holds fewer than ``block_size`` tokens; otherwise a
    block is taken from the free pool and appended to the Block Table.
    Returns the slot of the new token (token index ``length``)."""
    if length % block_size == 0:  # no block yet, or the last one is full
        table.append(free_pool.pop(0))
    return table[-1] * block_size + length % block_size


def free_request(table: list, free_pool: list) -> None:
    """A finished request returns every block of its Block Table to the pool
    at once ([LSHU] 收益分析: 即时回收)."""
    free_pool.extend(table)
    table.clear()


def materialize(cache_bits: np.ndarray, table_row: np.ndarray, length: int, block_size: int) -> np.ndarray:
    """Read a sequence's scattered blocks through its Block Table and return
    the logically contiguous sequence ``[Hkv, length, D]`` (bits).

    Token ``i`` lives in physical block ``table_row[i // block_size]`` at
    position ``i % block_size``.  Table entries past the last used block are
    never read.
    """
    pos = np.arange(length)
    blocks = np.asarray(table_row)[pos // block_size].astype(np.int64)
    offs = pos % block_size
    tok = cache_bits[blocks, :, offs, :]  # [length, Hkv, D]
    return np.ascontiguousarray(tok.transpose(1, 0, 2))


# ---------------------------------------------------------------------------
# Cache write and block copy
# ---------------------------------------------------------------------------

def reshape_and_cache(k_cache, v_cache, key, value, slot_mapping, block_size):
    """Write each new token's K and V (all kv heads) into the slot named by
    ``slot_mapping``; a negative slot is padding and writes nothing.

    ([ZZM]: the decode step appends the current token's K, V to the cache;
    [LSHU] 方案: the token goes into a slot of a block of its table.)
    Returns updated copies; the inputs are left unchanged.
    """
    kc = np.array(k_cache, copy=True)
    vc = np.array(v_cache, copy=True)
    for t, slot in enumerate(np.asarray(slot_mapping).tolist()):
        if slot < 0:
            continue
        b, o = slot_location(slot, block_size)
        kc[b, :, o, :] = key[t]
        vc[b, :, o, :] = value[t]
    return kc, vc


def copy_blocks(k_cache, v_cache, block_pairs):
    """Copy-on-write: for every (src, dst) pair the whole physical block dst
    (every kv head, every slot) becomes a copy of block src, in both the K and
    the V pool ([LSHU] 内存共享).  All pairs read the state before the call.
    Returns updated copies."""
    k0 = np.array(k_cache, copy=True)
    v0 = np.array(v_cache, copy=True)
    kc, vc = k0.copy(), v0.copy()
    for src, dst in np.asarray(block_pairs, dtype=np.int64).reshape(-1, 2).tolist():
        kc[dst] = k0[src]
        vc[dst] = v0[src]
    return kc, vc


# ---------------------------------------------------------------------------
# Attention
# ---------------------------------------------------------------------------

def attend(q: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float) -> np.ndarray:
    """Textbook softmax attention of query rows ``q [G, D]`` over one
    contiguous key/value sequence ``K, V [L, D]`` (float64).

    z_i = scale * <q, K_i>;  p = softmax(z) (max subtracted);  out = sum_i p_i V_i.
    An empty sequence gives a zero output.
    """
    q = np.asarray(q, dtype=np.float64)
    if K.shape[0] == 0:
        return np.zeros((q.shape[0], V.shape[1]), dtype=np.float64)
    z = scale * (q @ K.T)  # [G, L]
    z = z - z.max(axis=1, keepdims=True)
    e = np.exp(z)
    p = e / e.sum(axis=1, keepdims=True)
    return p @ V


def kv_head_of(h: int, num_q_heads: int, num_kv_heads: int) -> int:
    """Query head h reads kv head h // (Hq / Hkv): consecutive query heads form
    a group sharing one kv head (plain grouped-query reading; Hq = Hkv is
    multi-head attention)."""
    return h // (num_q_heads // num_kv_heads)


def decode_sequence(q_bits_s, k_cache, v_cache, table_row, length, block_size, scale, dtype,
                    kv_heads=None) -> np.ndarray:
    """Decode attention for one sequence: materialise its K/V through the
    Block Table ([LSHU] 方案: Kernel 根据每个请求的 Block Table 读取离散的 Block
    拼成逻辑上连续的 Key/Value 序列), then attend.  Returns ``[Hq, D]`` float64;
    query heads whose kv head is not in ``kv_heads`` are left as NaN."""
    Hq, D = q_bits_s.shape
    Hkv = k_cache.shape[1]
    G = Hq // Hkv
    out = np.full((Hq, D), np.nan)
    q = decode_bits(q_bits_s, dtype)
    heads = range(Hkv) if kv_heads is None else kv_heads
    Kall = materialize(k_cache, table_row, length, block_size)
    Vall = materialize(v_cache, table_row, length, block_size)
    for g in heads:
        K = decode_bits(Kall[g], dtype)
        V = decode_bits(Vall[g], dtype)
        rows = [h for h in range(Hq) if kv_head_of(h, Hq, Hkv) == g]
        out[rows] = attend(q[rows], K, V, scale)
    return out


def paged_attention_decode(q_bits, k_cache, v_cache, block_tables, context_lens, block_size,
                           scale, dtype, seqs=None) -> np.ndarray:
    """Decode attention for every sequence (or the listed ones).

    ``q_bits [S, Hq, D]``, caches ``[N, Hkv, B, D]`` (bits), ``block_tables
    [S, max_blocks]``, ``context_lens [S]``.  Returns float64 ``[S, Hq, D]``;
    rows of sequences not listed in ``seqs`` are NaN.
    """
    S, Hq, D = q_bits.shape
    out = np.full((S, Hq, D), np.nan)
    for s in (range(S) if seqs is None else seqs):
        out[s] = decode_sequence(q_bits[s], k_cache, v_cache, block_tables[s], int(context_lens[s]),
                                 block_size, scale, dtype)
    return out


# ---------------------------------------------------------------------------
# Split-K partial states and their log-sum-exp combine
# ---------------------------------------------------------------------------

def partial_state(q: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float):
    """Unnormalised softmax state of query rows ``q [G, D]`` over one slice of
    the context: m = max_i z_i, l = sum_i exp(z_i - m), o = sum_i exp(z_i - m) V_i.
    An empty slice gives m = -inf, l = 0, o = 0."""
    G, D = q.shape[0], V.shape[1]
    if K.shape[0] == 0:
        return np.full(G, -np.inf), np.zeros(G), np.zeros((G, D))
    z = scale * (q @ K.T)
    m = z.max(axis=1)
    e = np.exp(z - m[:, None])
    return m, e.sum(axis=1), e @ V


def lse_combine(ms: np.ndarray, ls: np.ndarray, os: np.ndarray) -> np.ndarray:
    """Merge partial states ``m [P, G]``, ``l [P, G]``, ``o [P, G, D]`` of
    disjoint slices into the softmax attention over their union:
    M = max_p m_p, w_p = exp(m_p - M), out = sum_p w_p o_p / sum_p w_p l_p.
    An all-empty input gives zeros."""
    ms = np.asarray(ms, dtype=np.float64)
    M = ms.max(axis=0)
    out = np.zeros(os.shape[1:])
    live = np.isfinite(M)
    if not live.any():
        return out
    w = np.where(np.isfinite(ms), np.exp(ms - np.where(live, M, 0.0)[None, :]), 0.0)
    num = (w[:, :, None] * os).sum(axis=0)
    den = (w * ls).sum(axis=0)
    out[live] = num[live] / den[live][:, None]
    return out


# ---------------------------------------------------------------------------
# 8-bit KV cache (E4M3)
# ---------------------------------------------------------------------------
# lshu.cn/news/11644, "性能关键路径与瓶颈": quantising the KV cache to FP8/INT8
# halves the bytes decode must read.  Format (OCP 8-bit floating point, E4M3):
# 1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits; exponent field 0
# holds subnormals m * 2^-9; there is no infinity; S.1111.111 is NaN, so the
# largest finite magnitude is 1.75 * 2^8 = 448.  Values are stored as
# e4m3(x / scale) with one fp32 scale per pool, rounded to nearest (ties to
# even) and saturated to +-448; they read back as e4m3 * scale.
# Pool layouts: K as [N][Hkv][B][D] (one row of D codes per token), V as
# [N][Hkv][D][B] (one row of B codes per dimension).

E4M3_MAX = 448.0


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """Exact float64 value of E4M3 codes (NaN for S.1111.111)."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    mag = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.ldexp(1.0, e - 7))
    mag = np.where((e == 0xF) & (m == 7), np.nan, mag)
    return sign * mag


def e4m3_encode(x: np.ndarray) -> np.ndarray:
    """Round values to the nearest E4M3 code (ties to even), saturating
    magnitudes above 448 to 448; NaN maps to 0x7F."""
    x = np.asarray(x, dtype=np.float64)
    sign = np.signbit(x)
    a = np.abs(x)
    nan = np.isnan(a)
    a = np.where(nan, 0.0, a)
    # quantum of the binade: 2^(e-3) for normals (e >= -6), 2^-9 below
    _, ex = np.frexp(a)  # a = f * 2^ex, 0.5 <= f < 1  ->  floor(log2 a) = ex - 1
    e = np.maximum(ex - 1, -6)
    quantum = np.ldexp(1.0, e - 3)
    q = np.rint(a / quantum) * quantum  # np.rint rounds half to even
    q = np.minimum(q, E4M3_MAX)
    # encode the (exactly representable) rounded magnitude
    _, ex2 = np.frexp(q)
    e2 = ex2 - 1
    normal = q >= 2.0 ** -6
    exp_field = np.where(normal, e2 + 7, 0)
    mant = np.where(normal, np.rint((q / np.ldexp(1.0, e2) - 1.0) * 8.0), np.rint(q / 2.0 ** -9))
    code = (exp_field.astype(np.int64) << 3) | mant.astype(np.int64)
    code = np.where(q == 0.0, 0, code)
    code = code | np.where(sign, 0x80, 0)
    code = np.where(nan, 0x7F, code)
    return code.astype(np.uint8)


def quantize_e4m3(x_bits: np.ndarray, dtype: str, scale: float) -> np.ndarray:
    """Codes stored for fp16/bf16 values x: e4m3(fp32(x) / fp32(scale)), the
    division done once in IEEE fp32 (round to nearest)."""
    x32 = decode_bits(x_bits, dtype).astype(np.float32)
    return e4m3_encode((x32 / np.float32(scale)).astype(np.float64))


def reshape_and_cache_fp8(k_cache, v_cache, key, value, slot_mapping, block_size, k_scale, v_scale,
                          dtype):
    """Quantising cache write: for t with slot p >= 0, K codes of token t go to
    k_cache[p // B][h][p % B][:] and V codes to v_cache[p // B][h][:][p % B].
    Returns updated copies."""
    kc = np.array(k_cache, copy=True)
    vc = np.array(v_cache, copy=True)
    kq = quantize_e4m3(key, dtype, k_scale)
    vq = quantize_e4m3(value, dtype, v_scale)
    for t, slot in enumerate(np.asarray(slot_mapping).tolist()):
        if slot < 0:
            continue
        b, o = slot_location(slot, block_size)
        kc[b, :, o, :] = kq[t]
        vc[b, :, :, o] = vq[t]
    return kc, vc


def materialize_fp8(k_cache, v_cache, table_row, length, block_size):
    """Contiguous K, V codes [Hkv, length, D] of one sequence from the 8-bit
    pools (V pool stored with dimensions before token positions)."""
    pos = np.arange(length)
    blocks = np.asarray(table_row)[pos // block_size].astype(np.int64)
    offs = pos % block_size
    K = k_cache[blocks, :, offs, :]  # [L, Hkv, D]
    V = v_cache[blocks, :, :, offs]  # [L, Hkv, D]
    return np.ascontiguousarray(K.transpose(1, 0, 2)), np.ascontiguousarray(V.transpose(1, 0, 2))


def paged_attention_decode_fp8(q_bits, k_cache, v_cache, block_tables, context_lens, block_size, scale,
                               k_scale, v_scale, dtype, seqs=None) -> np.ndarray:
    """Decode attention over 8-bit pools: K and V read back as code * scale
    (exactly, in float64), then textbook softmax attention."""
    S, Hq, D = q_bits.shape
    Hkv = k_cache.shape[1]
    out = np.full((S, Hq, D), np.nan)
    for s in (range(S) if seqs is None else seqs):
        L = int(context_lens[s])
        q = decode_bits(q_bits[s], dtype)
        Kc, Vc = materialize_fp8(k_cache, v_cache, block_tables[s], L, block_size)
        for g in range(Hkv):
            rows = [h for h in range(Hq) if kv_head_of(h, Hq, Hkv) == g]
            K = e4m3_decode(Kc[g]) * k_scale
            V = e4m3_decode(Vc[g]) * v_scale
            out[s, rows] = attend(q[rows], K, V, scale)
    return out
