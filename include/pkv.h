/*
 * pkv.h - C ABI of libpkv: the decode hot path of a paged KV cache on B200 (sm_100a).
 *
 * The KV cache of every attention layer is a pool of fixed-size physical
 * blocks; each sequence reaches its tokens through its own Block Table, which
 * maps logical block j (tokens j*B .. j*B+B-1) to a physical block id.  Sources:
 *   lshu.cn/news/11644 (vLLM architecture analysis), section
 *   "核心创新：PagedAttention 的设计逻辑": sub-section "方案：页式内存管理"
 *   (blocks of 16 tokens, Block Table per request, append rule, the attention
 *   kernel reading the scattered blocks through the table as one logical K/V
 *   sequence) and "内存共享" (prefix blocks shared read-only, copy-on-write on
 *   divergence); zzmblog.top "vLLM使用指南", section "核心原理 / Transformer推理
 *   与KV缓存" (a decode step computes only the current token's K and V, appends
 *   them to the cache, then computes attention).
 *
 * Conventions shared by every entry point
 *   - Pointers named d_* or described as device memory are device pointers
 *     owned by the caller.  The library allocates nothing and frees nothing.
 *   - Every compute call is asynchronous on `stream` (a cudaStream_t; NULL is
 *     the legacy default stream) and returns once its kernels are queued.
 *   - Host-detectable errors return a non-zero pkv_status before anything is
 *     queued; outputs are then untouched.
 *   - Errors that only the device can see (a block id outside the pool, a slot
 *     outside the pool, a context length the call's bounds cannot hold, a wait
 *     that ran out) are OR-ed as PKV_DEV_* bits into *d_status when d_status is
 *     not NULL (an int32 in device memory, to be read after the stream
 *     synchronises; the library never clears it).  Kernels never trap: an
 *     offending element is skipped or masked and the flag is raised.
 *   - Mutable global state is limited to caches filled on first use (the
 *     driver's tensor-map encoder; per device, its compute capability and each
 *     kernel's shared-memory limit; per host thread, recently encoded tensor
 *     maps) and the built-in scratch of pkv_paged_attention_decode_noalloc.
 *     The caches are atomic or per thread, so calls are thread-safe.
 *   - Calls can be captured in a CUDA graph (stream capture): they allocate
 *     nothing, never synchronise and queue only kernels (launched with
 *     programmatic dependent launch) plus at most one cudaMemsetAsync.  Make
 *     one call of each entry point per device before capturing, so that the
 *     first-use set-up above happens outside the capture.  A captured call
 *     keeps the pointers, sizes and max_context_len it was captured with; the
 *     contents of the device arrays (inputs, lengths, tables, slots) may
 *     change between replays.
 *   - Check build (PKV_CHECK).  The same sources compiled with PKV_CHECK
 *     defined give libpkv_check.so (`python -m paged_kv_cache_407_b200.build
 *     --check`), a debugging build that also verifies the caller guarantees
 *     the kernels cannot see cheaply: no slot repeats in one cache write, no
 *     copy destination repeats or is also a source.  Those calls then copy
 *     the index array to the host and synchronise the stream before queuing
 *     anything, so a check build cannot be captured in a CUDA graph (the call
 *     returns PKV_ERR_CUDA while its stream is capturing, PKV_ERR_TOO_LARGE
 *     when the host copy cannot be allocated).  pkv_check_build() tells the
 *     two builds apart.
 *
 * Cache layout ("HND"): k_cache and v_cache are separate pools, each
 *   [num_blocks][num_kv_heads][block_size][head_dim] row-major, element type
 *   fp16 or bf16.  Slot s names block s / block_size, position s % block_size.
 */
#ifndef PKV_H_
#define PKV_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define PKV_API __attribute__((visibility("default")))
#else
#define PKV_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *pkv_stream_t; /* same handle as cudaStream_t */

typedef enum {
  PKV_OK = 0,
  PKV_ERR_NULL_POINTER = 1,   /* a required pointer is NULL */
  PKV_ERR_BAD_DTYPE = 2,      /* dtype is not PKV_F16 / PKV_BF16 */
  PKV_ERR_BAD_SHAPE = 3,      /* unsupported head_dim / block_size / head counts / negative size */
  PKV_ERR_MISALIGNED = 4,     /* a pointer or stride breaks the stated alignment */
  PKV_ERR_WORKSPACE = 5,      /* workspace NULL or smaller than pkv_paged_attention_workspace_size
                                 (pkv_paged_prefill: smaller than PKV_PREFILL_WORKSPACE_BYTES) */
  PKV_ERR_BAD_PARTITION = 6,  /* partition_size not a positive multiple of block_size */
  PKV_ERR_TOO_LARGE = 7,      /* a size exceeds what the kernels index (see each call) */
  PKV_ERR_CUDA = 8,           /* a CUDA runtime/driver call failed (launch, attribute, tensor map) */
  PKV_ERR_DEVICE = 9,         /* current device is not compute capability 10.0 (B200 / sm_100a) */
  PKV_ERR_NO_BLOCKS = 10,     /* block manager: the free pool cannot supply the blocks asked for */
  PKV_ERR_BAD_SEQUENCE = 11,  /* block manager: unknown, repeated or already present sequence id */
  PKV_ERR_ALIAS = 12          /* check build only: a slot repeats within one cache write, or a
                                 copy pair's dst repeats or is also a src (see PKV_CHECK below) */
} pkv_status;

/* Device-side error bits OR-ed into *d_status. */
#define PKV_DEV_BAD_BLOCK 0x1  /* a Block Table entry or copy pair outside [0, num_blocks) */
#define PKV_DEV_BAD_SLOT 0x2   /* a slot >= num_blocks * block_size */
#define PKV_DEV_BAD_LEN 0x4    /* context_len < 0, > max_context_len or > max_blocks_per_seq * block_size */
#define PKV_DEV_TIMEOUT 0x8    /* a copy into shared memory did not complete within its limit (~1 s) */

typedef enum { PKV_F16 = 0, PKV_BF16 = 1, PKV_FP8_E4M3 = 2 } pkv_dtype;

/* Shape of one layer's block pool (shared by k_cache and v_cache). */
typedef struct {
  int32_t num_blocks;   /* N >= 1 */
  int32_t block_size;   /* B: tokens per block; 8, 16, 32 or 64 */
  int32_t num_kv_heads; /* Hkv >= 1 */
  int32_t head_dim;     /* D: 64 or 128 */
  pkv_dtype dtype;      /* element type of both pools (and, for fp16/bf16 pools,
                           of queries and outputs) */
} pkv_cache_desc;

/*
 * 8-bit pools (dtype PKV_FP8_E4M3).  Source: lshu.cn/news/11644, "性能关键路径
 * 与瓶颈": quantising the KV cache to FP8/INT8 is the most effective decode
 * optimisation, halving the bytes read.  Codes are OCP E4M3 (1 sign, 4
 * exponent bits with bias 7, 3 mantissa bits, subnormals, no infinity, largest
 * finite 448).  A value x is stored as e4m3(x / scale), the division done in
 * IEEE fp32 and the result rounded to nearest even and saturated to +-448;
 * it reads back as code * scale, with one fp32 scale per pool (k_scale,
 * v_scale).  Layouts: k_cache [num_blocks][num_kv_heads][block_size][head_dim]
 * (one row of head_dim codes per token) and v_cache
 * [num_blocks][num_kv_heads][head_dim][block_size] (one row of block_size
 * codes per dimension).  Supported: head_dim 128, block_size 16, 32 or 64.
 * pkv_copy_blocks works on 8-bit pools as on fp16/bf16 ones.
 */

/*
 * pkv_reshape_and_cache - write this step's new K/V tokens into their slots.
 *
 * Passage: the append rule of lshu.cn/news/11644 "方案：页式内存管理" (a new
 * token goes into the next free position of the sequence's last block, or of a
 * block newly taken from the free pool) together with zzmblog.top
 * "Transformer推理与KV缓存" (the step's K, V are appended before attention).
 * The host decides the slots; this call performs the writes:
 *   for t < num_tokens with p = slot_mapping[t] >= 0, for every kv head h:
 *     k_cache[p / B][h][p % B][:] = key[t][h][:]   and the same for value.
 * A negative slot marks a padding token and writes nothing.  Plain bit copy.
 *
 * key, value      device, [num_tokens][num_kv_heads][head_dim] with a token
 *                 stride of key_token_stride / value_token_stride elements
 *                 (0 means num_kv_heads*head_dim); heads of a token contiguous.
 * k_cache,v_cache device, layout above, 16-byte aligned.
 * slot_mapping    device, int64 [num_tokens].
 * Errors: NULL pointers (when num_tokens > 0), bad desc or 8-bit pools
 *   -> status; a slot >= num_blocks*B -> PKV_DEV_BAD_SLOT, that token skipped.
 *   Two tokens with the same slot in one call race (caller error, result
 *   unspecified); a check build returns PKV_ERR_ALIAS instead, before
 *   writing anything (negative slots may repeat).
 */
PKV_API pkv_status pkv_reshape_and_cache(const void *key, const void *value, int64_t key_token_stride,
                                 int64_t value_token_stride, void *k_cache, void *v_cache,
                                 pkv_cache_desc cache, const int64_t *slot_mapping,
                                 int32_t num_tokens, int32_t *d_status, pkv_stream_t stream);

/*
 * pkv_paged_attention_workspace_size - bytes of scratch that
 * pkv_paged_attention_decode needs for these sizes: 0 when no sequence can
 * span more than one partition; otherwise num_seqs * num_kv_heads int32
 * arrival counters and one int32 unit count (padded to 16 bytes), the plan's
 * list of num_seqs * max_partitions (sequence, partition) int32 pairs
 * (padded to 16 bytes), then num_seqs * num_q_heads * max_partitions *
 * (head_dim + 2) floats of partials.  partition_size follows the rules of
 * pkv_paged_attention_decode (0 = automatic).  Returns 0 for invalid sizes.
 */
PKV_API size_t pkv_paged_attention_workspace_size(int32_t num_seqs, int32_t num_q_heads,
                                          int32_t num_kv_heads, int32_t head_dim,
                                          int32_t block_size, int32_t max_context_len,
                                          int32_t partition_size);

/*
 * pkv_paged_attention_partition_size - the partition size (tokens) that
 * pkv_paged_attention_decode uses for these arguments: partition_size itself
 * when it is non-zero, otherwise the automatic choice: no split (the result
 * covers max_context_len) when max_context_len <= 2048 and num_seqs *
 * num_kv_heads >= 1776 (about 12 work units per SM); else 1024 tokens,
 * halved down to 256 while num_seqs * num_kv_heads * ceil(max_context_len /
 * size) stays below 1776.  Returns -1 for invalid arguments.  A result >=
 * max_context_len means no sequence is split.
 */
PKV_API int32_t pkv_paged_attention_partition_size(int32_t num_seqs, int32_t num_kv_heads,
                                           int32_t block_size, int32_t max_context_len,
                                           int32_t partition_size);

/*
 * pkv_paged_attention_decode - single-token decode attention over the paged
 * cache.
 *
 * Passage: lshu.cn/news/11644 "方案：页式内存管理" - the attention kernel reads
 * each request's scattered blocks through its Block Table and treats them as
 * one logically contiguous K/V sequence; "性能关键路径与瓶颈" - decode time is
 * the KV bytes over memory bandwidth, and the kernel should keep table lookups
 * cheap.  The attention itself is textbook softmax attention:
 *   for sequence s, query head h, kv head g = h / (num_q_heads / num_kv_heads):
 *     z_i = scale * <query[s][h], K_s[g][i]>  for i < context_lens[s],
 *     out[s][h] = sum_i softmax(z)_i * V_s[g][i],
 *   where K_s[g][i] = k_cache[block_tables[s][i / B]][g][i % B] (same for V).
 * Long contexts are cut into partitions of partition_size tokens; each
 * partition yields (max score, sum of exponentials, unnormalised output) and
 * they are merged by log-sum-exp (by the last partition of each sequence to
 * finish, or by a second kernel for splits of more than 32 partitions).  A
 * call whose longest sequence spans 3 to 32 partitions first runs a one-CTA
 * planning kernel that lists the non-empty (sequence, partition) units,
 * largest first, so the attention grid starts the long units first.  Arithmetic: fp16/bf16 products, fp32 accumulation
 * and softmax; the output is rounded once to fp16/bf16.
 *
 * out              device, [num_seqs][num_q_heads][head_dim], cache dtype.
 * query            device, [num_seqs][num_q_heads][head_dim], cache dtype.
 * k_cache, v_cache device, 16-byte aligned, layout above.
 * block_tables     device, int32 [num_seqs][max_blocks_per_seq]; entries at
 *                  or past ceil(context_len / B) are never read.
 * context_lens     device, int32 [num_seqs]: tokens attended by each sequence
 *                  (including the one written this step); 0 gives a zero row.
 * max_context_len  host bound >= every context_lens[s]; it sizes the grid.
 * num_q_heads      multiple of num_kv_heads; num_q_heads / num_kv_heads <= 16.
 * scale            softmax scale (e.g. 1/sqrt(head_dim)), > 0.
 * partition_size   0 = automatic; otherwise a positive multiple of B.
 * workspace        device, >= pkv_paged_attention_workspace_size(...) bytes,
 *                  16-byte aligned; may be NULL when that size is 0.  Holds
 *                  one arrival counter per (sequence, kv head) and the split
 *                  partials; the call zeroes the counters itself (in its
 *                  planning kernel, else with an async memset on `stream`),
 *                  so no content is expected on entry.
 * Errors: host checks -> status.  A table entry outside [0, num_blocks) ->
 *   PKV_DEV_BAD_BLOCK and that block is treated as empty; a context length
 *   outside [0, min(max_context_len, max_blocks_per_seq*B)] -> PKV_DEV_BAD_LEN
 *   and the length is clamped into that range.
 */
PKV_API pkv_status pkv_paged_attention_decode(void *out, const void *query, const void *k_cache,
                                      const void *v_cache, pkv_cache_desc cache,
                                      const int32_t *block_tables, int32_t max_blocks_per_seq,
                                      const int32_t *context_lens, int32_t num_seqs,
                                      int32_t num_q_heads, int32_t max_context_len, float scale,
                                      int32_t partition_size, void *workspace,
                                      size_t workspace_bytes, int32_t *d_status,
                                      pkv_stream_t stream);

/*
 * pkv_copy_blocks - copy-on-write of shared blocks.
 *
 * Passage: lshu.cn/news/11644 "内存共享" - requests with the same prompt prefix
 * read the same physical blocks; a later divergence is handled by copying the
 * block before writing to it.  For every pair i, block block_pairs[2i+1] of
 * both pools becomes a bit copy of block block_pairs[2i] (every kv head, every
 * position).
 *
 * block_pairs  device, int64 [num_pairs][2] = (src, dst).
 * Errors: a src or dst outside [0, num_blocks) -> PKV_DEV_BAD_BLOCK and that
 *   pair is skipped.  A dst that repeats, or that is also a src in the same
 *   call (its own included), races (caller error, result unspecified); a
 *   check build returns PKV_ERR_ALIAS instead, before copying anything
 *   (pairs the kernel would skip are left out of that check).
 */
PKV_API pkv_status pkv_copy_blocks(void *k_cache, void *v_cache, pkv_cache_desc cache,
                           const int64_t *block_pairs, int32_t num_pairs, int32_t *d_status,
                           pkv_stream_t stream);

/*
 * pkv_paged_attention_decode_noalloc - pkv_paged_attention_decode without a
 * caller-supplied workspace.  No counterpart in the paper: it exists for callers
 * that cannot allocate device memory, such as a serving engine that has already
 * reserved all free device memory for its block pool, a C host without a device
 * allocator of its own, or a loop that cannot afford cudaMalloc's implicit
 * device-wide synchronisation.
 *
 * Arguments, layouts, results and device flags are those of
 * pkv_paged_attention_decode minus (workspace, workspace_bytes).  The split-K
 * scratch is a buffer of PKV_NOALLOC_SCRATCH_BYTES compiled into the library;
 * every GPU that loads the library holds it until the process exits.  This call
 * allocates nothing and frees nothing.
 *   - Limit: when pkv_paged_attention_workspace_size(...) for these sizes
 *     exceeds PKV_NOALLOC_SCRATCH_BYTES the call returns PKV_ERR_TOO_LARGE
 *     before anything is queued; use pkv_paged_attention_decode instead.
 *   - Every call looks up the buffer's device address on the current device
 *     (cudaGetSymbolAddress), so the address stays right after the device's
 *     context is reset.  The first call on each device also loads the
 *     library's device code there; make that first call before any stream
 *     capture.
 *   - All calls on a device share the one buffer and it keeps the last call's
 *     contents.  The call clears the part that must start at zero (the split
 *     arrival counters) and writes every partial before reading it, but two
 *     calls whose kernels overlap on the GPU (for example on two streams) race
 *     on it.
 */
#define PKV_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)
PKV_API pkv_status pkv_paged_attention_decode_noalloc(
    void *out, const void *query, const void *k_cache, const void *v_cache, pkv_cache_desc cache,
    const int32_t *block_tables, int32_t max_blocks_per_seq, const int32_t *context_lens,
    int32_t num_seqs, int32_t num_q_heads, int32_t max_context_len, float scale,
    int32_t partition_size, int32_t *d_status, pkv_stream_t stream);

/*
 * pkv_reshape_and_cache_fp8 - pkv_reshape_and_cache into 8-bit pools: every
 * new K and V value is quantised as described above, K codes go to
 * k_cache[p / B][h][p % B][:] and V codes to v_cache[p / B][h][:][p % B].
 * key, value: fp16 or bf16 (input_dtype), same layout and strides as
 * pkv_reshape_and_cache; cache.dtype must be PKV_FP8_E4M3; k_scale, v_scale > 0.
 * Errors as pkv_reshape_and_cache (PKV_ERR_ALIAS included).
 */
PKV_API pkv_status pkv_reshape_and_cache_fp8(const void *key, const void *value,
                                             int64_t key_token_stride, int64_t value_token_stride,
                                             pkv_dtype input_dtype, void *k_cache, void *v_cache,
                                             pkv_cache_desc cache, const int64_t *slot_mapping,
                                             int32_t num_tokens, float k_scale, float v_scale,
                                             int32_t *d_status, pkv_stream_t stream);

/*
 * pkv_paged_attention_decode_fp8 - pkv_paged_attention_decode over 8-bit
 * pools: K and V read back as code * k_scale and code * v_scale.  query and
 * out are fp16 or bf16 (query_dtype); the products run on fp16 operands
 * (E4M3 codes are exact in fp16; bf16 queries are converted to fp16, exact
 * for zero and magnitudes in [2^-14, 65504], rounded to fp16 subnormals below
 * that) with fp32 accumulation.  cache.dtype must
 * be PKV_FP8_E4M3.  Other arguments, the workspace and errors as
 * pkv_paged_attention_decode.
 */
PKV_API pkv_status pkv_paged_attention_decode_fp8(
    void *out, const void *query, pkv_dtype query_dtype, const void *k_cache, const void *v_cache,
    pkv_cache_desc cache, const int32_t *block_tables, int32_t max_blocks_per_seq,
    const int32_t *context_lens, int32_t num_seqs, int32_t num_q_heads, int32_t max_context_len,
    float scale, float k_scale, float v_scale, int32_t partition_size, void *workspace,
    size_t workspace_bytes, int32_t *d_status, pkv_stream_t stream);

/*
 * pkv_paged_prefill - causal attention of chunks of new tokens over their
 * sequences' paged K/V (prompt prefill, or one chunk of a long prompt).
 *
 * lshu.cn/news/11644 (vLLM architecture analysis), sections "整体架构" (a
 * prompt is prefilled, a long one in chunks over several iterations) and
 * "性能关键路径与瓶颈" (prefill is compute-bound on the tensor cores).
 * Sequence s has context_lens[s] = L tokens, the last C = query_start[s+1] -
 * query_start[s] of which are this call's: rows query_start[s] ..
 * query_start[s+1] of query / out.  Their K/V must already be in the pools
 * (pkv_reshape_and_cache of the chunk, as in decode).  The chunk's token at
 * position p = L - C + j attends over positions 0 .. p of its own sequence:
 *   out[t][h] = sum_{i<=p} softmax_i(scale * <query[t][h], K_g[i]>) V_g[i],
 *   g = h / (num_q_heads / num_kv_heads).
 *
 * query, out : [num_tokens][num_q_heads][128] in the cache dtype (fp16/bf16),
 *              16-byte aligned device memory.
 * query_start: int32 [num_seqs + 1] device, non-decreasing, query_start[0] >= 0,
 *              query_start[num_seqs] <= num_tokens; rows outside every chunk
 *              are not written.
 * context_lens: int32 [num_seqs] device, C <= L <= max_blocks_per_seq * B.
 * block_tables: as for decode.  max_query_len >= every C (host value; it
 *              sets the number of 128-row query tiles per (sequence, kv
 *              head)).  PKV_ERR_TOO_LARGE when query tiles x num_kv_heads x
 *              num_seqs exceeds 2^31 - 1.
 * head_dim 128; num_q_heads / num_kv_heads in {1, 2, 4, 8, 16}.
 * Runs on tcgen05 tensor cores: 128-row query tiles x 128-token K/V tiles,
 * fp32 accumulation in tensor memory; a persistent grid of one CTA per SM.
 * workspace  : NULL, or at least PKV_PREFILL_WORKSPACE_BYTES of 4-byte-aligned
 *              device memory owned by the caller (PKV_ERR_WORKSPACE if
 *              smaller).  Given one, the call zeroes an item counter in it
 *              (cudaMemsetAsync on `stream`) and the CTAs take the work items
 *              (query tile, kv head, sequence) in order from it, each as it
 *              frees up, which keeps them evenly loaded when the chunks'
 *              lengths differ; two calls in flight at once need two
 *              workspaces.  NULL: a fixed assignment of items to CTAs.  The
 *              outputs are the same either way, bit for bit.
 * Device-detected errors: a sequence whose lengths break the rules above is
 * skipped with PKV_DEV_BAD_LEN; a block id outside the pool raises
 * PKV_DEV_BAD_BLOCK (that block's tokens are garbage); a wait past ~1 s
 * raises PKV_DEV_TIMEOUT.
 */
PKV_API pkv_status pkv_paged_prefill(void *out, const void *query, const void *k_cache,
                                     const void *v_cache, pkv_cache_desc cache,
                                     const int32_t *block_tables, int32_t max_blocks_per_seq,
                                     const int32_t *query_start, const int32_t *context_lens,
                                     int32_t num_seqs, int32_t num_tokens, int32_t max_query_len,
                                     int32_t num_q_heads, float scale, void *workspace,
                                     size_t workspace_bytes, int32_t *d_status, pkv_stream_t stream);

/* Workspace of pkv_paged_prefill (its item counter, with room to spare). */
#define PKV_PREFILL_WORKSPACE_BYTES 16

/*
 * pkv_paged_attention_decode_lse - decode attention over a part of each
 * sequence, returned as an attention state for a later merge.
 *
 * The same computation and arguments as pkv_paged_attention_decode (16-bit
 * pools), over the tokens that block_tables / context_lens describe, e.g. one
 * GPU's share of a sequence split across GPUs.  Instead of the T16 output it
 * writes, per (sequence, query head) row r = s * num_q_heads + h:
 *   out[r][0..head_dim)  fp32 normalised output  sum_i p_i V_i,
 *   lse[r]               fp32 ln(sum_i exp(z_i)), z_i = scale * <q, K_i>
 *                        (-inf for a row with no tokens, whose out is 0).
 * Split-K identity (textbook softmax; not printed on the pages): outputs over
 * disjoint token sets merge exactly with weights exp(lse_r - max lse).
 * out and lse are device memory, 4-byte aligned; PKV_ERR_NULL_POINTER when lse
 * is NULL.  Workspace and errors as pkv_paged_attention_decode.
 */
PKV_API pkv_status pkv_paged_attention_decode_lse(
    float *out, float *lse, const void *query, const void *k_cache, const void *v_cache,
    pkv_cache_desc cache, const int32_t *block_tables, int32_t max_blocks_per_seq,
    const int32_t *context_lens, int32_t num_seqs, int32_t num_q_heads, int32_t max_context_len,
    float scale, int32_t partition_size, void *workspace, size_t workspace_bytes,
    int32_t *d_status, pkv_stream_t stream);

/*
 * pkv_merge_attention_states - merge attention states of the same rows over
 * disjoint token sets (the all-gathered states of a sequence split across
 * GPUs).
 *
 * states (device, fp32): num_states states, state k starting at
 *   states + k * state_stride (floats), laid out as written by
 *   pkv_paged_attention_decode_lse into one buffer: out [num_rows][head_dim]
 *   followed by lse [num_rows].  state_stride >= num_rows * (head_dim + 1)
 *   when num_states > 1.
 * out (device, out_dtype = PKV_F16 / PKV_BF16): [num_rows][head_dim],
 *   out = sum_k w_k o_k / sum_k w_k with w_k = exp(lse_k - max_k lse_k); a row
 *   whose every lse is -inf (no tokens anywhere) gets 0.  num_states = 0 gives
 *   zero rows.  head_dim 64 or 128.  Asynchronous on stream.
 */
PKV_API pkv_status pkv_merge_attention_states(void *out, pkv_dtype out_dtype, const float *states,
                                              int64_t state_stride, int32_t num_states,
                                              int32_t num_rows, int32_t head_dim,
                                              pkv_stream_t stream);

/*
 * pkv_test_decode_withheld_load - fault injection for tests of the failure
 * path; not for production use and with no counterpart on the pages.
 *
 * Every wait of the decode kernel for a copy into shared memory is bounded:
 * past its limit the kernel raises PKV_DEV_TIMEOUT in *d_status, waits
 * (again bounded) for its other copies in flight, finishes its work unit
 * with what it has and exits, so the device stays usable.  This call runs
 * pkv_paged_attention_decode with one load withheld - logical block
 * withheld_block of sequence 0, kv head 0, never issued, so its barrier never
 * completes - and with every wait limited to wait_limit_us microseconds
 * (1 .. 1000000) instead of about one second.  Expected result: the call's
 * kernels end, *d_status has PKV_DEV_TIMEOUT, the rows of sequence 0's kv
 * head 0 are unspecified and every other row is the normal result.
 * Arguments as pkv_paged_attention_decode; only fp16 pools with head_dim 128
 * and block_size 16 and at most 8 query heads per kv head are accepted
 * (PKV_ERR_BAD_SHAPE otherwise), and withheld_block must lie in the first
 * partition (PKV_ERR_BAD_PARTITION otherwise).
 */
PKV_API pkv_status pkv_test_decode_withheld_load(
    void *out, const void *query, const void *k_cache, const void *v_cache, pkv_cache_desc cache,
    const int32_t *block_tables, int32_t max_blocks_per_seq, const int32_t *context_lens,
    int32_t num_seqs, int32_t num_q_heads, int32_t max_context_len, float scale,
    int32_t partition_size, void *workspace, size_t workspace_bytes, int32_t withheld_block,
    uint32_t wait_limit_us, int32_t *d_status, pkv_stream_t stream);

/* Static English text for a status code. */
PKV_API const char *pkv_status_string(pkv_status status);

/* Library version: major * 10000 + minor * 100 + patch. */
PKV_API int32_t pkv_version(void);

/* 1 in a check build (PKV_CHECK defined: libpkv_check.so), 0 otherwise. */
PKV_API int32_t pkv_check_build(void);

#ifdef __cplusplus
}
#endif

#endif /* PKV_H_ */
