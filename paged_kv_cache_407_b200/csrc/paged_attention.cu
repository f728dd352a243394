// paged_attention_decode: single-token decode attention over a paged KV cache,
// with split-K partitions and a log-sum-exp merge, for B200 (sm_100a).
//
// What it computes (lshu.cn/news/11644, vLLM architecture analysis, section
// "核心创新：PagedAttention 的设计逻辑" / "方案：页式内存管理"): the kernel reads
// each request's scattered blocks through its Block Table and uses them as one
// logically contiguous K/V sequence; the attention is textbook softmax
// attention of one query token per head over that sequence.  "性能关键路径与
// 瓶颈" in the same page: decode is bound by the bytes of KV cache read, and
// Block Table lookups are an overhead to keep small.
//
// Work unit: one partition (up to part_blocks consecutive blocks) of one
// (sequence s, kv head g).  All query heads of group g share each K/V block,
// so every block is read from HBM once.  A sequence with several partitions
// leaves one (m, l, unnormalised O) partial per partition in the workspace;
// the partitions count themselves in on a per-(s, g) counter and the last to
// arrive merges them by log-sum-exp (splits of more than kFuseMaxParts
// partitions are merged by lse_combine_kernel instead).
//
// One CTA per (g, s, partition) slot, three CTAs per SM (about 64 KB of
// shared memory each); slots past a sequence's last partition exit at once.
// Every warp of the CTA streams its share of the unit's blocks (w, w + WARPS,
// ...) through a private ring of shared-memory stages: each stage is one
// block's K and V tiles, loaded by tiled TMA (rank-4 tensor map over
// [N][Hkv][B][D], box 64 x B, 128-byte swizzle, L2 evict-first) and counted
// on an mbarrier; Block Table entries are read 32 at a time per warp, a
// window ahead.  The per-block math is decode_core.cuh.  At the end of the
// unit the warps merge through shared memory, one warp per query head row.
#include <algorithm>

#include "decode_core.cuh"
#include "pkv_host.h"

namespace pkv {
namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// Split sequences with at most this many partitions are merged inside the
// attention kernel by the last partition to finish; longer splits use the
// merge kernel.
constexpr int kFuseMaxParts = 32;

struct DecodeArgs {
  const void *query;
  void *out;          // [S][Hq][D] of T, or of float when lse is set
  float *lse;         // NULL, or [S][Hq]: natural log of the softmax denominator
  const int32_t *block_tables;
  const int32_t *context_lens;
  float *ws_m;        // [S][Hq][max_parts]
  float *ws_l;        // [S][Hq][max_parts]
  float *ws_o;        // [S][Hq][max_parts][D]
  int32_t *counters;  // [S][Hkv] arrivals of split partitions (zeroed per call)
  int32_t *d_status;
  int num_seqs;
  int max_blocks_per_seq;
  int num_q_heads;
  int num_kv_heads;
  int group;        // query heads per kv head
  int num_blocks;   // pool size
  int len_limit;    // largest valid context length
  int part_blocks;  // blocks per partition
  int max_parts;
  float scale_log2;  // softmax scale * log2(e) (times k_scale for 8-bit pools)
  float out_scale;   // 1, or v_scale for 8-bit pools
  const int2 *units;           // split calls: (sequence, partition) per unit, longest first
  const int32_t *unit_count;   // number of units in `units`
  // Fault-injection instance only (FAULT = true): the load of logical block
  // fault_block of sequence 0, kv head 0 is never issued, so its barrier
  // never completes and the wait gives up after fault_wait_ns.
  int fault_block;
  uint64_t fault_wait_ns;
};

// ---------------------------------------------------------------------------
// Result of one work unit, shared by both kernels.
// ---------------------------------------------------------------------------

// Write one finished row: acc = unnormalised output (lane's VPL dims), M / L =
// running max (log2 units of exp(score)) and denominator.  T output, or fp32
// output plus the row's log-sum-exp ln(sum_i exp(z_i)) = (M + log2 L) ln 2.
template <typename T, int D>
__device__ __forceinline__ void write_row(const DecodeArgs &a, size_t row, const float *acc,
                                          float M, float L, int lane) {
  constexpr int VPL = D / 32;
  const float inv = L > 0.f ? a.out_scale / L : 0.f;
  if (a.lse == nullptr) {
    uint32_t *dst = reinterpret_cast<uint32_t *>(static_cast<T *>(a.out) + row * D + lane * VPL);
#pragma unroll
    for (int j = 0; j < VPL; j += 2) dst[j / 2] = Pack<T>::pack(acc[j] * inv, acc[j + 1] * inv);
  } else {
    float *dst = static_cast<float *>(a.out) + row * D + lane * VPL;
#pragma unroll
    for (int j = 0; j < VPL; ++j) dst[j] = acc[j] * inv;
    if (lane == 0) a.lse[row] = L > 0.f ? (M + log2f(L)) * kLn2 : -INFINITY;
  }
}

// Store the result of one unit from `nw` deposited warp states (o at
// mo + w*G*D as [row][D] floats, m/l at mm/ml + w*G), one warp, rows
// h = h0, h0 + hstep, ... of the group.  Lane j owns dims j*VPL .. j*VPL+VPL-1.
// One partition: write the normalised output.  Otherwise write the partial.
template <typename T, int D>
__device__ __forceinline__ void store_unit_warp(const DecodeArgs &a, const float *mo,
                                                const float *mm, const float *ml, int nw, int s,
                                                int g, int part, int nparts, int h0, int hstep,
                                                int lane) {
  constexpr int VPL = D / 32;
  const int G = a.group;
  for (int h = h0; h < G; h += hstep) {
    float M = -INFINITY;
    for (int w = 0; w < nw; ++w) M = fmaxf(M, mm[w * G + h]);
    float acc[VPL];
#pragma unroll
    for (int j = 0; j < VPL; ++j) acc[j] = 0.f;
    float lsum = 0.f;
    if (M != -INFINITY) {
      for (int w = 0; w < nw; ++w) {
        const float wt = fast_exp2(mm[w * G + h] - M);
        lsum += wt * ml[w * G + h];
        const float *src = mo + (w * G + h) * D + lane * VPL;
#pragma unroll
        for (int j = 0; j < VPL; ++j) acc[j] += wt * src[j];
      }
    }
    const size_t row = static_cast<size_t>(s) * a.num_q_heads + static_cast<size_t>(g) * G + h;
    if (nparts == 1) {
      write_row<T, D>(a, row, acc, M, lsum, lane);
    } else {
      const size_t idx = row * a.max_parts + part;
      float *dst = a.ws_o + idx * D + lane * VPL;
#pragma unroll
      for (int j = 0; j < VPL; ++j) dst[j] = acc[j];
      if (lane == 0) {
        a.ws_m[idx] = M;
        a.ws_l[idx] = lsum;
      }
    }
  }
}

// Count one partition of (s, g) in; true for the last of its nparts
// partitions, which also resets the counter.  Call from a single thread after
// the partition's partials are written by its thread group.
__device__ __forceinline__ bool arrive_partition(const DecodeArgs &a, int s, int g, int nparts) {
  __threadfence();  // publish this partition's partials before counting it in
  int *cnt = a.counters + static_cast<size_t>(s) * a.num_kv_heads + g;
  const bool last = atomicAdd(cnt, 1) == nparts - 1;
  if (last) {
    *cnt = 0;  // leave the counter at zero for the next call
    __threadfence();
  }
  return last;
}

// Merge the nparts (<= 32) partials of (s, g) from the workspace into the
// output, one warp, rows h = h0, h0 + hstep, ...: lane p reads partition p's
// (m, l); the maximum and the weighted sum are warp reductions; the partial
// outputs are read eight partitions at a time so their loads overlap, the
// first eight together with (m, l).
template <typename T, int D>
__device__ __forceinline__ void merge_partials_warp(const DecodeArgs &a, int s, int g, int nparts,
                                                    int h0, int hstep, int lane) {
  constexpr int VPL = D / 32;
  const int G = a.group;
  for (int h = h0; h < G; h += hstep) {
    const size_t row = static_cast<size_t>(s) * a.num_q_heads + static_cast<size_t>(g) * G + h;
    const size_t base = row * a.max_parts;
    const float *o = a.ws_o + base * D + lane * VPL;
    // the first eight partial outputs are requested together with (m, l)
    float v[8][VPL];
#pragma unroll
    for (int u = 0; u < 8; ++u)
#pragma unroll
      for (int j = 0; j < VPL; ++j)
        v[u][j] = u < nparts ? __ldcg(o + static_cast<size_t>(u) * D + j) : 0.f;
    const float mp = lane < nparts ? __ldcg(a.ws_m + base + lane) : -INFINITY;
    const float lp = lane < nparts ? __ldcg(a.ws_l + base + lane) : 0.f;
    float M = mp;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(kFullMask, M, off));
    const float w = (lane < nparts && M != -INFINITY) ? fast_exp2(mp - M) : 0.f;
    float L = w * lp;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) L += __shfl_xor_sync(kFullMask, L, off);
    float acc[VPL];
#pragma unroll
    for (int j = 0; j < VPL; ++j) acc[j] = 0.f;
    for (int p0 = 0; p0 < nparts; p0 += 8) {
      if (p0 > 0) {
#pragma unroll
        for (int u = 0; u < 8; ++u)
#pragma unroll
          for (int j = 0; j < VPL; ++j)
            v[u][j] = p0 + u < nparts ? __ldcg(o + static_cast<size_t>(p0 + u) * D + j) : 0.f;
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const float wu = __shfl_sync(kFullMask, w, (p0 + u) & 31);
#pragma unroll
        for (int j = 0; j < VPL; ++j) acc[j] += wu * v[u][j];
      }
    }
    write_row<T, D>(a, row, acc, M, L, lane);
  }
}

__device__ __forceinline__ int clamp_len(const DecodeArgs &a, int s, bool report) {
  int len = a.context_lens[s];
  if (len < 0 || len > a.len_limit) {
    if (report) raise_flag(a.d_status, PKV_DEV_BAD_LEN);
    len = len < 0 ? 0 : a.len_limit;
  }
  return len;
}

__device__ __forceinline__ int parts_of(int nb, int part_blocks) {
  return nb > part_blocks ? (nb + part_blocks - 1) / part_blocks : 1;
}

// Issue the TMA loads of one block of 8-bit pools (K tile of BS rows x D
// codes, V tile of D rows x BS codes) into a stage; tile = block * Hkv + head.
template <int D, int BS>
__device__ __forceinline__ void load_block_fp8(uint32_t dst, const CUtensorMap *tmk,
                                               const CUtensorMap *tmv, uint32_t bar, int tile,
                                               uint64_t policy) {
  mbar_arrive_expect_tx(bar, 2 * BS * D);
  tma_load_5d(dst, tmk, bar, 0, 0, 0, 0, tile, policy);
  tma_load_3d(dst + BS * D, tmv, bar, 0, 0, tile, policy);
}

// Issue the TMA loads of one block (K and V tiles) into a stage.
template <int D, int BS>
__device__ __forceinline__ void load_block(uint32_t dst, const CUtensorMap *tmk,
                                           const CUtensorMap *tmv, uint32_t bar, int g, int id,
                                           uint64_t policy) {
  constexpr int kBoxBytes = BS * 128;
  constexpr int kTileBytes = (D / 64) * kBoxBytes;
  mbar_arrive_expect_tx(bar, 2 * kTileBytes);
#pragma unroll
  for (int bx = 0; bx < D / 64; ++bx) {
    tma_load_4d(dst + bx * kBoxBytes, tmk, bar, bx * 64, 0, g, id, policy);
    tma_load_4d(dst + kTileBytes + bx * kBoxBytes, tmv, bar, bx * 64, 0, g, id, policy);
  }
}

// ---------------------------------------------------------------------------
// Grid kernel: one CTA per (kv head, sequence, partition)
// ---------------------------------------------------------------------------

// Launch shape: a CTA's rings take about 64 KB so three CTAs fit on an SM
// (48 KB and four CTAs for 8-bit pools with 32-token blocks).  SHORT: calls
// whose work units (one partition of one (sequence, kv head)) are at most
// 1024 tokens long take, for 16-token blocks, CTAs of two warps (two stages
// of 16-bit blocks or four of 8-bit ones) and six CTAs per SM: the same
// warps per SM, twice the units in flight, so one unit's start (table,
// query and first tile in flight) overlaps more streaming.  Measured on the
// GQA batch (1024-token partitions): 94.8 -> 89.2 us (16-bit), 66.4 -> 58.6
// us (8-bit); on the 7B batch (whole 2048-token sequences) the same shape
// is 5-8 % slower, whose longer units make the last wave longer.
// LEAN: the 8-bit instances with the tokens on M (DecodeState8T, at most
// eight query heads per kv head), which need 128 registers per thread, so one
// more CTA per SM fits once the stages shrink: for 16-token blocks four CTAs
// of four warps x three stages (7B batch 99.8 -> 98.4 us per call), or eight
// of two warps x three stages for short units (GQA batch 53.4 -> 51.1 us).
template <int D, int BS, int ESZ = 2, bool SHORT = false, bool LEAN = false>
struct GridTune {
  static constexpr int kStage = 2 * BS * D * ESZ;
  // 8-bit pools with 32-token blocks: two warps with three stages each (four
  // CTAs per SM) measured best; four warps spill under the register cap.
  static constexpr bool kKv8Bs32 = ESZ == 1 && BS == 32;
  static constexpr bool kShort = SHORT && BS == 16;
  static constexpr bool kLean16 = LEAN && BS == 16;
  static constexpr int kWarps = kShort ? 2 : (kKv8Bs32 ? 2 : (kStage >= 16384 ? 2 : 4));
  static constexpr int kFit = kShort ? (ESZ == 1 ? (LEAN ? 3 : 4) : 2)
                                     : (kKv8Bs32 || kLean16 ? 3 : 65536 / (kWarps * kStage));
  static constexpr int kStages = kFit < 1 ? 1 : (kFit > 4 ? 4 : kFit);
  // Three CTAs per SM fit in shared memory; ask the register allocation for
  // three as well (at most 168 registers with four warps); six of two warps
  // (LEAN: four and eight, at most 128 registers).
  static constexpr int kMinBlocks = kShort ? (kLean16 ? 8 : 6) : (kLean16 ? 4 : 3);
  static constexpr int kRing = kWarps * kStages * kStage;
  static constexpr int kMerge = kWarps * 16 * (D + 2) * 4;
  static constexpr int kData = kRing > kMerge ? kRing : kMerge;
  static constexpr int kBarOff = (kData + 1023) / 1024 * 1024;
  static constexpr int kNvOff = kBarOff + kWarps * kStages * 8;
  static constexpr int kSmem = kNvOff + kWarps * kStages * 4 + 1024;
};

// FAULT: the fault-injection instance behind pkv_test_decode_withheld_load,
// which withholds one block's load (see DecodeArgs) to show that the bounded
// waits end the kernel with PKV_DEV_TIMEOUT; every other instance has
// FAULT = false and none of its code.
template <typename T, int D, int BS, int WARPS, int NST, bool BIG, bool KV8, bool FAULT = false,
          bool SHORT = false>
__global__ void __launch_bounds__(WARPS * 32, (GridTune<D, BS, KV8 ? 1 : 2, SHORT, KV8 && !BIG>::kMinBlocks))
    paged_decode_grid_kernel(const __grid_constant__ CUtensorMap tm_k,
                             const __grid_constant__ CUtensorMap tm_v, const DecodeArgs a) {
  using TN = GridTune<D, BS, KV8 ? 1 : 2, SHORT, KV8 && !BIG>;
  constexpr int kStageBytes = 2 * BS * D * (KV8 ? 1 : 2);
  using State = typename std::conditional<KV8 && !BIG, DecodeState8T<T, D, BS>,
                                          DecodeState<T, D, BS, BIG, KV8>>::type;
  pdl_trigger();
  pdl_wait();
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  // Without a plan: grid (kv head, sequence, partition slot).  With a plan:
  // one CTA per (unit, kv head) with the kv head fastest; the units come
  // longest first, so long partitions start early and the unused tail exits
  // at once.
  int g, s, part;
  if (a.units == nullptr) {
    g = blockIdx.x;
    s = blockIdx.y;
    part = blockIdx.z;
  } else {
    const int unit = static_cast<int>(blockIdx.x / static_cast<unsigned>(a.num_kv_heads));
    g = static_cast<int>(blockIdx.x % static_cast<unsigned>(a.num_kv_heads));
    if (unit >= __ldg(a.unit_count)) return;  // uniform over the CTA
    const int2 u = __ldg(a.units + unit);
    s = u.x;
    part = u.y;
  }
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int G = a.group;

  // The length, the query rows and the first Block Table window are loaded
  // together: none of them waits for another.
  const int b0 = part * a.part_blocks;
  const int32_t *trow = a.block_tables + static_cast<size_t>(s) * a.max_blocks_per_seq + b0 + warp;
  const int table_left = a.max_blocks_per_seq - b0 - warp;  // table entries from trow on
  auto load_window = [&](int w) -> int {
    const int k = (w << 5) + lane;
    return k * WARPS < table_left ? __ldg(trow + static_cast<size_t>(k) * WARPS) : 0;
  };
  int win_cur = load_window(0);
  State st_;
  st_.load_q(static_cast<const T *>(a.query) +
                 (static_cast<size_t>(s) * a.num_q_heads + static_cast<size_t>(g) * G) * D,
             G, lane);
  const int len = clamp_len(a, s, g == 0 && part == 0 && threadIdx.x == 0);
  const int nb = (len + BS - 1) / BS;
  const int nparts = parts_of(nb, a.part_blocks);
  if (part >= nparts) return;  // uniform over the CTA, before any barrier
  const int nblk = min(nb - b0, a.part_blocks);
  const int tail_nv = len - (nb - 1) * BS;
  const int cnt = nblk > warp ? (nblk - warp + WARPS - 1) / WARPS : 0;

  const uint32_t ring = smem_addr(smem) + warp * NST * kStageBytes;
  const uint32_t bars = smem_addr(smem + TN::kBarOff) + warp * NST * 8;
  volatile int *stage_nv = reinterpret_cast<volatile int *>(smem + TN::kNvOff) + warp * NST;
  if (lane == 0) {
#pragma unroll
    for (int st = 0; st < NST; ++st) mbar_init(bars + 8 * st, 1);
    fence_barrier_init();
    prefetch_tensormap(&tm_k);
    prefetch_tensormap(&tm_v);
  }
  __syncwarp();
  st_.reset();
  int win_next = cnt > 32 ? load_window(1) : 0;

  const uint64_t policy = l2_evict_first_policy();
  auto issue = [&](int k) {
    if ((k & 31) == 0 && k != 0) {
      win_cur = win_next;
      win_next = load_window((k >> 5) + 1);
    }
    const int id = __shfl_sync(kFullMask, win_cur, k & 31);
    if (lane == 0) {
      const int st = k % NST;
      const uint32_t bar = bars + 8 * st;
      const int blk = b0 + warp + k * WARPS;
      if (FAULT && s == 0 && g == 0 && blk == a.fault_block) {
        stage_nv[st] = 0;  // withheld: no load is issued and nothing arrives
      } else if (static_cast<unsigned>(id) < static_cast<unsigned>(a.num_blocks)) {
        stage_nv[st] = (blk == nb - 1) ? tail_nv : BS;
        fence_proxy_async_smem();
        if constexpr (KV8)
          load_block_fp8<D, BS>(ring + st * kStageBytes, &tm_k, &tm_v, bar,
                                id * a.num_kv_heads + g, policy);
        else
          load_block<D, BS>(ring + st * kStageBytes, &tm_k, &tm_v, bar, g, id, policy);
      } else {
        raise_flag(a.d_status, PKV_DEV_BAD_BLOCK);
        stage_nv[st] = 0;  // the whole block is masked
        mbar_arrive(bar);
      }
    }
  };

  int kp = 0;
  for (const int pro = cnt < NST ? cnt : NST; kp < pro; ++kp) issue(kp);
  int k = 0;
  bool ok = true;
  const uint64_t wait_ns = FAULT ? a.fault_wait_ns : kWaitLimitNs;
  for (; k < cnt; ++k) {
    const int st = k % NST;
    ok = __all_sync(kFullMask, mbar_wait(bars + 8 * st, (k / NST) & 1, wait_ns));
    if (!ok) break;
    const uint32_t kb = ring + st * kStageBytes;
    st_.block(kb, kb + kStageBytes / 2, stage_nv[st], a.scale_log2, lane);
    __syncwarp();
    if (kp < cnt) {
      issue(kp);
      ++kp;
    }
  }
  if (!ok) {
    if (lane == 0) raise_flag(a.d_status, PKV_DEV_TIMEOUT);
    // Let the copies still in flight land before the shared memory is reused.
    for (int j = k; j < kp; ++j) (void)mbar_wait(bars + 8 * (j % NST), (j / NST) & 1, wait_ns);
  }

  st_.reduce_l();
  __syncthreads();  // every ring is drained; reuse it for the merge
  float *mo = reinterpret_cast<float *>(smem);  // [WARPS][G][D]
  float *mm = mo + WARPS * 16 * D;              // [WARPS][G]
  float *ml = mm + WARPS * 16;                  // [WARPS][G]
  st_.store_rows(mo + warp * G * D, mm + warp * G, ml + warp * G, G, lane);
  __syncthreads();
  store_unit_warp<T, D>(a, mo, mm, ml, WARPS, s, g, part, nparts, warp, WARPS, lane);
  if (nparts == 1 || nparts > kFuseMaxParts) return;

  __shared__ int s_last;
  __syncthreads();  // this CTA's partials are written
  if (threadIdx.x == 0) s_last = arrive_partition(a, s, g, nparts);
  __syncthreads();
  if (s_last) merge_partials_warp<T, D>(a, s, g, nparts, warp, WARPS, lane);
}

// ---------------------------------------------------------------------------
// Log-sum-exp merge of long splits (more than kFuseMaxParts partitions):
//   M = max_p m_p,  w_p = 2^(m_p - M),  out = sum_p w_p o_p / sum_p w_p l_p.
// ---------------------------------------------------------------------------
struct CombineArgs {
  void *out;   // T, or float when lse is set
  float *lse;  // NULL, or [S][Hq] log-sum-exp
  const int32_t *context_lens;
  const float *ws_m;
  const float *ws_l;
  const float *ws_o;
  int num_q_heads;
  int block_size;
  int len_limit;
  int part_blocks;
  int max_parts;
  float out_scale;
};

template <int NT>
__device__ __forceinline__ float block_reduce(float v, bool is_max, float *scratch) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const float x = __shfl_xor_sync(kFullMask, v, off);
    v = is_max ? fmaxf(v, x) : v + x;
  }
  const int warp = threadIdx.x >> 5;
  __syncthreads();
  if ((threadIdx.x & 31) == 0) scratch[warp] = v;
  __syncthreads();
  v = scratch[0];
#pragma unroll
  for (int w = 1; w < NT / 32; ++w) v = is_max ? fmaxf(v, scratch[w]) : v + scratch[w];
  return v;
}

template <typename T, int D>
__global__ void __launch_bounds__(D) lse_combine_kernel(const CombineArgs c) {
  pdl_trigger();
  pdl_wait();
  __shared__ float scratch[D / 32];
  const int h = blockIdx.x;
  const int s = blockIdx.y;
  int len = c.context_lens[s];
  len = len < 0 ? 0 : (len > c.len_limit ? c.len_limit : len);
  const int nb = (len + c.block_size - 1) / c.block_size;
  const int nparts = parts_of(nb, c.part_blocks);
  if (nparts <= kFuseMaxParts) return;  // written by the attention kernel
  const size_t row = static_cast<size_t>(s) * c.num_q_heads + h;
  const float *pm = c.ws_m + row * c.max_parts;
  const float *pl = c.ws_l + row * c.max_parts;
  const float *po = c.ws_o + row * c.max_parts * D + threadIdx.x;

  float M = -INFINITY;
  for (int p = threadIdx.x; p < nparts; p += D) M = fmaxf(M, pm[p]);
  M = block_reduce<D>(M, true, scratch);
  float lsum = 0.f;
  if (M != -INFINITY)
    for (int p = threadIdx.x; p < nparts; p += D) lsum += fast_exp2(pm[p] - M) * pl[p];
  lsum = block_reduce<D>(lsum, false, scratch);

  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  if (M != -INFINITY) {
    int p = 0;
    for (; p + 4 <= nparts; p += 4) {
#pragma unroll
      for (int u = 0; u < 4; ++u)
        acc[u] += fast_exp2(pm[p + u] - M) * po[static_cast<size_t>(p + u) * D];
    }
    for (; p < nparts; ++p) acc[0] += fast_exp2(pm[p] - M) * po[static_cast<size_t>(p) * D];
  }
  const float total = (acc[0] + acc[1]) + (acc[2] + acc[3]);
  const float o = lsum > 0.f ? total * c.out_scale / lsum : 0.f;
  if (c.lse == nullptr) {
    static_cast<T *>(c.out)[row * D + threadIdx.x] = Pack<T>::from_float(o);
  } else {
    static_cast<float *>(c.out)[row * D + threadIdx.x] = o;
    if (threadIdx.x == 0) c.lse[row] = lsum > 0.f ? (M + log2f(lsum)) * kLn2 : -INFINITY;
  }
}

// ---------------------------------------------------------------------------
// Merge of attention states computed over disjoint parts of the same
// sequences (e.g. on different GPUs): state r holds, per row, the normalised
// fp32 output o_r[D] and its log-sum-exp lse_r.  With M = max_r lse_r and
// w_r = exp(lse_r - M): out = sum_r w_r o_r / sum_r w_r (0 when every lse_r
// is -inf).  One warp per row.
// ---------------------------------------------------------------------------
template <typename T, int D>
__global__ void __launch_bounds__(256)
    merge_states_kernel(void *out, const float *__restrict__ states, int64_t state_stride,
                        int num_states, int num_rows) {
  pdl_trigger();
  pdl_wait();
  constexpr int VPL = D / 32;
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (row >= num_rows) return;
  const size_t lse_off = static_cast<size_t>(num_rows) * D;
  float M = -INFINITY;
  for (int r = 0; r < num_states; ++r) M = fmaxf(M, states[r * state_stride + lse_off + row]);
  float acc[VPL];
#pragma unroll
  for (int j = 0; j < VPL; ++j) acc[j] = 0.f;
  float W = 0.f;
  if (M != -INFINITY) {
    for (int r = 0; r < num_states; ++r) {
      const float *st = states + r * state_stride;
      const float w = fast_exp2((st[lse_off + row] - M) * kLog2e);
      W += w;
      const float *o = st + static_cast<size_t>(row) * D + lane * VPL;
#pragma unroll
      for (int j = 0; j < VPL; ++j) acc[j] += w * o[j];
    }
  }
  const float inv = W > 0.f ? 1.f / W : 0.f;
  uint32_t *dst = reinterpret_cast<uint32_t *>(static_cast<T *>(out) + static_cast<size_t>(row) * D +
                                               lane * VPL);
#pragma unroll
  for (int j = 0; j < VPL; j += 2) dst[j / 2] = Pack<T>::pack(acc[j] * inv, acc[j + 1] * inv);
}

// ---------------------------------------------------------------------------
// Plan of a split call: every non-empty (sequence, partition) unit, ordered
// by its number of blocks, largest first (a counting sort; the order inside
// one size is arbitrary and does not change any result, since partitions are
// merged in partition order).  A sequence without tokens keeps one unit, which
// writes its zero output.  One CTA; it also zeroes the arrival counters.
// Every partition of a sequence but the last is full (part_blocks blocks), so
// a thread takes whole sequences: one read of the length, one count for the
// full partitions and one for the last; the counts of a warp are combined
// before they reach the shared histogram.
// ---------------------------------------------------------------------------
constexpr int kPlanThreads = 1024;
constexpr int kPlanBuckets = 1024;  // unit sizes of 1023 blocks and more share the top bucket

__device__ __forceinline__ int plan_len(const int32_t *lens, int s, int len_limit) {
  const int len = lens[s];
  return len < 0 ? 0 : (len > len_limit ? len_limit : len);
}

__global__ void __launch_bounds__(kPlanThreads)
    decode_plan_kernel(const int32_t *__restrict__ context_lens, int num_seqs, int block_size,
                       int part_blocks, int max_parts, int len_limit, int2 *__restrict__ units,
                       int32_t *__restrict__ unit_count, int32_t *__restrict__ counters,
                       int num_counters) {
  pdl_trigger();
  pdl_wait();
  __shared__ int hist[kPlanBuckets];
  __shared__ int warp_sums[kPlanThreads / 32];
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  hist[tid] = 0;
  for (int i = tid; i < num_counters; i += kPlanThreads) counters[i] = 0;
  const int full_key = min(part_blocks, kPlanBuckets - 1);
  // a sequence's partitions: np - 1 full ones and a last one of `last` blocks
  auto shape = [&](int s, int &np, int &last) {
    const int nb = (plan_len(context_lens, s, len_limit) + block_size - 1) / block_size;
    np = parts_of(nb, part_blocks);
    last = min(max(nb - (np - 1) * part_blocks, 0), kPlanBuckets - 1);
  };
  // sequences in rounds of kPlanThreads; the same rounds in both passes
  const int rounds = (num_seqs + kPlanThreads - 1) / kPlanThreads;
  __syncthreads();
  for (int r = 0; r < rounds; ++r) {
    const int s = r * kPlanThreads + tid;
    int np = 0, last = 0;
    if (s < num_seqs) shape(s, np, last);
    const int nfull = s < num_seqs ? np - 1 : 0;
    const int warp_full = __reduce_add_sync(0xffffffffu, nfull);
    if (lane == 0 && warp_full > 0) atomicAdd(&hist[full_key], warp_full);
    if (s < num_seqs) atomicAdd(&hist[last], 1);
  }
  __syncthreads();
  // offsets in descending key order: offs[k] = sum of hist[k'] over k' > k
  const int key = kPlanBuckets - 1 - tid;  // thread tid scans bucket key
  const int v = hist[key];
  int incl = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += t;
  }
  if (lane == 31) warp_sums[tid >> 5] = incl;
  __syncthreads();
  if (tid < 32) {  // exclusive scan of the 32 warp totals, in place
    const int w = warp_sums[tid];
    int x = w;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, x, off);
      if (tid >= off) x += t;
    }
    warp_sums[tid] = x - w;
    if (tid == 31) *unit_count = x;
  }
  __syncthreads();
  hist[key] = warp_sums[tid >> 5] + incl - v;  // now the next free position of each bucket
  __syncthreads();
  for (int r = 0; r < rounds; ++r) {
    const int s = r * kPlanThreads + tid;
    int np = 0, last = 0;
    if (s < num_seqs) shape(s, np, last);
    const int nfull = s < num_seqs ? np - 1 : 0;
    // this thread's full partitions take consecutive places: the warp's
    // running sum gives each thread its start within the warp's share
    int before = nfull;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, before, off);
      if (lane >= off) before += t;
    }
    const int warp_full = __shfl_sync(0xffffffffu, before, 31);
    before -= nfull;
    int base = 0;
    if (lane == 0 && warp_full > 0) base = atomicAdd(&hist[full_key], warp_full);
    base = __shfl_sync(0xffffffffu, base, 0) + before;
    for (int p = 0; p < nfull; ++p) units[base + p] = make_int2(s, p);
    if (s < num_seqs) units[atomicAdd(&hist[last], 1)] = make_int2(s, np - 1);
  }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
// Automatic partition size.  No split when the (sequence, kv head) units
// alone give about 12 per SM of a 148-SM B200 and no sequence exceeds 2048
// tokens (a whole sequence is then at most 128 blocks of 16 per CTA, short
// next to the call; splitting would only add the merge).  Otherwise 1024
// tokens, halved (down to 256) while the grid would hold fewer than 12 units
// per SM, judged from the largest possible batch (every sequence at
// max_context_len); long sequences are split so that none of them is a tail.
int auto_part_blocks(int block_size, int num_seqs, int num_kv_heads, int max_context_len) {
  const long long want = 148ll * 12;
  if (max_context_len <= 2048 && static_cast<long long>(num_seqs) * num_kv_heads >= want)
    return std::max(1, (max_context_len + block_size - 1) / block_size);
  int tokens = 1024;
  while (tokens > 256) {
    const long long parts = (max_context_len + tokens - 1) / tokens;
    if (static_cast<long long>(num_seqs) * num_kv_heads * std::max(1ll, parts) >= want) break;
    tokens /= 2;
  }
  return std::max(1, tokens / block_size);
}

bool valid_block_size(int bs) { return bs == 8 || bs == 16 || bs == 32 || bs == 64; }

struct Plan {
  int part_blocks;
  int max_parts;
  size_t ctrl_bytes;   // arrival counters and the unit count, zeroed per call
  size_t units_bytes;  // the plan's unit list
  size_t ws_bytes;
};

// Resolve the partitioning and the workspace; false for invalid arguments.
// Workspace (only when a sequence can span several partitions):
//   [arrival counters S*Hkv int32, padded to 16 B]
//   [o partials S*Hq*max_parts*D][m ...][l ...] (fp32).
bool make_plan(int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
               int32_t block_size, int32_t max_context_len, int32_t partition_size, Plan *plan) {
  if (!valid_block_size(block_size) || num_seqs < 0 || num_q_heads < 1 || num_kv_heads < 1 ||
      head_dim < 1 || max_context_len < 0 || partition_size < 0)
    return false;
  int part_blocks;
  if (partition_size == 0) {
    part_blocks = auto_part_blocks(block_size, num_seqs, num_kv_heads, max_context_len);
  } else {
    if (partition_size % block_size != 0) return false;
    part_blocks = partition_size / block_size;
  }
  const long long nb_max = (static_cast<long long>(max_context_len) + block_size - 1) / block_size;
  const long long parts = nb_max > part_blocks ? (nb_max + part_blocks - 1) / part_blocks : 1;
  plan->part_blocks = part_blocks;
  plan->max_parts = static_cast<int>(std::min<long long>(parts, 1ll << 30));
  const bool split = parts > 1 && num_seqs > 0;
  plan->ctrl_bytes = split ? (static_cast<size_t>(num_seqs) * num_kv_heads * 4 + 4 + 15) / 16 * 16 : 0;
  plan->units_bytes = split ? (static_cast<size_t>(num_seqs) * parts * 8 + 15) / 16 * 16 : 0;
  plan->ws_bytes = plan->ctrl_bytes + plan->units_bytes +
                   (split ? static_cast<size_t>(num_seqs) * num_q_heads * parts *
                                (static_cast<size_t>(head_dim) + 2) * sizeof(float)
                          : 0);
  return true;
}

template <typename T, int D, int BS, bool BIG, bool KV8, bool FAULT = false, bool SHORT = false>
pkv_status launch_grid(const CUtensorMap &tmk, const CUtensorMap &tmv, const DecodeArgs &args,
                       cudaStream_t stream) {
  using TN = GridTune<D, BS, KV8 ? 1 : 2, SHORT, KV8 && !BIG>;
  auto kern = paged_decode_grid_kernel<T, D, BS, TN::kWarps, TN::kStages, BIG, KV8, FAULT, SHORT>;
  static std::atomic<uint64_t> smem_set{0};  // per device, this instance
  dim3 grid = args.units == nullptr
                  ? dim3(static_cast<unsigned>(args.num_kv_heads), static_cast<unsigned>(args.num_seqs),
                         static_cast<unsigned>(args.max_parts))
                  : dim3(static_cast<unsigned>(args.num_kv_heads) * args.num_seqs * args.max_parts);
  return launch_with_smem(kern, grid, dim3(TN::kWarps * 32), TN::kSmem, stream, &smem_set, tmk, tmv, args);
}

// short_units: every work unit is at most 1024 tokens (see GridTune).
template <typename T, int D, int BS, bool BIG, bool KV8>
pkv_status launch_shape(const CUtensorMap &tmk, const CUtensorMap &tmv, const DecodeArgs &args,
                        bool short_units, cudaStream_t stream) {
  if (BS == 16 && short_units) return launch_grid<T, D, BS, BIG, KV8, false, true>(tmk, tmv, args, stream);
  return launch_grid<T, D, BS, BIG, KV8>(tmk, tmv, args, stream);
}

// 8-bit pools: head_dim 128, block_size 16, 32 or 64.
template <typename T>
pkv_status launch_decode_fp8(int block_size, bool big, bool short_units, const CUtensorMap &tmk,
                             const CUtensorMap &tmv, const DecodeArgs &args, cudaStream_t stream) {
#define PKV_BS8_CASE(BSV)                                                                   \
  case BSV:                                                                                 \
    return big ? launch_shape<T, 128, BSV, true, true>(tmk, tmv, args, short_units, stream)  \
               : launch_shape<T, 128, BSV, false, true>(tmk, tmv, args, short_units, stream);
  switch (block_size) {
    PKV_BS8_CASE(16)
    PKV_BS8_CASE(32)
    PKV_BS8_CASE(64)
  }
#undef PKV_BS8_CASE
  return PKV_ERR_BAD_SHAPE;
}

template <typename T, int D>
pkv_status launch_for_dim(int block_size, bool big, bool short_units, const CUtensorMap &tmk,
                          const CUtensorMap &tmv, const DecodeArgs &args, cudaStream_t stream) {
#define PKV_BS_CASE(BSV)                                                                   \
  case BSV:                                                                                \
    return big ? launch_shape<T, D, BSV, true, false>(tmk, tmv, args, short_units, stream)  \
               : launch_shape<T, D, BSV, false, false>(tmk, tmv, args, short_units, stream);
  switch (block_size) {
    PKV_BS_CASE(8)
    PKV_BS_CASE(16)
    PKV_BS_CASE(32)
    PKV_BS_CASE(64)
  }
#undef PKV_BS_CASE
  return PKV_ERR_BAD_SHAPE;
}

template <typename T, int D>
pkv_status launch_combine(const CombineArgs &c, int num_seqs, cudaStream_t stream) {
  dim3 grid(static_cast<unsigned>(c.num_q_heads), static_cast<unsigned>(num_seqs));
  return launch_pdl(lse_combine_kernel<T, D>, grid, dim3(D), 0, stream, c) == cudaSuccess ? PKV_OK
                                                                                         : PKV_ERR_CUDA;
}

}  // namespace
}  // namespace pkv

extern "C" size_t pkv_paged_attention_workspace_size(int32_t num_seqs, int32_t num_q_heads,
                                                     int32_t num_kv_heads, int32_t head_dim,
                                                     int32_t block_size, int32_t max_context_len,
                                                     int32_t partition_size) {
  pkv::Plan plan;
  if (!pkv::make_plan(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, max_context_len,
                      partition_size, &plan))
    return 0;
  return plan.ws_bytes;
}

extern "C" int32_t pkv_paged_attention_partition_size(int32_t num_seqs, int32_t num_kv_heads,
                                                      int32_t block_size, int32_t max_context_len,
                                                      int32_t partition_size) {
  pkv::Plan plan;
  if (!pkv::make_plan(num_seqs, num_kv_heads, num_kv_heads, 64, block_size, max_context_len,
                      partition_size, &plan))
    return -1;
  return plan.part_blocks * block_size;
}

namespace pkv {
namespace {

// Shared body of the decode entry points.  kv8: 8-bit pools with scales
// k_scale / v_scale; act: dtype of query (and of out unless lse is set, when
// out is fp32 and lse receives each row's log-sum-exp).
// The tensor maps of one pair of pools.
struct MapCache {
  bool valid = false;
  bool kv8 = false;
  const void *k = nullptr;
  const void *v = nullptr;
  pkv_cache_desc desc{};
  CUtensorMap tmk, tmv;
  bool matches(const void *k_, const void *v_, const pkv_cache_desc &d, bool kv8_) const {
    return valid && k == k_ && v == v_ && kv8 == kv8_ && desc.num_blocks == d.num_blocks &&
           desc.block_size == d.block_size && desc.num_kv_heads == d.num_kv_heads &&
           desc.head_dim == d.head_dim && desc.dtype == d.dtype;
  }
  void set(const void *k_, const void *v_, const pkv_cache_desc &d, bool kv8_) {
    k = k_;
    v = v_;
    desc = d;
    kv8 = kv8_;
    valid = true;
  }
};

// Fault injection (pkv_test_decode_withheld_load only): which load to
// withhold and how long a wait lasts.
struct FaultSpec {
  int block;
  uint64_t wait_ns;
};

pkv_status decode_impl(void *out, float *lse, const void *query, pkv_dtype act, const void *k_cache,
                       const void *v_cache, const pkv_cache_desc &cache, bool kv8,
                       const int32_t *block_tables, int32_t max_blocks_per_seq,
                       const int32_t *context_lens, int32_t num_seqs, int32_t num_q_heads,
                       int32_t max_context_len, float scale, float k_scale, float v_scale,
                       int32_t partition_size, void *workspace, size_t workspace_bytes,
                       int32_t *d_status, pkv_stream_t stream, const FaultSpec *fault = nullptr) {
  pkv_status st = check_cache_desc(cache);
  if (st != PKV_OK) return st;
  if (kv8 ? (cache.dtype != PKV_FP8_E4M3 || !is_16bit(act)) : !is_16bit(cache.dtype))
    return PKV_ERR_BAD_DTYPE;
  if (kv8 && (cache.head_dim != 128 || cache.block_size < 16)) return PKV_ERR_BAD_SHAPE;
  if (num_seqs < 0 || max_context_len < 0 || max_blocks_per_seq < 1 || num_q_heads < 1)
    return PKV_ERR_BAD_SHAPE;
  if (num_q_heads % cache.num_kv_heads != 0 || num_q_heads / cache.num_kv_heads > 16)
    return PKV_ERR_BAD_SHAPE;
  if (!(scale > 0.f) || !(scale < INFINITY)) return PKV_ERR_BAD_SHAPE;
  if (kv8 && (!(k_scale > 0.f) || !(k_scale < INFINITY) || !(v_scale > 0.f) ||
              !(v_scale < INFINITY)))
    return PKV_ERR_BAD_SHAPE;
  if (partition_size < 0 || (partition_size > 0 && partition_size % cache.block_size != 0))
    return PKV_ERR_BAD_PARTITION;
  if (num_seqs == 0) return PKV_OK;
  if (num_seqs > 65535) return PKV_ERR_TOO_LARGE;
  if (!out || !query || !k_cache || !v_cache || !block_tables || !context_lens)
    return PKV_ERR_NULL_POINTER;
  if (!aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(query, 4) || !aligned(out, 4) ||
      !aligned(block_tables, 4) || !aligned(context_lens, 4) || !aligned(lse, 4))
    return PKV_ERR_MISALIGNED;

  Plan plan;
  if (!make_plan(num_seqs, num_q_heads, cache.num_kv_heads, cache.head_dim, cache.block_size,
                 max_context_len, partition_size, &plan))
    return PKV_ERR_BAD_PARTITION;
  if (plan.max_parts > 65535) return PKV_ERR_TOO_LARGE;  // grid z without a plan
  if (static_cast<long long>(num_seqs) * plan.max_parts * cache.num_kv_heads > 2147483647ll)
    return PKV_ERR_TOO_LARGE;  // one CTA per (unit, kv head) in a 1-D grid with a plan
  if (plan.ws_bytes > 0) {
    if (workspace == nullptr || workspace_bytes < plan.ws_bytes) return PKV_ERR_WORKSPACE;
    if (!aligned(workspace, 16)) return PKV_ERR_MISALIGNED;
  }
  if ((st = check_device()) != PKV_OK) return st;

  // The two tensor maps depend only on the pools and their shape; a serving
  // loop calls with the same pools every step, so the last pair encoded on
  // this thread is kept and reused.
  thread_local MapCache last;
  if (!last.matches(k_cache, v_cache, cache, kv8)) {
    last.valid = false;
    if (kv8) {
      if ((st = encode_fp8_k_map(&last.tmk, k_cache, cache)) != PKV_OK) return st;
      if ((st = encode_fp8_v_map(&last.tmv, v_cache, cache)) != PKV_OK) return st;
    } else {
      if ((st = encode_cache_map(&last.tmk, k_cache, cache)) != PKV_OK) return st;
      if ((st = encode_cache_map(&last.tmv, v_cache, cache)) != PKV_OK) return st;
    }
    last.set(k_cache, v_cache, cache, kv8);
  }
  const CUtensorMap &tmk = last.tmk;
  const CUtensorMap &tmv = last.tmv;

  DecodeArgs args{};
  args.query = query;
  args.out = out;
  args.lse = lse;
  args.block_tables = block_tables;
  args.context_lens = context_lens;
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  args.counters = reinterpret_cast<int32_t *>(ws);
  const size_t rows = static_cast<size_t>(num_seqs) * num_q_heads * plan.max_parts;
  float *part = plan.ws_bytes ? reinterpret_cast<float *>(ws + plan.ctrl_bytes + plan.units_bytes) : nullptr;
  const bool split = plan.max_parts > 1;
  // A plan pays when lengths can be spread over several partitions that the
  // attention kernel merges itself (3 .. 32); with two partitions every tail
  // is short, and beyond 32 all sequences are long.
  const bool use_plan = split && plan.max_parts >= 3 && plan.max_parts <= kFuseMaxParts;
  // unit count right after the arrival counters, the unit list after that
  args.unit_count = use_plan ? reinterpret_cast<int32_t *>(ws) + static_cast<size_t>(num_seqs) * cache.num_kv_heads
                             : nullptr;
  args.units = use_plan ? reinterpret_cast<const int2 *>(ws + plan.ctrl_bytes) : nullptr;
  args.ws_o = split ? part : nullptr;
  args.ws_m = split ? part + rows * cache.head_dim : nullptr;
  args.ws_l = split ? part + rows * (cache.head_dim + 1) : nullptr;
  args.d_status = d_status;
  args.num_seqs = num_seqs;
  args.max_blocks_per_seq = max_blocks_per_seq;
  args.num_q_heads = num_q_heads;
  args.num_kv_heads = cache.num_kv_heads;
  args.group = num_q_heads / cache.num_kv_heads;
  args.num_blocks = cache.num_blocks;
  args.len_limit = static_cast<int>(std::min<long long>(
      max_context_len, static_cast<long long>(max_blocks_per_seq) * cache.block_size));
  args.part_blocks = plan.part_blocks;
  args.max_parts = plan.max_parts;
  args.scale_log2 = scale * kLog2e * (kv8 ? k_scale : 1.f);
  args.out_scale = kv8 ? v_scale : 1.f;
  args.fault_block = fault ? fault->block : -1;
  args.fault_wait_ns = fault ? fault->wait_ns : kWaitLimitNs;

  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (split && !use_plan && cudaMemsetAsync(ws, 0, plan.ctrl_bytes, s) != cudaSuccess)
    return PKV_ERR_CUDA;
  if (use_plan) {  // the plan (which also zeroes the arrival counters)
    if (launch_pdl(decode_plan_kernel, dim3(1), dim3(kPlanThreads), 0, s, context_lens, num_seqs,
                   static_cast<int>(cache.block_size), plan.part_blocks, plan.max_parts, args.len_limit,
                   reinterpret_cast<int2 *>(ws + plan.ctrl_bytes), const_cast<int32_t *>(args.unit_count),
                   args.counters, num_seqs * cache.num_kv_heads) != cudaSuccess)
      return PKV_ERR_CUDA;
  }
  const bool big = args.group > 8;
  const bool bf16 = act == PKV_BF16;
  const bool short_units = static_cast<long long>(plan.part_blocks) * cache.block_size <= 1024;
  if (fault != nullptr) {
    // the one fault-injection instance: fp16 pools, head_dim 128, 16-token
    // blocks, at most 8 query heads per kv head (checked by the caller)
    st = launch_grid<__half, 128, 16, false, false, true>(tmk, tmv, args, s);
  } else if (kv8)
    st = bf16 ? launch_decode_fp8<__nv_bfloat16>(cache.block_size, big, short_units, tmk, tmv, args, s)
              : launch_decode_fp8<__half>(cache.block_size, big, short_units, tmk, tmv, args, s);
  else if (cache.head_dim == 128)
    st = bf16 ? launch_for_dim<__nv_bfloat16, 128>(cache.block_size, big, short_units, tmk, tmv, args, s)
              : launch_for_dim<__half, 128>(cache.block_size, big, short_units, tmk, tmv, args, s);
  else
    st = bf16 ? launch_for_dim<__nv_bfloat16, 64>(cache.block_size, big, short_units, tmk, tmv, args, s)
              : launch_for_dim<__half, 64>(cache.block_size, big, short_units, tmk, tmv, args, s);
  if (st != PKV_OK || plan.max_parts <= kFuseMaxParts) return st;

  CombineArgs c{};
  c.out = out;
  c.lse = lse;
  c.context_lens = context_lens;
  c.ws_m = args.ws_m;
  c.ws_l = args.ws_l;
  c.ws_o = args.ws_o;
  c.num_q_heads = num_q_heads;
  c.block_size = cache.block_size;
  c.len_limit = args.len_limit;
  c.part_blocks = plan.part_blocks;
  c.max_parts = plan.max_parts;
  c.out_scale = args.out_scale;
  if (cache.head_dim == 128)
    return bf16 ? launch_combine<__nv_bfloat16, 128>(c, num_seqs, s)
                : launch_combine<__half, 128>(c, num_seqs, s);
  return bf16 ? launch_combine<__nv_bfloat16, 64>(c, num_seqs, s)
              : launch_combine<__half, 64>(c, num_seqs, s);
}

}  // namespace
}  // namespace pkv

extern "C" pkv_status pkv_paged_attention_decode(
    void *out, const void *query, const void *k_cache, const void *v_cache, pkv_cache_desc cache,
    const int32_t *block_tables, int32_t max_blocks_per_seq, const int32_t *context_lens,
    int32_t num_seqs, int32_t num_q_heads, int32_t max_context_len, float scale,
    int32_t partition_size, void *workspace, size_t workspace_bytes, int32_t *d_status,
    pkv_stream_t stream) {
  return pkv::decode_impl(out, nullptr, query, cache.dtype, k_cache, v_cache, cache, false, block_tables,
                          max_blocks_per_seq, context_lens, num_seqs, num_q_heads, max_context_len,
                          scale, 1.f, 1.f, partition_size, workspace, workspace_bytes, d_status,
                          stream);
}

extern "C" pkv_status pkv_paged_attention_decode_fp8(
    void *out, const void *query, pkv_dtype query_dtype, const void *k_cache, const void *v_cache,
    pkv_cache_desc cache, const int32_t *block_tables, int32_t max_blocks_per_seq,
    const int32_t *context_lens, int32_t num_seqs, int32_t num_q_heads, int32_t max_context_len,
    float scale, float k_scale, float v_scale, int32_t partition_size, void *workspace,
    size_t workspace_bytes, int32_t *d_status, pkv_stream_t stream) {
  return pkv::decode_impl(out, nullptr, query, query_dtype, k_cache, v_cache, cache, true, block_tables,
                          max_blocks_per_seq, context_lens, num_seqs, num_q_heads, max_context_len,
                          scale, k_scale, v_scale, partition_size, workspace, workspace_bytes,
                          d_status, stream);
}

extern "C" pkv_status pkv_paged_attention_decode_lse(
    float *out, float *lse, const void *query, const void *k_cache, const void *v_cache,
    pkv_cache_desc cache, const int32_t *block_tables, int32_t max_blocks_per_seq,
    const int32_t *context_lens, int32_t num_seqs, int32_t num_q_heads, int32_t max_context_len,
    float scale, int32_t partition_size, void *workspace, size_t workspace_bytes,
    int32_t *d_status, pkv_stream_t stream) {
  if (lse == nullptr && num_seqs > 0) return PKV_ERR_NULL_POINTER;
  return pkv::decode_impl(out, lse, query, cache.dtype, k_cache, v_cache, cache, false,
                          block_tables, max_blocks_per_seq, context_lens, num_seqs, num_q_heads,
                          max_context_len, scale, 1.f, 1.f, partition_size, workspace,
                          workspace_bytes, d_status, stream);
}

extern "C" pkv_status pkv_merge_attention_states(void *out, pkv_dtype out_dtype, const float *states,
                                                 int64_t state_stride, int32_t num_states,
                                                 int32_t num_rows, int32_t head_dim,
                                                 pkv_stream_t stream) {
  using namespace pkv;
  if (!is_16bit(out_dtype)) return PKV_ERR_BAD_DTYPE;
  if (num_states < 0 || num_rows < 0 || (head_dim != 64 && head_dim != 128))
    return PKV_ERR_BAD_SHAPE;
  if (num_rows == 0) return PKV_OK;
  if (out == nullptr || (num_states > 0 && states == nullptr)) return PKV_ERR_NULL_POINTER;
  const int64_t need = static_cast<int64_t>(num_rows) * (head_dim + 1);
  if (num_states > 1 && state_stride < need) return PKV_ERR_BAD_SHAPE;
  if (!aligned(out, 4) || !aligned(states, 4)) return PKV_ERR_MISALIGNED;
  if (num_rows > (1 << 30) / 8) return PKV_ERR_TOO_LARGE;
  pkv_status st = check_device();
  if (st != PKV_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const dim3 grid(static_cast<unsigned>((num_rows + 7) / 8));
  const bool bf16 = out_dtype == PKV_BF16;
  cudaError_t err;
  if (head_dim == 128)
    err = bf16 ? launch_pdl(merge_states_kernel<__nv_bfloat16, 128>, grid, dim3(256), 0, s, out, states,
                            state_stride, num_states, num_rows)
               : launch_pdl(merge_states_kernel<__half, 128>, grid, dim3(256), 0, s, out, states, state_stride,
                            num_states, num_rows);
  else
    err = bf16 ? launch_pdl(merge_states_kernel<__nv_bfloat16, 64>, grid, dim3(256), 0, s, out, states,
                            state_stride, num_states, num_rows)
               : launch_pdl(merge_states_kernel<__half, 64>, grid, dim3(256), 0, s, out, states, state_stride,
                            num_states, num_rows);
  return err == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

extern "C" pkv_status pkv_test_decode_withheld_load(
    void *out, const void *query, const void *k_cache, const void *v_cache, pkv_cache_desc cache,
    const int32_t *block_tables, int32_t max_blocks_per_seq, const int32_t *context_lens,
    int32_t num_seqs, int32_t num_q_heads, int32_t max_context_len, float scale,
    int32_t partition_size, void *workspace, size_t workspace_bytes, int32_t withheld_block,
    uint32_t wait_limit_us, int32_t *d_status, pkv_stream_t stream) {
  using namespace pkv;
  if (cache.dtype != PKV_F16 || cache.head_dim != 128 || cache.block_size != 16 ||
      cache.num_kv_heads < 1 || num_q_heads % cache.num_kv_heads != 0 ||
      num_q_heads / cache.num_kv_heads > 8)
    return PKV_ERR_BAD_SHAPE;
  if (withheld_block < 0 || wait_limit_us < 1 || wait_limit_us > 1000000u) return PKV_ERR_BAD_SHAPE;
  const int32_t part = pkv_paged_attention_partition_size(num_seqs, cache.num_kv_heads, 16,
                                                          max_context_len, partition_size);
  if (part < 0 || withheld_block >= part / 16) return PKV_ERR_BAD_PARTITION;
  const FaultSpec fault{withheld_block, static_cast<uint64_t>(wait_limit_us) * 1000ull};
  return decode_impl(out, nullptr, query, cache.dtype, k_cache, v_cache, cache, false,
                     block_tables, max_blocks_per_seq, context_lens, num_seqs, num_q_heads,
                     max_context_len, scale, 1.f, 1.f, partition_size, workspace, workspace_bytes,
                     d_status, stream, &fault);
}
