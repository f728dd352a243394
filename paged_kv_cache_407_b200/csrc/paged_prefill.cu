// Paged (chunked) prefill attention on the fifth-generation tensor cores.
//
// lshu.cn/news/11644 (vLLM architecture analysis): "整体架构" (a new request's
// prompt is prefilled, a long prompt in chunks over several iterations) and
// "性能关键路径与瓶颈" (prefill is compute-bound on the tensor cores).  For each
// sequence, the chunk's token at position p = L - C + j (its K/V already
// written to the cache) attends over positions 0..p through the Block Table.
//
// A work item is a (128-row query tile, kv head, sequence); a tile row is one
// (token, query head of the group) pair, so 128 / G tokens per tile.  The
// grid is persistent (one CTA per SM): each CTA takes its next item from a
// counter in the caller's workspace as it frees up (or, without one, walks a
// fixed share of the items), so that the next item's Q tile and first K/V
// tiles load while the current one finishes.  Roles (warp-specialised,
// synchronised only through mbarriers):
//   warps 0-7  softmax, 16 rows per warp: read with the 16-lane tcgen05.ld
//              shape, a row's 128 scores of a tile sit with the four threads
//              of one quad (32 each, two rows per thread), so the row max and
//              sum are two shuffles and one O accumulator serves the row.
//              Causal mask, lazy rescaling (the reference max moves only when
//              the row max grows by more than 2^8; then O in TMEM is rescaled,
//              after P V(j-1) is done), P written back into the S buffer as
//              the A operand (fp16, or bf16 high + bf16 residual, since bf16
//              alone would round P by 2^-9), finally O / l;
//   warp 8     takes the items and publishes each index to the other warps
//              (a four-slot ring in shared memory); TMA: the Q tiles (rank-3
//              map over [T][Hq][D], two buffers) and the K tiles, 128 tokens
//              gathered through the Block Table, one TMA box per block (a
//              rank-5 view of [N][Hkv][B][D] that lands the block as groups of
//              8 rows, so that the tile's 8-row groups sit at one fixed stride
//              for the tensor core), lane b issuing block b's box, the block
//              ids read ahead by cp.async; two stages;
//   warp 9     TMA: the V tiles, the same way, two stages;
//   warp 10    tcgen05.mma, one thread: S(j) = Q K(j)^T (128x128x128) into
//              one of three TMEM buffers, once P V(j-3) has read that buffer;
//   warp 11    tcgen05.mma, one thread: O += P(j) V(j) with P read from tensor
//              memory (the S buffer) and V from shared memory (MN-major).
//              Two issuers, because a thread that has just
//              issued a batch of MMAs waits for the tensor pipe to take them
//              before its next barrier test completes: with one issuer every
//              operand wait sat on the pipe's critical path.
// Every wait is bounded; after a timeout every role stops, PKV_DEV_TIMEOUT is
// raised, outstanding tensor-core work and loads are drained (bounded) and
// TMEM is freed.
#include <cudaTypedefs.h>

#include <type_traits>

#include "pkv_device.cuh"
#include "pkv_host.h"
#include "tcgen05.cuh"

namespace pkv {
namespace {

constexpr int kRows = 128;    // query rows per tile (MMA M)
constexpr int kKv = 128;      // tokens per K/V tile
constexpr int kDim = 128;     // head_dim
constexpr int kSoftmaxWarps = 8;  // warps 0-7: (query row, token half) per thread
constexpr int kSoftmaxThreads = 32 * kSoftmaxWarps;
constexpr int kLoadKWarp = 8;     // TMA loads of K tiles (and Q)
constexpr int kLoadVWarp = 9;     // TMA loads of V tiles
constexpr int kMmaWarp = 10;      // issues the S = Q K^T MMAs
constexpr int kPvWarp = 11;       // issues the O += P V MMAs
constexpr int kThreads = 32 * 12;
constexpr uint32_t kChunk = 128u * 128u;  // [128 rows][64 elements] of 16-bit: 16 KB
constexpr uint32_t kTile = 2u * kChunk;   // [128][128] of 16-bit: 32 KB
constexpr uint32_t kQOff = 0;               // two Q buffers (this item's, the next one's)
constexpr uint32_t kKOff = 2u * kTile;       // two K stages
constexpr uint32_t kVOff = 4u * kTile;       // two V stages
constexpr uint32_t kXOff = 6u * kTile;       // final (m, l) exchange of the softmax halves
constexpr int kSBufs = 3;                    // S buffers in tensor memory
constexpr uint32_t kTmemCols = 512;          // S buffers [0, 384), O [384, 512)
constexpr float kLazyRescale = 8.f;               // log2 of the largest P allowed
constexpr uint32_t kFullMask = 0xffffffffu;

// One 32-bit word from global to shared memory, asynchronously (no register
// is written, so nothing waits on it until cp_async_wait).
__device__ __forceinline__ void cp_async_4(uint32_t dst, const void *src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
// Until at most N of this thread's most recent groups are still in flight.
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// max(a, b, c) in one instruction (three-input max.f32, sm_100).
__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// K/V tiles in shared memory: 16 groups of 8 token rows, group i at 2048 i;
// within a group the two 64-element halves of head_dim at +0 / +1024, each
// 8 rows of 128 bytes (128-byte swizzle).  Token groups are 2048 bytes apart
// whatever the block size, so one descriptor stride covers a whole tile.
constexpr uint32_t kGroupBytes = 2048;

template <typename T>
struct PrefillTune {
  static constexpr bool kSplit = std::is_same<T, __nv_bfloat16>::value;
  static constexpr uint32_t kBarOff = kXOff + 2u * kRows * 8u;
  // block-id rings of the two load warps: [warp][3 tiles][16 entries]
  static constexpr uint32_t kTabOff = kBarOff + 320u;
  static constexpr uint32_t kSmem = kTabOff + 2u * 3u * 16u * 4u + 1024u;
};

struct PrefillArgs {
  void *out;
  const int32_t *block_tables;
  const int32_t *query_start;
  const int32_t *context_lens;
  int32_t *d_status;
  int num_tokens;
  int num_seqs;
  int max_blocks_per_seq;
  int num_q_heads;
  int group;
  int num_blocks;
  int num_kv_heads;
  int qtiles;      // query tiles of the longest chunk
  int items;       // qtiles * num_kv_heads * num_seqs work items
  float scale_log2;
  // Non-null: CTAs take items in index order from this counter (zeroed
  // before the launch), each as it frees up.  Null: the static order of
  // item_index.
  unsigned int *ticket;
};

// One work item: a 128-row query tile of one (sequence, kv head).  Items are
// numbered in groups of kPairsPerGroup (sequence, kv head) pairs; inside a
// group, longest first (query tile qtiles - 1 of each pair, then qtiles - 2,
// ...: later query tiles see more keys).  The CTAs working at one time then
// share the K/V of a few pairs, which stay in L2 (one pair per group measured
// best: 1 to 4 % over groups of 2 to 8 pairs).
constexpr int kPairsPerGroup = 1;
struct Item {
  int s, g, t_begin, C, L, tok0, ntiles, nb;
};

template <int BS>
__device__ __forceinline__ bool item_at(const PrefillArgs &a, int i, Item &it, bool report) {
  const int pairs = a.num_kv_heads * a.num_seqs;
  const int group_items = kPairsPerGroup * a.qtiles;
  const int full = pairs / kPairsPerGroup;  // complete groups
  const int grp = i / group_items;
  const int width = grp < full ? kPairsPerGroup : pairs - full * kPairsPerGroup;
  const int rem = i - grp * group_items;
  const int qt = a.qtiles - 1 - rem / width;
  const int pair = grp * kPairsPerGroup + rem % width;
  it.g = pair % a.num_kv_heads;
  it.s = pair / a.num_kv_heads;
  it.t_begin = a.query_start[it.s];
  const int t_end = a.query_start[it.s + 1];
  it.C = t_end - it.t_begin;
  it.L = a.context_lens[it.s];
  if (it.C < 0 || it.t_begin < 0 || t_end > a.num_tokens || it.L < it.C ||
      static_cast<long long>(it.L) > static_cast<long long>(a.max_blocks_per_seq) * BS) {
    if (report && it.g == 0 && qt == 0) raise_flag(a.d_status, PKV_DEV_BAD_LEN);
    return false;
  }
  it.tok0 = qt * (kRows / a.group);
  if (it.tok0 >= it.C) return false;
  const int last_tok = min(it.tok0 + kRows / a.group, it.C) - 1;
  it.ntiles = (it.L - it.C + last_tok + kKv) / kKv;  // K/V tiles up to the largest position
  it.nb = (it.L + BS - 1) / BS;
  return true;
}

// The k-th item of this CTA (-1 past the end): rounds of gridDim.x items,
// alternate rounds walked in opposite directions so that every CTA gets a
// similar share of long and short items.
__device__ __forceinline__ int item_index(const PrefillArgs &a, int k) {
  const int P = static_cast<int>(gridDim.x);
  const int c = static_cast<int>(blockIdx.x);
  const long long i = static_cast<long long>(k) * P + ((k & 1) ? P - 1 - c : c);
  return i < a.items ? static_cast<int>(i) : -1;
}

template <typename T, int BS>
__global__ void __launch_bounds__(kThreads, 1)
    paged_prefill_kernel(const __grid_constant__ CUtensorMap tm_q,
                         const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v, const PrefillArgs a) {
  using TN = PrefillTune<T>;
  constexpr bool kSplit = TN::kSplit;
  constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
  constexpr int kBlocksPerTile = kKv / BS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sb = smem_addr(smem);
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int G = a.group;

  // ---- barriers (see the role loops for who arrives on which) ------------
  // Every role walks the same items in the same order and keeps running
  // counts (items, K/V tiles), so stage indices and phase parities carry on
  // across items.
  const uint32_t bars = sb + TN::kBarOff;
  const uint32_t bar_q = bars;            // [2] Q buffer loaded (TMA bytes)
  const uint32_t bar_qfree = bars + 16;   // [2] Q buffer read by the item's last S (MMA commit)
  const uint32_t bar_k = bars + 32;       // [2] K stage loaded (TMA bytes)
  const uint32_t bar_kfree = bars + 48;   // [2] K stage read by S (MMA commit)
  const uint32_t bar_v = bars + 64;       // [2] V stage loaded
  const uint32_t bar_vfree = bars + 80;   // [2] V stage read by P V
  const uint32_t bar_s = bars + 96;       // [3] S buffer written (MMA commit)
  // P-ready comes one per S buffer: a softmax warp may arrive for tile j+1
  // before a slower one arrives for tile j, and those arrivals must not
  // count towards the same phase.
  const uint32_t bar_p = bars + 120;      // [3] P in TMEM, O rescaled (one arrival per softmax warp)
  // [3] P V of the buffer's tile done (MMA commit): frees the S buffer, and
  // tells the softmax that O holds that tile's product (for the rescale, and
  // for the epilogue after an item's last tile).  A wait on it cannot be
  // ambiguous: its next phase needs P of three tiles on, which the waiting
  // warp has not written.
  const uint32_t bar_pfree = bars + 144;
  const uint32_t bar_done = bars + 176;   // drain on the error path
  const uint32_t holder = bars + 184;
  volatile uint32_t *holder_ptr = reinterpret_cast<volatile uint32_t *>(smem + TN::kBarOff + 184);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + TN::kBarOff + 188);
  // The CTA's item sequence: the K-load warp takes each item (from the
  // ticket counter, or the static order) and publishes its index in slot
  // k % 4 of a ring; every other role reads it there, so all walk the same
  // items.  [4] index published (1 arrival) / read by every other role.
  const uint32_t bar_item = bars + 192;
  const uint32_t bar_itemfree = bars + 224;
  constexpr int kItemReaders = 3 + kSoftmaxWarps;  // V-load, S-issue, P V-issue and softmax warps
  // [4] int32 slots.  Its address is derived from the shared window's base
  // where it is used, so no register holds it through the other roles' loops.
  auto item_slot = [&](int slot) -> uint32_t {
    return ((smem_addr(smem_raw) + 1023u) & ~1023u) + TN::kBarOff + 256u + 4u * static_cast<uint32_t>(slot);
  };

  pdl_trigger();
  pdl_wait();  // before any global access and before taking tensor memory
  if (warp == 0) tc::tmem_alloc(holder, kTmemCols);
  if (tid == 0) {
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar_q + 8 * i, 1);
      mbar_init(bar_qfree + 8 * i, 1);
      mbar_init(bar_k + 8 * i, 1);
      mbar_init(bar_kfree + 8 * i, 1);
      mbar_init(bar_v + 8 * i, 1);
      mbar_init(bar_vfree + 8 * i, 1);
    }
#pragma unroll
    for (int i = 0; i < kSBufs; ++i) {
      mbar_init(bar_s + 8 * i, 1);
      mbar_init(bar_p + 8 * i, kSoftmaxWarps);
      mbar_init(bar_pfree + 8 * i, 1);
    }
    mbar_init(bar_done, 2);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      mbar_init(bar_item + 8 * i, 1);
      mbar_init(bar_itemfree + 8 * i, kItemReaders);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *holder_ptr;
  const uint32_t tO = tmem + kSBufs * kKv;  // O [128 rows][128 columns]

  // A wait that gives up after ~1 s (then every role stops).
  auto wait = [&](uint32_t bar, uint32_t parity) -> bool {
    if (*abort_flag) return false;
    if (mbar_wait(bar, parity)) return true;
    *abort_flag = 1;
    return false;
  };
  // The k-th item of this CTA as the roles other than the K-load warp see
  // it: false if a wait ran out; i = -1 past the last item.
  auto read_item = [&](int k, int &i) -> bool {
    const int slot = k & 3;
    if (!wait(bar_item + 8 * slot, (k >> 2) & 1)) return false;
    asm volatile("ld.volatile.shared.s32 %0, [%1];" : "=r"(i) : "r"(item_slot(slot)) : "memory");
    __syncwarp();
    if (lane == 0) mbar_arrive(bar_itemfree + 8 * slot);
    return true;
  };

  if (warp == kLoadKWarp || warp == kLoadVWarp) {
    // ---------------------------------------------------------- producers
    const bool is_k = warp == kLoadKWarp;
    const CUtensorMap *map = is_k ? &tm_k : &tm_v;
    if (lane == 0) {
      prefetch_tensormap(map);
      if (is_k) prefetch_tensormap(&tm_q);
    }
    const uint64_t policy = l2_evict_first_policy();
    const uint32_t full = is_k ? bar_k : bar_v;
    const uint32_t empty = is_k ? bar_kfree : bar_vfree;
    const uint32_t stage0 = sb + (is_k ? kKOff : kVOff);
    bool run = true;
    int n = 0;   // items so far
    int jt = 0;  // K/V tiles so far
    for (int k = 0; run; ++k) {
      int i;
      if (is_k) {
        // take the CTA's k-th item and publish it to the other roles, once
        // they have all read the index the slot held four items back
        const int slot = k & 3;
        if (k >= 4 && !(run = wait(bar_itemfree + 8 * slot, ((k - 4) >> 2) & 1))) break;
        int idx = 0;
        if (lane == 0) {
          idx = a.ticket != nullptr ? static_cast<int>(min(atomicAdd(a.ticket, 1u), 0x7fffffffu))
                                    : item_index(a, k);
          if (idx >= a.items) idx = -1;
          asm volatile("st.volatile.shared.s32 [%0], %1;" ::"r"(item_slot(slot)), "r"(idx) : "memory");
          mbar_arrive(bar_item + 8 * slot);
        }
        i = __shfl_sync(kFullMask, idx, 0);
      } else if (!(run = read_item(k, i))) {
        break;
      }
      if (i < 0) break;
      Item it;
      if (!item_at<BS>(a, i, it, false)) continue;
      if (is_k) {
        // the item's Q tile into Q buffer n % 2, once the item two back has
        // done its last S
        const int qb = n & 1;
        if (n >= 2 && !(run = wait(bar_qfree + 8 * qb, ((n - 2) >> 1) & 1))) break;
        if (lane == 0) {
          mbar_arrive_expect_tx(bar_q + 8 * qb, kTile);
#pragma unroll
          for (int c = 0; c < 2; ++c)
            tma_load_3d(sb + kQOff + qb * kTile + c * kChunk, &tm_q, bar_q + 8 * qb, c * 64, it.g * G,
                        it.t_begin + it.tok0, policy);
        }
      }
      const int32_t *trow = a.block_tables + static_cast<size_t>(it.s) * a.max_blocks_per_seq;
      // The block ids of tile t reach slot t % 3 of this warp's ring by
      // cp.async two tiles before use, so the Block Table's latency stays
      // off this loop.  Lane b < kBlocksPerTile owns entry b of every slot:
      // it copies that entry in and reads it back itself, so no other
      // lane's copy needs ordering.
      int32_t *ring = reinterpret_cast<int32_t *>(smem + TN::kTabOff) + (is_k ? 0 : 3 * 16);
      auto fetch = [&](int t) {
        const int lb = t * kBlocksPerTile + lane;
        if (t < it.ntiles && lane < kBlocksPerTile && lb < it.nb)
          cp_async_4(smem_addr(ring + (t % 3) * 16 + lane), trow + lb);
        cp_async_commit();  // a group per tile, empty or not
      };
      fetch(0);
      fetch(1);
      for (int j = 0; j < it.ntiles; ++j, ++jt) {
        const int st = jt & 1;
        fetch(j + 2);  // slot (j + 2) % 3 was read back at tile j - 1
        if (jt >= 2 && !(run = wait(empty + 8 * st, ((jt - 2) >> 1) & 1))) break;
        cp_async_wait<2>();  // this lane's entry of tile j is in
        const bool in_tile = lane < kBlocksPerTile && j * kBlocksPerTile + lane < it.nb;
        const int id = in_tile ? ring[(j % 3) * 16 + lane] : -1;
        const bool ok = in_tile && static_cast<unsigned>(id) < static_cast<unsigned>(a.num_blocks);
        if (in_tile && !ok) raise_flag(a.d_status, PKV_DEV_BAD_BLOCK);
        // one vote instead of a shuffle per block: this warp shares its
        // sub-partition's MIO queue with two softmax warps' exponentials, and
        // every shuffle waits its turn there
        const uint32_t bytes = static_cast<uint32_t>(__popc(__ballot_sync(kFullMask, ok))) * (256u * BS);
        const uint32_t bar = full + 8 * st;
        if (lane == 0) {
          fence_proxy_async_smem();
          if (bytes == 0) mbar_arrive(bar);
          else mbar_arrive_expect_tx(bar, bytes);
        }
        __syncwarp();
        // lane b issues block b's box: one TMA instruction for the tile
        // instead of kBlocksPerTile issued one after another
        if (ok)
          tma_load_5d(stage0 + st * kTile + lane * (BS / 8) * kGroupBytes, map, bar, 0, 0, 0, 0,
                      id * a.num_kv_heads + it.g, policy);
      }
      ++n;
    }
    cp_async_wait<0>();  // no copy into the ring outlives the loop
  } else if (warp == kMmaWarp || warp == kPvWarp) {
    // --------------------------------------------------------- MMA issuers
    // Two issuing warps feed the one tensor pipe, so that neither kind of
    // MMA waits behind the other's operands: S(j) goes as soon as K(j) is in
    // and P V(j-2) has read the S buffer it overwrites; P V(j) as soon as
    // V(j) and P(j) are ready.
    constexpr uint32_t kIdescS = tc::idesc_f16(kBf16, false, 128, 128);
    constexpr uint32_t kIdescO = tc::idesc_f16(kBf16, true, 128, 128);
    const bool is_s = warp == kMmaWarp;
    bool run = true;
    int n = 0;
    int jt = 0;
    for (int k = 0; run; ++k) {
      int i;
      if (!(run = read_item(k, i))) break;
      if (i < 0) break;
      Item it;
      if (!item_at<BS>(a, i, it, false)) continue;
      const int qb = n & 1;
      if (is_s) {
        if (!(run = wait(bar_q + 8 * qb, (n >> 1) & 1))) break;
        const uint32_t qbase = sb + kQOff + qb * kTile;
        for (int j = 0; j < it.ntiles; ++j, ++jt) {
          const int b = jt % kSBufs;  // S buffer
          const int ks = jt & 1;      // K stage
          if (jt >= kSBufs && !(run = wait(bar_pfree + 8 * b, (jt / kSBufs - 1) & 1))) break;
          if (!(run = wait(bar_k + 8 * ks, (jt >> 1) & 1))) break;
          if (lane == 0) {
            tc::fence_after_sync();
            const uint32_t kb = sb + kKOff + ks * kTile;
#pragma unroll
            for (int kk = 0; kk < kDim / 16; ++kk) {
              const uint32_t qoff = (kk >> 2) * kChunk + (kk & 3) * 32u;
              const uint32_t koff = (kk >> 2) * 1024u + (kk & 3) * 32u;
              tc::mma_f16_ss(tmem + b * kKv, tc::smem_desc_sw128(qbase + qoff, 16u, 1024u),
                             tc::smem_desc_sw128(kb + koff, 16u, kGroupBytes), kIdescS, kk > 0 ? 1u : 0u);
            }
            tc::commit(bar_s + 8 * b);
            tc::commit(bar_kfree + 8 * ks);
            if (j == it.ntiles - 1) tc::commit(bar_qfree + 8 * qb);
          }
          __syncwarp();
        }
      } else {
        for (int j = 0; j < it.ntiles; ++j, ++jt) {
          const int b = jt % kSBufs;  // S buffer holding P
          const int vs = jt & 1;      // V stage
          if (!(run = wait(bar_v + 8 * vs, (jt >> 1) & 1))) break;
          if (!(run = wait(bar_p + 8 * b, (jt / kSBufs) & 1))) break;
          // The first P V of an item overwrites O.  It needs P from every
          // softmax warp, which each writes only after reading out the
          // previous item's O, so bar_p orders that too.
          if (lane == 0) {
            tc::fence_after_sync();
            const uint32_t vb = sb + kVOff + vs * kTile;
            // O += P V: P of tokens 16kk .. 16kk + 15 sits in columns 8kk ..
            // 8kk + 7 of the S buffer (bf16 residuals 64 columns on) and meets
            // V rows 16kk .. 16kk + 15.
#pragma unroll
            for (int kk = 0; kk < kKv / 16; ++kk) {
              const uint32_t pcol = tmem + b * kKv + kk * 8u;
              const uint64_t vdesc = tc::smem_desc_sw128(vb + kk * 2u * kGroupBytes, 1024u, kGroupBytes);
              tc::mma_f16_ts(tO, pcol, vdesc, kIdescO, (j > 0 || kk > 0) ? 1u : 0u);
              if constexpr (kSplit) tc::mma_f16_ts(tO, pcol + 64u, vdesc, kIdescO, 1u);
            }
            tc::commit(bar_vfree + 8 * vs);
            tc::commit(bar_pfree + 8 * b);
          }
          __syncwarp();
        }
      }
      ++n;
    }
  } else if (warp < kSoftmaxWarps) {
    // -------------------------- softmax, 16 rows per warp, 2 rows per thread
    // Warp w reads TMEM lanes (tile rows) 32 (w % 4) + 16 (w / 4) .. + 15
    // with the 16-lane shapes: thread t holds rows r0 = base + t/4 and
    // r1 = r0 + 8, columns 2c, 2c + 1 (c = t % 4) of every 8-column group.
    // The four threads of a row are one quad of the warp, so the row max and
    // sum are two shuffles, one O accumulator serves the row and tensor
    // memory holds three S buffers.  P of the token pair (8i + 2c, + 1) goes
    // to column c + 4i (the A-operand layout), with the 16x128b shape.
    const int base = 32 * (warp & 3) + 16 * (warp >> 2);
    const int c = lane & 3;
    const uint32_t lane_off = static_cast<uint32_t>(base) << 16;
    bool run = true;
    int n = 0;
    int jt = 0;
    for (int k = 0; run; ++k) {
      int i;
      if (!(run = read_item(k, i))) break;
      if (i < 0) break;
      Item it;
      if (!item_at<BS>(a, i, it, tid == 0)) continue;
      int t_row[2], h_row[2], p_row[2];
      bool row_valid[2];
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int row = base + (lane >> 2) + 8 * r;
        t_row[r] = it.tok0 + row / G;  // chunk token of the row
        h_row[r] = row % G;
        row_valid[r] = t_row[r] < it.C;
        p_row[r] = it.L - it.C + t_row[r];  // >= L for rows past the chunk
      }
      float m_ref[2] = {-INFINITY, -INFINITY};  // reference maxima (log2 units)
      float l_sum[2] = {0.f, 0.f};              // this thread's 32 columns of each row
      for (int j = 0; j < it.ntiles; ++j, ++jt) {
        const int b = jt % kSBufs;
        if (!(run = wait(bar_s + 8 * b, (jt / kSBufs) & 1))) break;
        tc::fence_after_sync();
        float x[64];  // x[4g + 2r + e]: row r, token 8g + 2c + e
        {
          uint32_t rr[64];
          tc::ld_16x256b_x16(tmem + b * kKv + lane_off, rr);
          tc::wait_ld();
#pragma unroll
          for (int q = 0; q < 64; ++q) x[q] = __uint_as_float(rr[q]);
        }
        int lim[2];
#pragma unroll
        for (int r = 0; r < 2; ++r) lim[r] = min(p_row[r] + 1, it.L) - j * kKv;  // tokens < lim are visible
        if (lim[0] < kKv || lim[1] < kKv) {
#pragma unroll
          for (int g = 0; g < 16; ++g)
#pragma unroll
            for (int r = 0; r < 2; ++r)
#pragma unroll
              for (int e = 0; e < 2; ++e)
                x[4 * g + 2 * r + e] = 8 * g + 2 * c + e < lim[r] ? x[4 * g + 2 * r + e] : -INFINITY;
        }
        float alpha[2] = {1.f, 1.f};
        bool move_any = false;
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          float m0 = fmaxf(x[2 * r], x[2 * r + 1]), m1 = fmaxf(x[4 + 2 * r], x[4 + 2 * r + 1]);
#pragma unroll
          for (int g = 2; g < 16; g += 2) {
            m0 = max3(m0, x[4 * g + 2 * r], x[4 * g + 2 * r + 1]);
            m1 = max3(m1, x[4 * g + 4 + 2 * r], x[4 * g + 4 + 2 * r + 1]);
          }
          float mt = fmaxf(m0, m1);
          mt = fmaxf(mt, __shfl_xor_sync(kFullMask, mt, 1));
          mt = fmaxf(mt, __shfl_xor_sync(kFullMask, mt, 2));
          mt *= a.scale_log2;  // scale > 0: the max of the scaled scores
          if (mt > m_ref[r] + kLazyRescale) {
            alpha[r] = fast_exp2(m_ref[r] - mt);  // 0 while m_ref is -inf
            m_ref[r] = mt;
            l_sum[r] *= alpha[r];
            move_any = true;
          }
        }
        if (j > 0 && __any_sync(kFullMask, move_any)) {
          // O must hold P V(j-1) before it is rescaled; P V(j) needs this
          // warp's P(j), so nothing else writes O meanwhile.
          const int jp = jt - 1;
          if (!(run = wait(bar_pfree + 8 * (jp % kSBufs), (jp / kSBufs) & 1))) break;
          tc::fence_after_sync();
#pragma unroll
          for (int ch = 0; ch < 4; ++ch) {
            uint32_t o[16];
            tc::ld_16x256b_x4(tO + lane_off + 32u * ch, o);
            tc::wait_ld();
#pragma unroll
            for (int q = 0; q < 16; ++q) o[q] = __float_as_uint(__uint_as_float(o[q]) * alpha[(q >> 1) & 1]);
            tc::st_16x256b_x4(tO + lane_off + 32u * ch, o);
          }
          tc::wait_st();
        }
        // P into the S buffer (A operand of P V in tensor memory): high parts
        // in columns 0 .. 63, bf16 residuals in 64 .. 127; two halves of the
        // token range, so fewer values are live at once
        const float2 sc = make_float2(a.scale_log2, a.scale_log2);
        float2 nm[2];
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const float mr = m_ref[r] == -INFINITY ? 0.f : m_ref[r];  // no visible token yet: P = 0
          nm[r] = make_float2(-mr, -mr);
        }
        float2 ls[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          uint32_t hi[16], lo[16];  // [2 g' + r]: group 8 hf + g', row r
#pragma unroll
          for (int g2 = 0; g2 < 8; ++g2) {
            const int g = 8 * hf + g2;
#pragma unroll
            for (int r = 0; r < 2; ++r) {
              const float2 t = __ffma2_rn(make_float2(x[4 * g + 2 * r], x[4 * g + 2 * r + 1]), sc, nm[r]);
              const float2 p = make_float2(fast_exp2(t.x), fast_exp2(t.y));
              ls[r] = __fadd2_rn(ls[r], p);
              hi[2 * g2 + r] = Pack<T>::pack(p.x, p.y);
              if constexpr (kSplit) {
                const float2 q2 = __ffma2_rn(Pack<T>::unpack(hi[2 * g2 + r]), make_float2(-1.f, -1.f), p);
                lo[2 * g2 + r] = Pack<T>::pack(q2.x, q2.y);
              }
            }
          }
          const uint32_t pcol = tmem + b * kKv + lane_off + 32u * hf;
          tc::st_16x128b_x8(pcol, hi);
          if constexpr (kSplit) tc::st_16x128b_x8(pcol + 64u, lo);
        }
#pragma unroll
        for (int r = 0; r < 2; ++r) l_sum[r] += ls[r].x + ls[r].y;
        tc::wait_st();
        // V(j) landed; tokens past the context get zero rows, so that P = 0
        // never meets a NaN in stale shared memory
        const int valid_tok = min(kKv, it.L - j * kKv);
        if (valid_tok < kKv) {
          const int vs = jt & 1;
          if (!(run = wait(bar_v + 8 * vs, (jt >> 1) & 1))) break;
          uint8_t *vt = smem + kVOff + vs * kTile;
          for (int u = valid_tok * 16 + tid; u < kKv * 16; u += kSoftmaxThreads) {
            const int r = u >> 4, w = u & 15;  // token row, 16-byte unit of its 256 bytes
            *reinterpret_cast<uint4 *>(vt + (r >> 3) * kGroupBytes + (w >> 3) * 1024 + (r & 7) * 128 +
                                       (w & 7) * 16) = make_uint4(0u, 0u, 0u, 0u);
          }
          fence_proxy_async_smem();
        }
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_p + 8 * b);
      }
      if (!run) break;
      // ---- epilogue of the item: row sums over the quad, O / l, once the
      // item's last P V is done
      const int jl = jt - 1;
      if (!(run = wait(bar_pfree + 8 * (jl % kSBufs), (jl / kSBufs) & 1))) break;
      tc::fence_after_sync();
      float inv[2];
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        float L = l_sum[r];
        L += __shfl_xor_sync(kFullMask, L, 1);
        L += __shfl_xor_sync(kFullMask, L, 2);
        inv[r] = L > 0.f ? 1.f / L : 0.f;
      }
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
        uint32_t o[16];  // [4 g' + 2 r + e]: row r, column 32 ch + 8 g' + 2c + e
        tc::ld_16x256b_x4(tO + lane_off + 32u * ch, o);
        tc::wait_ld();
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          if (!row_valid[r]) continue;
          T *orow = static_cast<T *>(a.out) +
                    (static_cast<size_t>(it.t_begin + t_row[r]) * a.num_q_heads + it.g * G + h_row[r]) * kDim;
#pragma unroll
          for (int g2 = 0; g2 < 4; ++g2) {
            const float2 v = __fmul2_rn(make_float2(__uint_as_float(o[4 * g2 + 2 * r]), __uint_as_float(o[4 * g2 + 2 * r + 1])),
                                        make_float2(inv[r], inv[r]));
            *reinterpret_cast<uint32_t *>(orow + 32 * ch + 8 * g2 + 2 * c) = Pack<T>::pack(v.x, v.y);
          }
        }
      }
      ++n;
    }
  }

  // ---- teardown -----------------------------------------------------------
  tc::fence_before_sync();
  __syncthreads();
  if (*abort_flag) {
    // A wait ran out: report it, let the issued tensor-core work and the
    // loads still in flight finish (bounded) before TMEM and shared memory
    // are released.
    if (tid == 0) raise_flag(a.d_status, PKV_DEV_TIMEOUT);
    if ((warp == kMmaWarp || warp == kPvWarp) && lane == 0) tc::commit(bar_done);
    (void)mbar_wait(bar_done, 0);
    for (int i = 0; i < 2; ++i) {
      (void)mbar_wait(bar_q + 8 * i, 0);
      (void)mbar_wait(bar_q + 8 * i, 1);
      (void)mbar_wait(bar_k + 8 * i, 0);
      (void)mbar_wait(bar_k + 8 * i, 1);
      (void)mbar_wait(bar_v + 8 * i, 0);
      (void)mbar_wait(bar_v + 8 * i, 1);
    }
    __syncthreads();
  }
  if (warp == 0) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
}

// Rank-5 view of a pool [N][Hkv][B][D] (16-bit, D = 128) for one box per
// block: (64 elements, 8 rows, 2 halves of head_dim, B / 8 row groups,
// N * Hkv (block, head) pairs); the box is a whole block, landing as
// [row group][half][8 rows][128 B].
pkv_status encode_grouped_map(CUtensorMap *map, const void *pool, const pkv_cache_desc &c) {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
    void *f = nullptr;
    cudaDriverEntryPointQueryResult q{};
    return (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
               ? reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f)
               : nullptr;
  }();
  if (fn == nullptr) return PKV_ERR_CUDA;
  const cuuint64_t row = static_cast<cuuint64_t>(c.head_dim) * 2;
  cuuint64_t dims[5] = {64, 8, 2, static_cast<cuuint64_t>(c.block_size / 8),
                        static_cast<cuuint64_t>(c.num_blocks) * c.num_kv_heads};
  cuuint64_t strides[4] = {row, 128, 8 * row, static_cast<cuuint64_t>(c.block_size) * row};
  cuuint32_t box[5] = {64, 8, 2, static_cast<cuuint32_t>(c.block_size / 8), 1};
  cuuint32_t estride[5] = {1, 1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT16, 5, const_cast<void *>(pool), dims, strides, box, estride,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? PKV_OK : PKV_ERR_CUDA;
}

template <typename T>
pkv_status launch_prefill_bs(int block_size, dim3 grid, const CUtensorMap &tq, const CUtensorMap &tk,
                             const CUtensorMap &tv, const PrefillArgs &args, cudaStream_t stream) {
#define PKV_PREFILL_CASE(BSV)                                                               \
  case BSV: {                                                                               \
    static std::atomic<uint64_t> smem_set{0};                                               \
    return launch_with_smem(paged_prefill_kernel<T, BSV>, grid, dim3(kThreads),             \
                            PrefillTune<T>::kSmem, stream, &smem_set, tq, tk, tv, args);    \
  }
  switch (block_size) {
    PKV_PREFILL_CASE(8)
    PKV_PREFILL_CASE(16)
    PKV_PREFILL_CASE(32)
    PKV_PREFILL_CASE(64)
  }
#undef PKV_PREFILL_CASE
  return PKV_ERR_BAD_SHAPE;
}

}  // namespace
}  // namespace pkv

extern "C" pkv_status pkv_paged_prefill(void *out, const void *query, const void *k_cache,
                                        const void *v_cache, pkv_cache_desc cache,
                                        const int32_t *block_tables, int32_t max_blocks_per_seq,
                                        const int32_t *query_start, const int32_t *context_lens,
                                        int32_t num_seqs, int32_t num_tokens,
                                        int32_t max_query_len, int32_t num_q_heads, float scale,
                                        void *workspace, size_t workspace_bytes,
                                        int32_t *d_status, pkv_stream_t stream) {
  using namespace pkv;
  pkv_status st = check_cache_desc(cache);
  if (st != PKV_OK) return st;
  if (!is_16bit(cache.dtype)) return PKV_ERR_BAD_DTYPE;
  if (cache.head_dim != kDim) return PKV_ERR_BAD_SHAPE;
  if (num_seqs < 0 || num_tokens < 0 || max_query_len < 0 || num_q_heads < 1 ||
      max_blocks_per_seq < 1)
    return PKV_ERR_BAD_SHAPE;
  if (num_q_heads % cache.num_kv_heads != 0) return PKV_ERR_BAD_SHAPE;
  const int G = num_q_heads / cache.num_kv_heads;
  if (G > 16 || (kRows % G) != 0) return PKV_ERR_BAD_SHAPE;
  if (!(scale > 0.f) || !(scale < INFINITY)) return PKV_ERR_BAD_SHAPE;
  if (num_seqs == 0 || num_tokens == 0 || max_query_len == 0) return PKV_OK;
  if (cache.num_kv_heads > 65535) return PKV_ERR_TOO_LARGE;
  if (!out || !query || !k_cache || !v_cache || !block_tables || !query_start || !context_lens)
    return PKV_ERR_NULL_POINTER;
  if (!aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(query, 16) || !aligned(out, 16) ||
      !aligned(block_tables, 4) || !aligned(query_start, 4) || !aligned(context_lens, 4) ||
      !aligned(workspace, 4))
    return PKV_ERR_MISALIGNED;
  if (workspace != nullptr && workspace_bytes < PKV_PREFILL_WORKSPACE_BYTES) return PKV_ERR_WORKSPACE;
  const long long qtiles = (static_cast<long long>(max_query_len) * G + kRows - 1) / kRows;
  const long long items = qtiles * cache.num_kv_heads * num_seqs;
  if (items > 2147483647ll) return PKV_ERR_TOO_LARGE;
  if ((st = check_device()) != PKV_OK) return st;

  CUtensorMap tq, tk, tv;
  if ((st = encode_query_map(&tq, query, num_tokens, num_q_heads, kDim, G)) != PKV_OK) return st;
  if ((st = encode_grouped_map(&tk, k_cache, cache)) != PKV_OK) return st;
  if ((st = encode_grouped_map(&tv, v_cache, cache)) != PKV_OK) return st;

  PrefillArgs args{};
  args.out = out;
  args.block_tables = block_tables;
  args.query_start = query_start;
  args.context_lens = context_lens;
  args.d_status = d_status;
  args.num_tokens = num_tokens;
  args.max_blocks_per_seq = max_blocks_per_seq;
  args.num_q_heads = num_q_heads;
  args.group = G;
  args.num_blocks = cache.num_blocks;
  args.num_kv_heads = cache.num_kv_heads;
  args.num_seqs = num_seqs;
  args.qtiles = static_cast<int>(qtiles);
  args.items = static_cast<int>(items);
  args.scale_log2 = scale * 1.4426950408889634f;
  // Persistent grid: one CTA per SM (the kernel's shared memory and tensor
  // memory allow one), each walking its share of the items.
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1)
    return PKV_ERR_CUDA;
  dim3 grid(static_cast<unsigned>(items < sms ? items : sms));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (workspace != nullptr) {
    // the item counter starts at zero for this launch
    if (cudaMemsetAsync(workspace, 0, sizeof(unsigned int), s) != cudaSuccess) return PKV_ERR_CUDA;
    args.ticket = static_cast<unsigned int *>(workspace);
  }
  return cache.dtype == PKV_BF16 ? launch_prefill_bs<__nv_bfloat16>(cache.block_size, grid, tq, tk, tv, args, s)
                                 : launch_prefill_bs<__half>(cache.block_size, grid, tq, tk, tv, args, s);
}
