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
// How (B200 design):
//   * One CTA per (kv head g, sequence s, partition p).  All query heads of
//     the group g share each K/V block, so every block is read from HBM once.
//   * Every warp streams its own share of the partition's blocks (blocks
//     w, w + WARPS, ...) through a private ring of NST shared-memory stages.
//     One stage = one block's K tile and V tile, each loaded by tiled TMA
//     (rank-4 tensor map over [N][Hkv][B][D], box 64 x B, 128-byte swizzle)
//     and counted on an mbarrier.  Block Table entries are fetched 32 at a
//     time per warp with one coalesced load, prefetched a window ahead.
//   * Scores S^T = Q K^T and the update O += P V run on mma.sync.m16n8k16
//     (fp16/bf16 in, fp32 accumulate) with the group's query heads on M, so
//     the score accumulator fragment is already the A operand of P V.  P is
//     split into a 16-bit high part and a 16-bit residual (two MMAs), which
//     keeps the probabilities at about fp32 precision.  Tensor cores are used
//     to keep instruction issue far below the HBM rate, not for throughput.
//   * Online softmax in the log2 domain (scores pre-multiplied by
//     scale*log2 e), max/sum reduced over the 4 lanes that share a row with
//     shuffles; the output is rescaled only when some row's max grows.
//   * At the end the warps' (m, l, O) states are merged through shared
//     memory; a single-partition sequence writes its output directly, other
//     partitions write (m, l, unnormalised O) to the workspace and count
//     themselves in on a per-(sequence, kv head) counter; the last partition
//     to arrive merges them all by log-sum-exp and resets the counter.  Only
//     splits of more than kFuseMaxParts partitions use the separate merge
//     kernel.
#include <algorithm>

#include "pkv_device.cuh"
#include "pkv_host.h"

namespace pkv {
namespace {

constexpr uint32_t kFull = 0xffffffffu;
constexpr float kLog2e = 1.4426950408889634f;

struct DecodeArgs {
  const void *query;
  void *out;
  const int32_t *block_tables;
  const int32_t *context_lens;
  float *ws_m;  // [S][Hq][max_parts]
  float *ws_l;  // [S][Hq][max_parts]
  float *ws_o;  // [S][Hq][max_parts][D]
  int32_t *counters;  // [S][Hkv] arrivals of split partitions (zero between calls)
  int32_t *d_status;
  int max_blocks_per_seq;
  int num_q_heads;
  int num_kv_heads;
  int group;       // query heads per kv head
  int num_blocks;  // pool size
  int len_limit;   // largest valid context length
  int part_blocks; // blocks per partition
  int max_parts;
  float scale_log2;  // scale * log2(e)
};

// Launch shape per (head_dim, block_size): warps per CTA and ring depth,
// chosen so a CTA's rings take about 64 KB of shared memory and three CTAs fit
// on an SM (measured best on B200 for 8..64-token blocks).
template <int D, int BS>
struct Tune {
  static constexpr int kStage = 2 * BS * D * 2;  // bytes of one K+V stage
  static constexpr int kWarps = kStage >= 16384 ? 2 : 4;
  static constexpr int kFit = 65536 / (kWarps * kStage);
  static constexpr int kStages = kFit < 1 ? 1 : (kFit > 4 ? 4 : kFit);
};

// Split sequences with at most this many partitions are merged inside the
// attention kernel by the last CTA to finish; longer splits use the merge kernel.
constexpr int kFuseMaxParts = 32;

template <int D, int BS, int WARPS, int NST>
struct Layout {
  static constexpr int kBoxes = D / 64;                     // TMA boxes per tile
  static constexpr int kBoxBytes = BS * 128;                // BS rows of 128 B
  static constexpr int kTileBytes = kBoxes * kBoxBytes;     // one K (or V) tile
  static constexpr int kStageBytes = 2 * kTileBytes;        // K + V
  static constexpr int kRingBytes = WARPS * NST * kStageBytes;
  static constexpr int kMergeBytes = WARPS * 16 * (D + 2) * 4;
  static constexpr int kDataBytes = kRingBytes > kMergeBytes ? kRingBytes : kMergeBytes;
  static constexpr int kBarOff = (kDataBytes + 1023) / 1024 * 1024;
  static constexpr int kNvOff = kBarOff + WARPS * NST * 8;
  static constexpr int kSmem = kNvOff + WARPS * NST * 4 + 1024;  // + base alignment slack
  static constexpr int kNT = BS / 8;  // 8-token column tiles per block
  static constexpr int kDT = D / 8;   // 8-wide column tiles of the output
  static constexpr int kKS = D / 16;  // 16-deep steps of the score product
};

// Byte offset of 16-byte chunk `chunk` (= d / 8) of token row `tok` inside a
// tile of D/64 boxes, each BS rows x 128 B, written by TMA with the 128-byte
// swizzle (chunk index XOR row index within each 8-row, 1024-byte group).
template <int BS>
__device__ __forceinline__ uint32_t tile_off(int tok, int chunk) {
  return static_cast<uint32_t>((chunk >> 3) * (BS * 128) + tok * 128 +
                               (((chunk & 7) ^ (tok & 7)) << 4));
}

template <typename T, int D, int BS, int WARPS, int NST, bool BIG>
__global__ void __launch_bounds__(WARPS * 32)
    paged_decode_kernel(const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, const DecodeArgs a) {
  using Lt = Layout<D, BS, WARPS, NST>;
  using MMA = Mma<T>;
  using PK = Pack<T>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

  const int g = blockIdx.x;
  const int s = blockIdx.y;
  const int part = blockIdx.z;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int G = a.group;

  // ---- sequence bounds -------------------------------------------------
  int len = a.context_lens[s];
  if (len < 0 || len > a.len_limit) {
    if (threadIdx.x == 0 && g == 0 && part == 0) raise_flag(a.d_status, PKV_DEV_BAD_LEN);
    len = len < 0 ? 0 : a.len_limit;
  }
  const int nb = (len + BS - 1) / BS;
  const int nparts = nb > a.part_blocks ? (nb + a.part_blocks - 1) / a.part_blocks : 1;
  if (part >= nparts) return;  // uniform over the CTA, before any barrier
  const int b0 = part * a.part_blocks;
  const int nblk = min(nb - b0, a.part_blocks);
  const int tail_nv = len - (nb - 1) * BS;  // valid tokens of the sequence's last block
  const int cnt = nblk > warp ? (nblk - warp + WARPS - 1) / WARPS : 0;

  // ---- per-warp ring and barriers --------------------------------------
  const uint32_t ring = smem_addr(smem) + warp * NST * Lt::kStageBytes;
  const uint32_t bars = smem_addr(smem + Lt::kBarOff) + warp * NST * 8;
  volatile int *stage_nv = reinterpret_cast<volatile int *>(smem + Lt::kNvOff) + warp * NST;
  if (lane == 0) {
#pragma unroll
    for (int st = 0; st < NST; ++st) mbar_init(bars + 8 * st, 1);
    fence_barrier_init();
    prefetch_tensormap(&tm_k);
    prefetch_tensormap(&tm_v);
  }
  __syncwarp();

  // ---- query fragments (A operand: rows = query heads of the group) ----
  const int r = lane >> 2;        // fragment row of this lane
  const int c2 = (lane & 3) * 2;  // fragment column pair of this lane
  const uint32_t *q32 = reinterpret_cast<const uint32_t *>(
      static_cast<const T *>(a.query) +
      (static_cast<size_t>(s) * a.num_q_heads + static_cast<size_t>(g) * G) * D);
  uint32_t qa0[Lt::kKS], qa1[Lt::kKS], qa2[Lt::kKS], qa3[Lt::kKS];
#pragma unroll
  for (int kk = 0; kk < Lt::kKS; ++kk) {
    qa0[kk] = r < G ? q32[(r * D + 16 * kk + c2) >> 1] : 0u;
    qa2[kk] = r < G ? q32[(r * D + 16 * kk + 8 + c2) >> 1] : 0u;
    if constexpr (BIG) {
      qa1[kk] = r + 8 < G ? q32[((r + 8) * D + 16 * kk + c2) >> 1] : 0u;
      qa3[kk] = r + 8 < G ? q32[((r + 8) * D + 16 * kk + 8 + c2) >> 1] : 0u;
    } else {
      qa1[kk] = 0u;
      qa3[kk] = 0u;
    }
  }

  // ---- Block Table window: lane j holds the id of block 32*w + j ---------
  const int32_t *trow = a.block_tables + static_cast<size_t>(s) * a.max_blocks_per_seq + b0 + warp;
  auto load_window = [&](int w) -> int {
    const int k = (w << 5) + lane;
    return k < cnt ? __ldg(trow + static_cast<size_t>(k) * WARPS) : 0;
  };
  int win_cur = load_window(0);
  int win_next = cnt > 32 ? load_window(1) : 0;

  const uint64_t policy = l2_evict_first_policy();
  auto issue = [&](int k) {
    if ((k & 31) == 0 && k != 0) {
      win_cur = win_next;
      win_next = load_window((k >> 5) + 1);
    }
    const int id = __shfl_sync(kFull, win_cur, k & 31);
    if (lane == 0) {
      const int st = k % NST;
      const uint32_t bar = bars + 8 * st;
      const int blk = b0 + warp + k * WARPS;
      if (static_cast<unsigned>(id) < static_cast<unsigned>(a.num_blocks)) {
        stage_nv[st] = (blk == nb - 1) ? tail_nv : BS;
        fence_proxy_async_smem();
        mbar_arrive_expect_tx(bar, Lt::kStageBytes);
        const uint32_t dst = ring + st * Lt::kStageBytes;
#pragma unroll
        for (int bx = 0; bx < Lt::kBoxes; ++bx) {
          tma_load_4d(dst + bx * Lt::kBoxBytes, &tm_k, bar, bx * 64, 0, g, id, policy);
          tma_load_4d(dst + Lt::kTileBytes + bx * Lt::kBoxBytes, &tm_v, bar, bx * 64, 0, g, id,
                      policy);
        }
      } else {
        raise_flag(a.d_status, PKV_DEV_BAD_BLOCK);
        stage_nv[st] = 0;  // the whole block is masked
        mbar_arrive(bar);
      }
    }
  };

  int kp = 0;
  {
    const int pro = cnt < NST ? cnt : NST;
    for (; kp < pro; ++kp) issue(kp);
  }

  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  float o[Lt::kDT][4];
#pragma unroll
  for (int dt = 0; dt < Lt::kDT; ++dt) o[dt][0] = o[dt][1] = o[dt][2] = o[dt][3] = 0.f;

  const int mi = lane >> 3;  // ldmatrix: which 8x8 matrix this lane addresses
  const int ri = lane & 7;   // ldmatrix: which row of it
  int k = 0;
  bool ok = true;
  for (; k < cnt; ++k) {
    const int st = k % NST;
    ok = __all_sync(kFull, mbar_wait(bars + 8 * st, (k / NST) & 1));
    if (!ok) break;
    const int nv = stage_nv[st];
    const uint32_t kb = ring + st * Lt::kStageBytes;
    const uint32_t vb = kb + Lt::kTileBytes;

    // ---- S^T[16 x BS] = Q[16 x D] . K^T --------------------------------
    float sc[Lt::kNT][4];
#pragma unroll
    for (int nt = 0; nt < Lt::kNT; ++nt) sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
    if constexpr (BS >= 16) {
#pragma unroll
      for (int kk = 0; kk < Lt::kKS; ++kk) {
#pragma unroll
        for (int tp = 0; tp < BS / 16; ++tp) {
          uint32_t b0r, b1r, b2r, b3r;
          ldsm_x4(kb + tile_off<BS>(tp * 16 + ri + ((mi >> 1) << 3), 2 * kk + (mi & 1)), b0r, b1r,
                  b2r, b3r);
          MMA::k16(sc[2 * tp], qa0[kk], qa1[kk], qa2[kk], qa3[kk], b0r, b1r);
          MMA::k16(sc[2 * tp + 1], qa0[kk], qa1[kk], qa2[kk], qa3[kk], b2r, b3r);
        }
      }
    } else {
#pragma unroll
      for (int kk = 0; kk < Lt::kKS; kk += 2) {
        uint32_t b0r, b1r, b2r, b3r;
        ldsm_x4(kb + tile_off<BS>(ri, 2 * kk + mi), b0r, b1r, b2r, b3r);
        MMA::k16(sc[0], qa0[kk], qa1[kk], qa2[kk], qa3[kk], b0r, b1r);
        MMA::k16(sc[0], qa0[kk + 1], qa1[kk + 1], qa2[kk + 1], qa3[kk + 1], b2r, b3r);
      }
    }

    // ---- scale, mask past the context, online softmax ------------------
    const bool partial = nv < BS;
#pragma unroll
    for (int nt = 0; nt < Lt::kNT; ++nt)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float v = sc[nt][j] * a.scale_log2;
        if (partial && nt * 8 + c2 + (j & 1) >= nv) v = -INFINITY;
        sc[nt][j] = v;
      }
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < Lt::kNT; ++nt) {
      mx0 = fmaxf(mx0, fmaxf(sc[nt][0], sc[nt][1]));
      if constexpr (BIG) mx1 = fmaxf(mx1, fmaxf(sc[nt][2], sc[nt][3]));
    }
    mx0 = fmaxf(mx0, __shfl_xor_sync(kFull, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(kFull, mx0, 2));
    const float mn0 = fmaxf(m0, mx0);
    const float base0 = mn0 == -INFINITY ? 0.f : mn0;
    const float al0 = fast_exp2(m0 - base0);
    m0 = mn0;
    float al1 = 1.f, base1 = 0.f;
    if constexpr (BIG) {
      mx1 = fmaxf(mx1, __shfl_xor_sync(kFull, mx1, 1));
      mx1 = fmaxf(mx1, __shfl_xor_sync(kFull, mx1, 2));
      const float mn1 = fmaxf(m1, mx1);
      base1 = mn1 == -INFINITY ? 0.f : mn1;
      al1 = fast_exp2(m1 - base1);
      m1 = mn1;
    }
    float rs0 = 0.f, rs1 = 0.f;
#pragma unroll
    for (int nt = 0; nt < Lt::kNT; ++nt) {
      sc[nt][0] = fast_exp2(sc[nt][0] - base0);
      sc[nt][1] = fast_exp2(sc[nt][1] - base0);
      rs0 += sc[nt][0] + sc[nt][1];
      if constexpr (BIG) {
        sc[nt][2] = fast_exp2(sc[nt][2] - base1);
        sc[nt][3] = fast_exp2(sc[nt][3] - base1);
        rs1 += sc[nt][2] + sc[nt][3];
      }
    }
    l0 = l0 * al0 + rs0;
    if constexpr (BIG) l1 = l1 * al1 + rs1;
    const bool moved = BIG ? (al0 != 1.f || al1 != 1.f) : (al0 != 1.f);
    if (__any_sync(kFull, moved)) {
#pragma unroll
      for (int dt = 0; dt < Lt::kDT; ++dt) {
        o[dt][0] *= al0;
        o[dt][1] *= al0;
        if constexpr (BIG) {
          o[dt][2] *= al1;
          o[dt][3] *= al1;
        }
      }
    }

    // ---- O[16 x D] += P[16 x BS] . V ------------------------------------
    if constexpr (BS >= 16) {
#pragma unroll
      for (int tp = 0; tp < BS / 16; ++tp) {
        const uint32_t h0 = PK::pack(sc[2 * tp][0], sc[2 * tp][1]);
        const uint32_t h2 = PK::pack(sc[2 * tp + 1][0], sc[2 * tp + 1][1]);
        const float2 f0 = PK::unpack(h0);
        const float2 f2 = PK::unpack(h2);
        const uint32_t e0 = PK::pack(sc[2 * tp][0] - f0.x, sc[2 * tp][1] - f0.y);
        const uint32_t e2 = PK::pack(sc[2 * tp + 1][0] - f2.x, sc[2 * tp + 1][1] - f2.y);
        uint32_t h1 = 0u, h3 = 0u, e1 = 0u, e3 = 0u;
        if constexpr (BIG) {
          h1 = PK::pack(sc[2 * tp][2], sc[2 * tp][3]);
          h3 = PK::pack(sc[2 * tp + 1][2], sc[2 * tp + 1][3]);
          const float2 f1 = PK::unpack(h1);
          const float2 f3 = PK::unpack(h3);
          e1 = PK::pack(sc[2 * tp][2] - f1.x, sc[2 * tp][3] - f1.y);
          e3 = PK::pack(sc[2 * tp + 1][2] - f3.x, sc[2 * tp + 1][3] - f3.y);
        }
        const bool vmask = partial && (tp * 16 + 16 > nv);
        const int t0 = tp * 16 + c2;
        const uint32_t mlo = (t0 < nv ? 0x0000ffffu : 0u) | (t0 + 1 < nv ? 0xffff0000u : 0u);
        const uint32_t mhi = (t0 + 8 < nv ? 0x0000ffffu : 0u) | (t0 + 9 < nv ? 0xffff0000u : 0u);
#pragma unroll
        for (int dp = 0; dp < Lt::kDT / 2; ++dp) {
          uint32_t v0, v1, v2, v3;
          ldsm_x4_trans(vb + tile_off<BS>(tp * 16 + ri + ((mi & 1) << 3), 2 * dp + (mi >> 1)), v0,
                        v1, v2, v3);
          if (vmask) {
            v0 &= mlo;
            v2 &= mlo;
            v1 &= mhi;
            v3 &= mhi;
          }
          MMA::k16(o[2 * dp], h0, h1, h2, h3, v0, v1);
          MMA::k16(o[2 * dp], e0, e1, e2, e3, v0, v1);
          MMA::k16(o[2 * dp + 1], h0, h1, h2, h3, v2, v3);
          MMA::k16(o[2 * dp + 1], e0, e1, e2, e3, v2, v3);
        }
      }
    } else {
      const uint32_t h0 = PK::pack(sc[0][0], sc[0][1]);
      const float2 f0 = PK::unpack(h0);
      const uint32_t e0 = PK::pack(sc[0][0] - f0.x, sc[0][1] - f0.y);
      uint32_t h1 = 0u, e1 = 0u;
      if constexpr (BIG) {
        h1 = PK::pack(sc[0][2], sc[0][3]);
        const float2 f1 = PK::unpack(h1);
        e1 = PK::pack(sc[0][2] - f1.x, sc[0][3] - f1.y);
      }
      const uint32_t mlo = (c2 < nv ? 0x0000ffffu : 0u) | (c2 + 1 < nv ? 0xffff0000u : 0u);
#pragma unroll
      for (int dq = 0; dq < Lt::kDT / 4; ++dq) {
        uint32_t v[4];
        ldsm_x4_trans(vb + tile_off<BS>(ri, 4 * dq + mi), v[0], v[1], v[2], v[3]);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          if (partial) v[j] &= mlo;
          MMA::k8(o[4 * dq + j], h0, h1, v[j]);
          MMA::k8(o[4 * dq + j], e0, e1, v[j]);
        }
      }
    }

    __syncwarp();
    if (kp < cnt) {
      issue(kp);
      ++kp;
    }
  }
  if (!ok) {
    if (lane == 0) raise_flag(a.d_status, PKV_DEV_TIMEOUT);
    // Let the copies still in flight land before the shared memory is reused.
    for (int j = k; j < kp; ++j) (void)mbar_wait(bars + 8 * (j % NST), (j / NST) & 1);
  }

  // ---- merge the warps' softmax states ---------------------------------
  l0 += __shfl_xor_sync(kFull, l0, 1);
  l0 += __shfl_xor_sync(kFull, l0, 2);
  if constexpr (BIG) {
    l1 += __shfl_xor_sync(kFull, l1, 1);
    l1 += __shfl_xor_sync(kFull, l1, 2);
  }
  __syncthreads();  // every ring is drained; reuse it for the merge
  float *mo = reinterpret_cast<float *>(smem);  // [WARPS][16][D]
  float *mm = mo + WARPS * 16 * D;              // [WARPS][16]
  float *ml = mm + WARPS * 16;                  // [WARPS][16]
  if (r < G) {
#pragma unroll
    for (int dt = 0; dt < Lt::kDT; ++dt)
      *reinterpret_cast<float2 *>(&mo[(warp * 16 + r) * D + dt * 8 + c2]) =
          make_float2(o[dt][0], o[dt][1]);
    if ((lane & 3) == 0) {
      mm[warp * 16 + r] = m0;
      ml[warp * 16 + r] = l0;
    }
  }
  if constexpr (BIG) {
    if (r + 8 < G) {
#pragma unroll
      for (int dt = 0; dt < Lt::kDT; ++dt)
        *reinterpret_cast<float2 *>(&mo[(warp * 16 + r + 8) * D + dt * 8 + c2]) =
            make_float2(o[dt][2], o[dt][3]);
      if ((lane & 3) == 0) {
        mm[warp * 16 + r + 8] = m1;
        ml[warp * 16 + r + 8] = l1;
      }
    }
  }
  __syncthreads();

  const bool single = nparts == 1;
  T *out = static_cast<T *>(a.out);
  for (int e = threadIdx.x; e < G * D; e += WARPS * 32) {
    const int h = e / D;
    const int d = e - h * D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < WARPS; ++w) M = fmaxf(M, mm[w * 16 + h]);
    float acc = 0.f, lsum = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < WARPS; ++w) {
        const float wt = fast_exp2(mm[w * 16 + h] - M);
        acc += wt * mo[(w * 16 + h) * D + d];
        lsum += wt * ml[w * 16 + h];
      }
    }
    const size_t row = static_cast<size_t>(s) * a.num_q_heads + static_cast<size_t>(g) * G + h;
    if (single) {
      out[row * D + d] = PK::from_float(lsum > 0.f ? acc / lsum : 0.f);
    } else {
      const size_t idx = row * a.max_parts + part;
      a.ws_o[idx * D + d] = acc;
      if (d == 0) {
        a.ws_m[idx] = M;
        a.ws_l[idx] = lsum;
      }
    }
  }
  if (single || nparts > kFuseMaxParts) return;

  // ---- split sequence: the last of its partitions to finish merges them ---
  __shared__ int s_last;
  __syncthreads();  // this CTA's partials are written
  if (threadIdx.x == 0) {
    __threadfence();  // publish them before counting this partition in
    int *cnt = a.counters + static_cast<size_t>(s) * a.num_kv_heads + g;
    const int last = atomicAdd(cnt, 1) == nparts - 1;
    if (last) {
      *cnt = 0;  // leave the counter at zero for the next call
      __threadfence();
    }
    s_last = last;
  }
  __syncthreads();
  if (!s_last) return;
  for (int e = threadIdx.x; e < G * D; e += WARPS * 32) {
    const int h = e / D;
    const int d = e - h * D;
    const size_t row = static_cast<size_t>(s) * a.num_q_heads + static_cast<size_t>(g) * G + h;
    const size_t base = row * a.max_parts;
    float M = -INFINITY;
    for (int p = 0; p < nparts; ++p) M = fmaxf(M, __ldcg(a.ws_m + base + p));
    float acc = 0.f, lsum = 0.f;
    if (M != -INFINITY) {
      for (int p = 0; p < nparts; ++p) {
        const float wt = fast_exp2(__ldcg(a.ws_m + base + p) - M);
        acc += wt * __ldcg(a.ws_o + (base + p) * D + d);
        lsum += wt * __ldcg(a.ws_l + base + p);
      }
    }
    out[row * D + d] = PK::from_float(lsum > 0.f ? acc / lsum : 0.f);
  }
}

// ---------------------------------------------------------------------------
// Log-sum-exp merge of the partitions of each (sequence, query head):
//   M = max_p m_p,  w_p = 2^(m_p - M),  out = sum_p w_p o_p / sum_p w_p l_p.
// ---------------------------------------------------------------------------
struct CombineArgs {
  void *out;
  const int32_t *context_lens;
  const float *ws_m;
  const float *ws_l;
  const float *ws_o;
  int num_q_heads;
  int block_size;
  int len_limit;
  int part_blocks;
  int max_parts;
};

template <int NT>
__device__ __forceinline__ float block_reduce(float v, bool is_max, float *scratch) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const float x = __shfl_xor_sync(kFull, v, off);
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
  __shared__ float scratch[D / 32];
  const int h = blockIdx.x;
  const int s = blockIdx.y;
  int len = c.context_lens[s];
  len = len < 0 ? 0 : (len > c.len_limit ? c.len_limit : len);
  const int nb = (len + c.block_size - 1) / c.block_size;
  const int nparts = nb > c.part_blocks ? (nb + c.part_blocks - 1) / c.part_blocks : 1;
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
  static_cast<T *>(c.out)[row * D + threadIdx.x] =
      Pack<T>::from_float(lsum > 0.f ? total / lsum : 0.f);
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
int auto_part_blocks(int block_size) {
  // 512-token partitions (at least 8 blocks): 32 blocks of 16 tokens, 16 of 32.
  return block_size >= 64 ? 8 : 512 / block_size;
}

bool valid_block_size(int bs) { return bs == 8 || bs == 16 || bs == 32 || bs == 64; }

struct Plan {
  int part_blocks;
  int max_parts;
  size_t ws_bytes;
};

// Resolve the partitioning; false for invalid arguments.
bool make_plan(int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
               int32_t block_size, int32_t max_context_len, int32_t partition_size, Plan *plan) {
  if (!valid_block_size(block_size) || num_seqs < 0 || num_q_heads < 1 || num_kv_heads < 1 ||
      head_dim < 1 || max_context_len < 0 || partition_size < 0)
    return false;
  int part_blocks;
  if (partition_size == 0) {
    part_blocks = auto_part_blocks(block_size);
  } else {
    if (partition_size % block_size != 0) return false;
    part_blocks = partition_size / block_size;
  }
  const long long nb_max = (static_cast<long long>(max_context_len) + block_size - 1) / block_size;
  const long long parts = nb_max > part_blocks ? (nb_max + part_blocks - 1) / part_blocks : 1;
  plan->part_blocks = part_blocks;
  plan->max_parts = static_cast<int>(std::min<long long>(parts, 1ll << 30));
  // partials (o, m, l) then one arrival counter per (sequence, kv head)
  plan->ws_bytes = parts > 1 ? static_cast<size_t>(num_seqs) * num_q_heads * parts *
                                       (static_cast<size_t>(head_dim) + 2) * sizeof(float) +
                                   static_cast<size_t>(num_seqs) * num_kv_heads * sizeof(int32_t)
                             : 0;
  return true;
}

template <typename T, int D, int BS, bool BIG>
pkv_status launch_decode(const CUtensorMap &tmk, const CUtensorMap &tmv, const DecodeArgs &args,
                         int num_kv_heads, int num_seqs, cudaStream_t stream) {
  constexpr int WARPS = Tune<D, BS>::kWarps;
  constexpr int NST = Tune<D, BS>::kStages;
  using Lt = Layout<D, BS, WARPS, NST>;
  auto kern = paged_decode_kernel<T, D, BS, WARPS, NST, BIG>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Lt::kSmem) !=
      cudaSuccess)
    return PKV_ERR_CUDA;
  dim3 grid(static_cast<unsigned>(num_kv_heads), static_cast<unsigned>(num_seqs),
            static_cast<unsigned>(args.max_parts));
  kern<<<grid, WARPS * 32, Lt::kSmem, stream>>>(tmk, tmv, args);
  return launch_status();
}

template <typename T, int D>
pkv_status launch_for_dim(int block_size, bool big, const CUtensorMap &tmk, const CUtensorMap &tmv,
                          const DecodeArgs &args, int num_kv_heads, int num_seqs,
                          cudaStream_t stream) {
#define PKV_BS_CASE(BSV)                                                                       \
  case BSV:                                                                                    \
    return big ? launch_decode<T, D, BSV, true>(tmk, tmv, args, num_kv_heads, num_seqs, stream) \
               : launch_decode<T, D, BSV, false>(tmk, tmv, args, num_kv_heads, num_seqs, stream);
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
  lse_combine_kernel<T, D><<<grid, D, 0, stream>>>(c);
  return launch_status();
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

extern "C" pkv_status pkv_paged_attention_decode(
    void *out, const void *query, const void *k_cache, const void *v_cache, pkv_cache_desc cache,
    const int32_t *block_tables, int32_t max_blocks_per_seq, const int32_t *context_lens,
    int32_t num_seqs, int32_t num_q_heads, int32_t max_context_len, float scale,
    int32_t partition_size, void *workspace, size_t workspace_bytes, int32_t *d_status,
    pkv_stream_t stream) {
  using namespace pkv;
  pkv_status st = check_cache_desc(cache);
  if (st != PKV_OK) return st;
  if (num_seqs < 0 || max_context_len < 0 || max_blocks_per_seq < 1 || num_q_heads < 1)
    return PKV_ERR_BAD_SHAPE;
  if (num_q_heads % cache.num_kv_heads != 0 || num_q_heads / cache.num_kv_heads > 16)
    return PKV_ERR_BAD_SHAPE;
  if (!(scale > 0.f) || !(scale < INFINITY)) return PKV_ERR_BAD_SHAPE;
  if (partition_size < 0 || (partition_size > 0 && partition_size % cache.block_size != 0))
    return PKV_ERR_BAD_PARTITION;
  if (num_seqs == 0) return PKV_OK;
  if (num_seqs > 65535) return PKV_ERR_TOO_LARGE;
  if (!out || !query || !k_cache || !v_cache || !block_tables || !context_lens)
    return PKV_ERR_NULL_POINTER;
  if (!aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(query, 4) || !aligned(out, 4) ||
      !aligned(block_tables, 4) || !aligned(context_lens, 4))
    return PKV_ERR_MISALIGNED;

  Plan plan;
  if (!make_plan(num_seqs, num_q_heads, cache.num_kv_heads, cache.head_dim, cache.block_size,
                 max_context_len, partition_size, &plan))
    return PKV_ERR_BAD_PARTITION;
  if (plan.max_parts > 65535) return PKV_ERR_TOO_LARGE;
  if (plan.ws_bytes > 0) {
    if (workspace == nullptr || workspace_bytes < plan.ws_bytes) return PKV_ERR_WORKSPACE;
    if (!aligned(workspace, 16)) return PKV_ERR_MISALIGNED;
  }
  if ((st = check_device()) != PKV_OK) return st;

  CUtensorMap tmk, tmv;
  if ((st = encode_cache_map(&tmk, k_cache, cache)) != PKV_OK) return st;
  if ((st = encode_cache_map(&tmv, v_cache, cache)) != PKV_OK) return st;

  DecodeArgs args{};
  args.query = query;
  args.out = out;
  args.block_tables = block_tables;
  args.context_lens = context_lens;
  const size_t rows = static_cast<size_t>(num_seqs) * num_q_heads * plan.max_parts;
  float *ws = static_cast<float *>(workspace);
  args.ws_o = plan.ws_bytes ? ws : nullptr;
  args.ws_m = plan.ws_bytes ? ws + rows * cache.head_dim : nullptr;
  args.ws_l = plan.ws_bytes ? ws + rows * (cache.head_dim + 1) : nullptr;
  args.counters =
      plan.ws_bytes ? reinterpret_cast<int32_t *>(ws + rows * (cache.head_dim + 2)) : nullptr;
  args.d_status = d_status;
  args.max_blocks_per_seq = max_blocks_per_seq;
  args.num_q_heads = num_q_heads;
  args.num_kv_heads = cache.num_kv_heads;
  args.group = num_q_heads / cache.num_kv_heads;
  args.num_blocks = cache.num_blocks;
  args.len_limit = static_cast<int>(std::min<long long>(
      max_context_len, static_cast<long long>(max_blocks_per_seq) * cache.block_size));
  args.part_blocks = plan.part_blocks;
  args.max_parts = plan.max_parts;
  args.scale_log2 = scale * kLog2e;

  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (plan.max_parts > 1 &&
      cudaMemsetAsync(args.counters, 0,
                      static_cast<size_t>(num_seqs) * cache.num_kv_heads * sizeof(int32_t),
                      s) != cudaSuccess)
    return PKV_ERR_CUDA;
  const bool big = args.group > 8;
  const bool bf16 = cache.dtype == PKV_BF16;
  if (cache.head_dim == 128)
    st = bf16 ? launch_for_dim<__nv_bfloat16, 128>(cache.block_size, big, tmk, tmv, args,
                                                  cache.num_kv_heads, num_seqs, s)
              : launch_for_dim<__half, 128>(cache.block_size, big, tmk, tmv, args,
                                            cache.num_kv_heads, num_seqs, s);
  else
    st = bf16 ? launch_for_dim<__nv_bfloat16, 64>(cache.block_size, big, tmk, tmv, args,
                                                 cache.num_kv_heads, num_seqs, s)
              : launch_for_dim<__half, 64>(cache.block_size, big, tmk, tmv, args,
                                           cache.num_kv_heads, num_seqs, s);
  if (st != PKV_OK || plan.max_parts <= kFuseMaxParts) return st;

  CombineArgs c{};
  c.out = out;
  c.context_lens = context_lens;
  c.ws_m = args.ws_m;
  c.ws_l = args.ws_l;
  c.ws_o = args.ws_o;
  c.num_q_heads = num_q_heads;
  c.block_size = cache.block_size;
  c.len_limit = args.len_limit;
  c.part_blocks = plan.part_blocks;
  c.max_parts = plan.max_parts;
  if (cache.head_dim == 128)
    return bf16 ? launch_combine<__nv_bfloat16, 128>(c, num_seqs, s)
                : launch_combine<__half, 128>(c, num_seqs, s);
  return bf16 ? launch_combine<__nv_bfloat16, 64>(c, num_seqs, s)
              : launch_combine<__half, 64>(c, num_seqs, s);
}
