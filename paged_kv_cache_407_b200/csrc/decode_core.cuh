// Per-warp decode-attention state and the math of one K/V block, shared by the
// attention kernels.
//
// A warp holds the softmax state of the query heads of one group (rows of an
// m16n8k16 tile, query head h of the group on row h) over the blocks it has
// seen: running max m and sum l per row (log2 domain), and the unnormalised
// output O[16 x D] as mma accumulator fragments.  One call of `block` folds
// one K/V block (B tokens) into that state:
//   S^T = Q K^T on mma.sync with the query heads on M, scale and mask,
//   online softmax update, O = O * 2^(m_old - m_new) + P V.
// The score accumulator fragment is, element for element, the A fragment of
// P V, so P never moves between lanes.  With bf16 operands P enters the second
// MMA as a bf16 high part plus a bf16 residual (bf16 alone would round P by up
// to 2^-8 relative); with fp16 operands one fp16 P (at most 2^-11) is enough.
//
// 8-bit pools (KV8): K tiles hold one 128-byte row of E4M3 codes per token, V
// tiles one row of BS codes per dimension (V stored transposed).  ldmatrix on
// such rows hands each lane four consecutive codes, which two cvt
// instructions turn into the two fp16 pairs of an MMA fragment.  To make the
// token order of the score fragment match those V fragments, the K rows of
// 8-token column tile 2t+u are tokens {0,1,4,5,8,9,12,13} + 2u of the 16-token
// group t, so a lane's scores are tokens 4c..4c+3 of the group (c = lane % 4);
// the head-dimension order inside each 16-wide step is permuted the same way
// for Q and K.  Operands are fp16 (E4M3 codes are exact in fp16).  The K tile
// arrives with those eight tokens on consecutive shared-memory rows
// (row 8t + i of tile half u = token 16t + 4(i/2) + i%2 + 2u), and the V tile
// as rows of 128 bytes, so both ldmatrix patterns are free of bank conflicts
// under the 128-byte swizzle.  With at most eight query heads per kv head the
// 8-bit pools use DecodeState8T instead (end of this file): the same tiles and
// the same fragments read as the other operand, with the tokens on M, half the
// MMAs and half the accumulator registers.
#pragma once

#include <type_traits>

#include "pkv_device.cuh"

namespace pkv {

constexpr uint32_t kFullMask = 0xffffffffu;

// Byte offset of 16-byte chunk `chunk` (= d / 8) of token row `tok` inside a
// tile of D/64 boxes, each BS rows x 128 B, written by TMA with the 128-byte
// swizzle (chunk index XOR row index within each 8-row, 1024-byte group).
template <int BS>
__device__ __forceinline__ uint32_t tile_off(int tok, int chunk) {
  return static_cast<uint32_t>((chunk >> 3) * (BS * 128) + tok * 128 +
                               (((chunk & 7) ^ (tok & 7)) << 4));
}

// Byte offset of 16-byte chunk `chunk` of dimension row `row` (BS bytes) in an
// 8-bit V tile moved as 128-byte rows with the 128-byte swizzle.
template <int BS>
__device__ __forceinline__ uint32_t v8_off(int row, int chunk) {
  const uint32_t b = static_cast<uint32_t>(row * BS + chunk * 16);
  return (b & ~127u) | ((((b >> 4) ^ (b >> 7)) & 7u) << 4);
}

template <typename T, int D, int BS, bool BIG, bool KV8 = false>
struct DecodeState {
  static constexpr int kNT = BS / 8;  // 8-token column tiles per block
  static constexpr int kDT = D / 8;   // 8-wide column tiles of the output
  static constexpr int kKS = D / 16;  // 16-deep steps of the score product
  using OP = typename std::conditional<KV8, __half, T>::type;  // MMA operand type
  using MMA = Mma<OP>;
  using PK = Pack<OP>;
  static constexpr bool kSplitP = std::is_same<OP, __nv_bfloat16>::value;

  uint32_t qa0[kKS], qa1[kKS], qa2[kKS], qa3[kKS];  // Q as A fragments (rows r, r + 8)
  float m0, m1, l0, l1;                             // running max / sum, rows r and r + 8
  float o[kDT][4];                                  // O accumulators

  // Query rows of the group: q points at G consecutive rows of D elements.
  __device__ __forceinline__ void load_q(const T *q, int G, int lane) {
    if constexpr (KV8) {
      load_q_kv8(q, G, lane);
      return;
    }
    const int r = lane >> 2;
    const int c2 = (lane & 3) * 2;
    const uint32_t *q32 = reinterpret_cast<const uint32_t *>(q);
#pragma unroll
    for (int kk = 0; kk < kKS; ++kk) {
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
  }

  // Two consecutive query elements as one fp16x2 operand word.
  static __device__ __forceinline__ uint32_t q_pair(const T *p) {
    if constexpr (std::is_same<T, __half>::value) {
      return *reinterpret_cast<const uint32_t *>(p);
    } else {
      const float2 f = Pack<T>::unpack(*reinterpret_cast<const uint32_t *>(p));
      return Pack<__half>::pack(f.x, f.y);
    }
  }

  // KV8 order: within each 16-wide step kk, lane c's k-slots {2c, 2c+1} are
  // dims 16kk + 4c + {0, 1} and k-slots {2c+8, 2c+9} are dims 16kk + 4c + {2, 3}.
  __device__ __forceinline__ void load_q_kv8(const T *q, int G, int lane) {
    const int r = lane >> 2;
    const int c4 = (lane & 3) * 4;
#pragma unroll
    for (int kk = 0; kk < kKS; ++kk) {
      qa0[kk] = r < G ? q_pair(q + r * D + 16 * kk + c4) : 0u;
      qa2[kk] = r < G ? q_pair(q + r * D + 16 * kk + c4 + 2) : 0u;
      if constexpr (BIG) {
        qa1[kk] = r + 8 < G ? q_pair(q + (r + 8) * D + 16 * kk + c4) : 0u;
        qa3[kk] = r + 8 < G ? q_pair(q + (r + 8) * D + 16 * kk + c4 + 2) : 0u;
      } else {
        qa1[kk] = 0u;
        qa3[kk] = 0u;
      }
    }
  }

  __device__ __forceinline__ void reset() {
    m0 = m1 = -INFINITY;
    l0 = l1 = 0.f;
#pragma unroll
    for (int dt = 0; dt < kDT; ++dt) o[dt][0] = o[dt][1] = o[dt][2] = o[dt][3] = 0.f;
  }

  // Fold one block into the state.  kb / vb: shared-memory addresses of the
  // block's K and V tiles; nv: tokens of the block inside the context (the
  // rest are masked, whatever the tile holds).
  __device__ __forceinline__ void block(uint32_t kb, uint32_t vb, int nv, float scale_log2,
                                        int lane) {
    const int mi = lane >> 3;  // ldmatrix: which 8x8 matrix this lane addresses
    const int ri = lane & 7;   // ldmatrix: which row of it
    const int c2 = (lane & 3) * 2;

    // ---- S^T[16 x BS] = Q[16 x D] . K^T ----------------------------------
    float sc[kNT][4];
#pragma unroll
    for (int nt = 0; nt < kNT; ++nt) sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
    if constexpr (KV8) {
      // matrices: 0 = tile 2tp, step 2kk2; 1 = tile 2tp+1, step 2kk2; 2, 3 = step 2kk2+1
#pragma unroll
      for (int kk2 = 0; kk2 < kKS / 2; ++kk2) {
#pragma unroll
        for (int tp = 0; tp < BS / 16; ++tp) {
          uint32_t r0, r1, r2, r3;
          const int row = (mi & 1) * (BS / 2) + tp * 8 + ri;
          const int chunk = 2 * kk2 + (mi >> 1);
          ldsm_x4(kb + row * 128 + ((chunk ^ ri) << 4), r0, r1, r2, r3);
          const int k0 = 2 * kk2, k1 = 2 * kk2 + 1;
          uint32_t f0, f1;
          e4m3x4_to_f16x2x2(r0, f0, f1);
          MMA::k16(sc[2 * tp], qa0[k0], qa1[k0], qa2[k0], qa3[k0], f0, f1);
          e4m3x4_to_f16x2x2(r1, f0, f1);
          MMA::k16(sc[2 * tp + 1], qa0[k0], qa1[k0], qa2[k0], qa3[k0], f0, f1);
          e4m3x4_to_f16x2x2(r2, f0, f1);
          MMA::k16(sc[2 * tp], qa0[k1], qa1[k1], qa2[k1], qa3[k1], f0, f1);
          e4m3x4_to_f16x2x2(r3, f0, f1);
          MMA::k16(sc[2 * tp + 1], qa0[k1], qa1[k1], qa2[k1], qa3[k1], f0, f1);
        }
      }
    } else if constexpr (BS >= 16) {
#pragma unroll
      for (int kk = 0; kk < kKS; ++kk) {
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
      for (int kk = 0; kk < kKS; kk += 2) {
        uint32_t b0r, b1r, b2r, b3r;
        ldsm_x4(kb + tile_off<BS>(ri, 2 * kk + mi), b0r, b1r, b2r, b3r);
        MMA::k16(sc[0], qa0[kk], qa1[kk], qa2[kk], qa3[kk], b0r, b1r);
        MMA::k16(sc[0], qa0[kk + 1], qa1[kk + 1], qa2[kk + 1], qa3[kk + 1], b2r, b3r);
      }
    }

    // ---- scale, mask past the context, online softmax --------------------
    const bool partial = nv < BS;
#pragma unroll
    for (int nt = 0; nt < kNT; ++nt)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float v = sc[nt][j] * scale_log2;
        // token of this score: tile nt column c2 + (j & 1), or in KV8 order
        // group nt/2, tokens 4c + 2 * (nt & 1) + (j & 1)
        const int tok = KV8 ? (nt >> 1) * 16 + 2 * c2 + ((nt & 1) << 1) + (j & 1)
                            : nt * 8 + c2 + (j & 1);
        if (partial && tok >= nv) v = -INFINITY;
        sc[nt][j] = v;
      }
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < kNT; ++nt) {
      mx0 = fmaxf(mx0, fmaxf(sc[nt][0], sc[nt][1]));
      if constexpr (BIG) mx1 = fmaxf(mx1, fmaxf(sc[nt][2], sc[nt][3]));
    }
    mx0 = fmaxf(mx0, __shfl_xor_sync(kFullMask, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(kFullMask, mx0, 2));
    const float mn0 = fmaxf(m0, mx0);
    const float base0 = mn0 == -INFINITY ? 0.f : mn0;
    const float al0 = fast_exp2(m0 - base0);
    m0 = mn0;
    float al1 = 1.f, base1 = 0.f;
    if constexpr (BIG) {
      mx1 = fmaxf(mx1, __shfl_xor_sync(kFullMask, mx1, 1));
      mx1 = fmaxf(mx1, __shfl_xor_sync(kFullMask, mx1, 2));
      const float mn1 = fmaxf(m1, mx1);
      base1 = mn1 == -INFINITY ? 0.f : mn1;
      al1 = fast_exp2(m1 - base1);
      m1 = mn1;
    }
    float rs0 = 0.f, rs1 = 0.f;
#pragma unroll
    for (int nt = 0; nt < kNT; ++nt) {
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
    if (__any_sync(kFullMask, moved)) {
#pragma unroll
      for (int dt = 0; dt < kDT; ++dt) {
        o[dt][0] *= al0;
        o[dt][1] *= al0;
        if constexpr (BIG) {
          o[dt][2] *= al1;
          o[dt][3] *= al1;
        }
      }
    }

    // ---- O[16 x D] += P[16 x BS] . V --------------------------------------
    if constexpr (KV8) {
#pragma unroll
      for (int tp = 0; tp < BS / 16; ++tp) {
        // a lane's P for the group: tokens 4c, 4c+1 (k-slots 2c, 2c+1) and
        // 4c+2, 4c+3 (k-slots 2c+8, 2c+9)
        const uint32_t h0 = PK::pack(sc[2 * tp][0], sc[2 * tp][1]);
        const uint32_t h2 = PK::pack(sc[2 * tp + 1][0], sc[2 * tp + 1][1]);
        uint32_t h1 = 0u, h3 = 0u;
        if constexpr (BIG) {
          h1 = PK::pack(sc[2 * tp][2], sc[2 * tp][3]);
          h3 = PK::pack(sc[2 * tp + 1][2], sc[2 * tp + 1][3]);
        }
        const int t0 = tp * 16 + 2 * c2;  // first of this lane's four tokens
        const bool vmask = partial && (tp * 16 + 16 > nv);
        const uint32_t bmask = (t0 < nv ? 0x000000ffu : 0u) | (t0 + 1 < nv ? 0x0000ff00u : 0u) |
                               (t0 + 2 < nv ? 0x00ff0000u : 0u) | (t0 + 3 < nv ? 0xff000000u : 0u);
#pragma unroll
        for (int dq = 0; dq < D / 32; ++dq) {
          uint32_t v[4];
          ldsm_x4(vb + v8_off<BS>(32 * dq + 8 * mi + ri, tp), v[0], v[1], v[2], v[3]);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            uint32_t b01, b23;
            e4m3x4_to_f16x2x2(vmask ? (v[j] & bmask) : v[j], b01, b23);
            MMA::k16(o[4 * dq + j], h0, h1, h2, h3, b01, b23);
          }
        }
      }
    } else if constexpr (BS >= 16) {
#pragma unroll
      for (int tp = 0; tp < BS / 16; ++tp) {
        const uint32_t h0 = PK::pack(sc[2 * tp][0], sc[2 * tp][1]);
        const uint32_t h2 = PK::pack(sc[2 * tp + 1][0], sc[2 * tp + 1][1]);
        uint32_t h1 = 0u, h3 = 0u, e0 = 0u, e1 = 0u, e2 = 0u, e3 = 0u;
        if constexpr (BIG) {
          h1 = PK::pack(sc[2 * tp][2], sc[2 * tp][3]);
          h3 = PK::pack(sc[2 * tp + 1][2], sc[2 * tp + 1][3]);
        }
        if constexpr (kSplitP) {
          const float2 f0 = PK::unpack(h0);
          const float2 f2 = PK::unpack(h2);
          e0 = PK::pack(sc[2 * tp][0] - f0.x, sc[2 * tp][1] - f0.y);
          e2 = PK::pack(sc[2 * tp + 1][0] - f2.x, sc[2 * tp + 1][1] - f2.y);
          if constexpr (BIG) {
            const float2 f1 = PK::unpack(h1);
            const float2 f3 = PK::unpack(h3);
            e1 = PK::pack(sc[2 * tp][2] - f1.x, sc[2 * tp][3] - f1.y);
            e3 = PK::pack(sc[2 * tp + 1][2] - f3.x, sc[2 * tp + 1][3] - f3.y);
          }
        }
        const bool vmask = partial && (tp * 16 + 16 > nv);
        const int t0 = tp * 16 + c2;
        const uint32_t mlo = (t0 < nv ? 0x0000ffffu : 0u) | (t0 + 1 < nv ? 0xffff0000u : 0u);
        const uint32_t mhi = (t0 + 8 < nv ? 0x0000ffffu : 0u) | (t0 + 9 < nv ? 0xffff0000u : 0u);
#pragma unroll
        for (int dp = 0; dp < kDT / 2; ++dp) {
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
          MMA::k16(o[2 * dp + 1], h0, h1, h2, h3, v2, v3);
          if constexpr (kSplitP) {
            MMA::k16(o[2 * dp], e0, e1, e2, e3, v0, v1);
            MMA::k16(o[2 * dp + 1], e0, e1, e2, e3, v2, v3);
          }
        }
      }
    } else {
      const uint32_t h0 = PK::pack(sc[0][0], sc[0][1]);
      uint32_t h1 = 0u, e0 = 0u, e1 = 0u;
      if constexpr (BIG) h1 = PK::pack(sc[0][2], sc[0][3]);
      if constexpr (kSplitP) {
        const float2 f0 = PK::unpack(h0);
        e0 = PK::pack(sc[0][0] - f0.x, sc[0][1] - f0.y);
        if constexpr (BIG) {
          const float2 f1 = PK::unpack(h1);
          e1 = PK::pack(sc[0][2] - f1.x, sc[0][3] - f1.y);
        }
      }
      const uint32_t mlo = (c2 < nv ? 0x0000ffffu : 0u) | (c2 + 1 < nv ? 0xffff0000u : 0u);
#pragma unroll
      for (int dq = 0; dq < kDT / 4; ++dq) {
        uint32_t v[4];
        ldsm_x4_trans(vb + tile_off<BS>(ri, 4 * dq + mi), v[0], v[1], v[2], v[3]);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          if (partial) v[j] &= mlo;
          MMA::k8(o[4 * dq + j], h0, h1, v[j]);
          if constexpr (kSplitP) MMA::k8(o[4 * dq + j], e0, e1, v[j]);
        }
      }
    }
  }

  // Sum l over the four lanes that share a row.
  __device__ __forceinline__ void reduce_l() {
    l0 += __shfl_xor_sync(kFullMask, l0, 1);
    l0 += __shfl_xor_sync(kFullMask, l0, 2);
    if constexpr (BIG) {
      l1 += __shfl_xor_sync(kFullMask, l1, 1);
      l1 += __shfl_xor_sync(kFullMask, l1, 2);
    }
  }

  // Write rows < G of the state to shared memory: O as [row][D] floats at
  // `mo`, m and l per row at `mm`, `ml` (call after reduce_l).
  __device__ __forceinline__ void store_rows(float *mo, float *mm, float *ml, int G, int lane) const {
    const int r = lane >> 2;
    const int c2 = (lane & 3) * 2;
    if (r < G) {
#pragma unroll
      for (int dt = 0; dt < kDT; ++dt)
        *reinterpret_cast<float2 *>(&mo[r * D + dt * 8 + c2]) = make_float2(o[dt][0], o[dt][1]);
      if ((lane & 3) == 0) {
        mm[r] = m0;
        ml[r] = l0;
      }
    }
    if constexpr (BIG) {
      if (r + 8 < G) {
#pragma unroll
        for (int dt = 0; dt < kDT; ++dt)
          *reinterpret_cast<float2 *>(&mo[(r + 8) * D + dt * 8 + c2]) =
              make_float2(o[dt][2], o[dt][3]);
        if ((lane & 3) == 0) {
          mm[r + 8] = m1;
          ml[r + 8] = l1;
        }
      }
    }
  }
};

// 8-bit pools with at most 8 query heads per kv head: the same computation
// with the tokens on the MMA's M dimension and the heads on N, so one
// m16n8k16 covers 16 tokens for all (up to eight) heads of the group
// instead of a 16-row query tile that is mostly padding.  Per 16 tokens:
//   S[16 slots x 8 heads] = K[16 slots x D] . Q^T          (8 MMAs)
//   O^T[D x 8 heads]     += V^T[D x 16 slots] . P^T        (8 MMAs)
// The K tile's rows are already in the permuted token order of the 8-bit
// layout: 16-token group tp of a block sits in rows tp*8 .. tp*8 + 7 and
// B/2 + tp*8 .. + 7, and slot s of a group (s < 8 the first run, s >= 8 the
// second) holds token 16tp + 4((s & 7) >> 1) + 2(s >> 3) + (s & 1).  That
// order is what makes the A fragments line up: ldmatrix gives lane (g, t) the
// four codes 4t .. 4t + 3 of slot g's 16-dimension chunk (k-slots 2t, 2t + 1
// and 2t + 8, 2t + 9 in the head-dimension order that load_q uses for Q), and
// of dimension g's row of V^T the tokens 16tp + 4t .. + 3, which are exactly
// the group's slots 2t, 2t + 1, 2t + 8, 2t + 9.  P moves from the accumulator
// layout of S (slot rows) to the B layout of P^T (head rows) with two 8x8
// transposes per group.
template <typename T, int D, int BS>
struct DecodeState8T {
  static_assert(BS % 16 == 0, "blocks of whole 16-token groups");
  static constexpr int kTP = BS / 16;  // 16-token groups per block
  static constexpr int kMT = D / 16;   // 16-dimension m-tiles of O^T
  static constexpr int kKS = D / 16;   // 16-deep steps of the score product
  using MMA = Mma<__half>;
  using PK = Pack<__half>;

  uint32_t qb0[kKS], qb1[kKS];  // Q^T as B fragments (head g = lane / 4)
  float ma, mb, la, lb;         // running max / sum of heads 2t and 2t + 1
  float o[kMT][4];              // O^T: dims g, g + 8 of each m-tile x heads 2t, 2t + 1

  static __device__ __forceinline__ uint32_t q_pair(const T *p) {
    if constexpr (std::is_same<T, __half>::value) {
      return *reinterpret_cast<const uint32_t *>(p);
    } else {
      const float2 f = Pack<T>::unpack(*reinterpret_cast<const uint32_t *>(p));
      return Pack<__half>::pack(f.x, f.y);
    }
  }

  // B fragment of step kk for head g: k-slots {2t, 2t + 1} are dims
  // 16kk + 4t + {0, 1}, k-slots {2t + 8, 2t + 9} dims 16kk + 4t + {2, 3}.
  __device__ __forceinline__ void load_q(const T *q, int G, int lane) {
    const int g = lane >> 2;
    const int c4 = (lane & 3) * 4;
#pragma unroll
    for (int kk = 0; kk < kKS; ++kk) {
      qb0[kk] = g < G ? q_pair(q + g * D + 16 * kk + c4) : 0u;
      qb1[kk] = g < G ? q_pair(q + g * D + 16 * kk + c4 + 2) : 0u;
    }
  }

  __device__ __forceinline__ void reset() {
    ma = mb = -INFINITY;
    la = lb = 0.f;
#pragma unroll
    for (int mt = 0; mt < kMT; ++mt) o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.f;
  }

  static __device__ __forceinline__ uint32_t transpose8x8(uint32_t a) {
    uint32_t d;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(d) : "r"(a));
    return d;
  }

  __device__ __forceinline__ void block(uint32_t kb, uint32_t vb, int nv, float scale_log2, int lane) {
    const int mi = lane >> 3;  // ldmatrix: which 8x8 matrix this lane addresses
    const int ri = lane & 7;   // ldmatrix: which row of it
    const int g = lane >> 2;
    const int t = lane & 3;

    // ---- S[16 slots x 8 heads] per group = K . Q^T; even and odd steps in
    // two chains
    float s[kTP][4];
#pragma unroll
    for (int tp = 0; tp < kTP; ++tp) {
      float s2[4] = {0.f, 0.f, 0.f, 0.f};
      s[tp][0] = s[tp][1] = s[tp][2] = s[tp][3] = 0.f;
#pragma unroll
      for (int kk2 = 0; kk2 < kKS / 2; ++kk2) {
        // matrices: slots 0-7 / 8-15 of chunk 2 kk2, then of chunk 2 kk2 + 1
        uint32_t r0, r1, r2, r3;
        const int row = (mi & 1) * (BS / 2) + tp * 8 + ri;
        const int chunk = 2 * kk2 + (mi >> 1);
        ldsm_x4(kb + row * 128 + ((chunk ^ ri) << 4), r0, r1, r2, r3);
        uint32_t lo_g, hi_g, lo_g8, hi_g8;
        e4m3x4_to_f16x2x2(r0, lo_g, hi_g);
        e4m3x4_to_f16x2x2(r1, lo_g8, hi_g8);
        MMA::k16(s[tp], lo_g, lo_g8, hi_g, hi_g8, qb0[2 * kk2], qb1[2 * kk2]);
        e4m3x4_to_f16x2x2(r2, lo_g, hi_g);
        e4m3x4_to_f16x2x2(r3, lo_g8, hi_g8);
        MMA::k16(s2, lo_g, lo_g8, hi_g, hi_g8, qb0[2 * kk2 + 1], qb1[2 * kk2 + 1]);
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) s[tp][j] += s2[j];
    }
    // s[tp][0], [1]: slot g x heads 2t, 2t + 1; [2], [3]: slot g + 8
    const bool partial = nv < BS;
    const int tok_g = ((g >> 1) << 2) + (g & 1);  // token of slot g in its group; slot g + 8: + 2
    float mxa = -INFINITY, mxb = -INFINITY;
#pragma unroll
    for (int tp = 0; tp < kTP; ++tp) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float v = s[tp][j] * scale_log2;
        if (partial && 16 * tp + tok_g + ((j >> 1) << 1) >= nv) v = -INFINITY;
        s[tp][j] = v;
      }
      mxa = fmaxf(mxa, fmaxf(s[tp][0], s[tp][2]));
      mxb = fmaxf(mxb, fmaxf(s[tp][1], s[tp][3]));
    }
#pragma unroll
    for (int d = 4; d < 32; d <<= 1) {
      mxa = fmaxf(mxa, __shfl_xor_sync(kFullMask, mxa, d));
      mxb = fmaxf(mxb, __shfl_xor_sync(kFullMask, mxb, d));
    }
    const float mna = fmaxf(ma, mxa), mnb = fmaxf(mb, mxb);
    const float ba = mna == -INFINITY ? 0.f : mna, bb = mnb == -INFINITY ? 0.f : mnb;
    const float ala = fast_exp2(ma - ba), alb = fast_exp2(mb - bb);
    ma = mna;
    mb = mnb;
    float rsa = 0.f, rsb = 0.f;
    uint32_t pb0[kTP], pb1[kTP];  // P^T as B operands: k-slots 2t, 2t + 1 / 2t + 8, 2t + 9 of head g
#pragma unroll
    for (int tp = 0; tp < kTP; ++tp) {
      const float p0 = fast_exp2(s[tp][0] - ba), p1 = fast_exp2(s[tp][1] - bb);
      const float p2 = fast_exp2(s[tp][2] - ba), p3 = fast_exp2(s[tp][3] - bb);
      rsa += p0 + p2;
      rsb += p1 + p3;
      pb0[tp] = transpose8x8(PK::pack(p0, p1));
      pb1[tp] = transpose8x8(PK::pack(p2, p3));
    }
    la = la * ala + rsa;
    lb = lb * alb + rsb;
    if (__any_sync(kFullMask, ala != 1.f || alb != 1.f)) {
#pragma unroll
      for (int mt = 0; mt < kMT; ++mt) {
        o[mt][0] *= ala;
        o[mt][1] *= alb;
        o[mt][2] *= ala;
        o[mt][3] *= alb;
      }
    }

    // ---- O^T[D x 8] += V^T . P^T per group; lane t's codes of group tp are
    // tokens 16tp + 4t .. + 3
#pragma unroll
    for (int tp = 0; tp < kTP; ++tp) {
      const int t0 = 16 * tp + 4 * t;
      const bool vmask = partial && (16 * tp + 16 > nv);
      const uint32_t bmask = (t0 < nv ? 0x000000ffu : 0u) | (t0 + 1 < nv ? 0x0000ff00u : 0u) |
                             (t0 + 2 < nv ? 0x00ff0000u : 0u) | (t0 + 3 < nv ? 0xff000000u : 0u);
#pragma unroll
      for (int dq = 0; dq < D / 32; ++dq) {
        uint32_t v[4];  // dims 32dq + 8j + (lane's row) for matrix j
        ldsm_x4(vb + v8_off<BS>(32 * dq + 8 * mi + ri, tp), v[0], v[1], v[2], v[3]);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t lo_g, hi_g, lo_g8, hi_g8;
          e4m3x4_to_f16x2x2(vmask ? (v[2 * h] & bmask) : v[2 * h], lo_g, hi_g);
          e4m3x4_to_f16x2x2(vmask ? (v[2 * h + 1] & bmask) : v[2 * h + 1], lo_g8, hi_g8);
          MMA::k16(o[2 * dq + h], lo_g, lo_g8, hi_g, hi_g8, pb0[tp], pb1[tp]);
        }
      }
    }
  }

  // Sum l over the eight lanes that share a head pair.
  __device__ __forceinline__ void reduce_l() {
#pragma unroll
    for (int d = 4; d < 32; d <<= 1) {
      la += __shfl_xor_sync(kFullMask, la, d);
      lb += __shfl_xor_sync(kFullMask, lb, d);
    }
  }

  // Rows < G of the state to shared memory as DecodeState::store_rows does.
  __device__ __forceinline__ void store_rows(float *mo, float *mm, float *ml, int G, int lane) const {
    const int g = lane >> 2;
    const int ha = 2 * (lane & 3), hb = ha + 1;
#pragma unroll
    for (int mt = 0; mt < kMT; ++mt) {
      if (ha < G) {
        mo[ha * D + 16 * mt + g] = o[mt][0];
        mo[ha * D + 16 * mt + g + 8] = o[mt][2];
      }
      if (hb < G) {
        mo[hb * D + 16 * mt + g] = o[mt][1];
        mo[hb * D + 16 * mt + g + 8] = o[mt][3];
      }
    }
    if (g == 0) {
      if (ha < G) {
        mm[ha] = ma;
        ml[ha] = la;
      }
      if (hb < G) {
        mm[hb] = mb;
        ml[hb] = lb;
      }
    }
  }
};

}  // namespace pkv
