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
// under the 128-byte swizzle.
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

}  // namespace pkv
