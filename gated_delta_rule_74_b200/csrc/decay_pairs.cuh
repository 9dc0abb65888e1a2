// Exact pairwise decay terms for channels whose decay is too strong for the
// reference-point factoring of the chunk Gram matrices (device code shared by the
// tensor-core prefill and the chunked decode; not part of the C ABI).
//
// The chunked form needs, per pair of rows i <= r of a chunk and key channel c,
// the factor exp(G_rc - G_ic) (miniKimiK3 model card, "Kimi Delta Attention"
// bullet: per-channel gated decay; the chunked parallel form equals the
// recurrence).  The tensor-core kernels split it through a reference point P of
// the row block, (k_r e^{G_r - P}) (k_i e^{P - G_i}), so that one matrix product
// over the channels gives every pair of the block.  Inside a block that factoring
// needs the block's own decay, P - G at its last row, to stay within the fp32
// exponent range; a channel whose decay inside one block is stronger (per-token g
// below about -4 on average, or a gate that closes, g -> -inf) is "unsafe" there.
// Its within-block pairs are taken out of the product (its growing factor is
// zeroed) and added here exactly instead, as running products of the per-token
// factors al_j = exp(g_j) <= 1: nothing overflows, and a product reaches zero only
// where the true factor is below the fp32 range.
#pragma once

#include <stdint.h>

namespace kda {

// A channel is unsafe in a block when its decay inside the block exceeds this
// (in log units).  Below it every factor of the split lies in [e^-60, e^60], so the
// bf16 operands stay normal and a product's factors never flush to zero while the
// product itself is above e^-27 relative to the block's largest entries.
constexpr float kUnsafeDecay = 60.f;

// Sum over the warp's 32 lanes of each of 16 per-lane values; lane l returns the
// total of value l / 2 (transpose-reduce: halves exchanged at lane distance 16,
// 8, 4, 2, then one butterfly step).
__device__ __forceinline__ float rowsum16(const float (&v)[16], int lane) {
  float x8[8], x4[4], x2[2];
  const bool b16 = lane & 16, b8 = lane & 8, b4 = lane & 4, b2 = lane & 2;
#pragma unroll
  for (int i = 0; i < 8; ++i)
    x8[i] = (b16 ? v[i + 8] : v[i]) + __shfl_xor_sync(0xffffffffu, b16 ? v[i] : v[i + 8], 16);
#pragma unroll
  for (int i = 0; i < 4; ++i)
    x4[i] = (b8 ? x8[i + 4] : x8[i]) + __shfl_xor_sync(0xffffffffu, b8 ? x8[i] : x8[i + 4], 8);
#pragma unroll
  for (int i = 0; i < 2; ++i)
    x2[i] = (b4 ? x4[i + 2] : x4[i]) + __shfl_xor_sync(0xffffffffu, b4 ? x4[i] : x4[i + 2], 4);
  float x = (b2 ? x2[1] : x2[0]) + __shfl_xor_sync(0xffffffffu, b2 ? x2[0] : x2[1], 2);
  return x + __shfl_xor_sync(0xffffffffu, x, 1);
}

// For one block of NR rows (NR = 8 or 16), the calling lane's NC channels:
//   al[j][c] = exp(g_j) of row j, kv / qv = k and q of the row.
// Adds, summed over the warp's 32 lanes and all their channels,
//   corrA[r * 16 + i] += sum_c k_rc k_ic prod_{j=i+1..r} al_jc      (i <  r)
//   corrQ[r * 16 + i] += sum_c q_rc k_ic prod_{j=i+1..r} al_jc      (i <= r)
// (row stride 16) with shared-memory atomics, so several warps may add to one
// block.  Every lane of the warp must call it; a lane with nothing to add passes
// k = q = 0.
template <int NC, int NR>
__device__ __forceinline__ void add_pair_terms(const float (&al)[NR][NC], const float (&kv)[NR][NC],
                                               const float (&qv)[NR][NC], float* corrA,
                                               float* corrQ, int lane) {
  static_assert(NR == 8 || NR == 16, "block of 8 or 16 rows");
#pragma unroll 1
  for (int r = 0; r < NR; ++r) {
    float kr[NC], qr[NC], p[NC];
#pragma unroll
    for (int c = 0; c < NC; ++c) {
      kr[c] = 0.f;
      qr[c] = 0.f;
      p[c] = 1.f;
    }
#pragma unroll
    for (int e = 0; e < NR; ++e)
      if (e == r) {
#pragma unroll
        for (int c = 0; c < NC; ++c) {
          kr[c] = kv[e][c];
          qr[c] = qv[e][c];
        }
      }
    // vals[i]: the A term of pair (r, i); vals[NR + i]: the Aqk term
    float vals[2 * NR];
#pragma unroll
    for (int i = NR - 1; i >= 0; --i) {
      if (i + 1 < NR && i < r) {
#pragma unroll
        for (int c = 0; c < NC; ++c) p[c] *= al[i + 1][c];
      }
      float sa = 0.f, sq = 0.f;
#pragma unroll
      for (int c = 0; c < NC; ++c) {
        const float t = kv[i][c] * p[c];
        sa = fmaf(kr[c], t, sa);
        sq = fmaf(qr[c], t, sq);
      }
      vals[i] = i < r ? sa : 0.f;
      vals[NR + i] = i <= r ? sq : 0.f;
    }
#pragma unroll
    for (int grp = 0; grp < 2 * NR / 16; ++grp) {
      float v16[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) v16[e] = vals[16 * grp + e];
      const float tot = rowsum16(v16, lane);
      const int idx = 16 * grp + (lane >> 1);
      if ((lane & 1) == 0) {
        if (idx < NR) {
          if (idx < r) atomicAdd(corrA + r * 16 + idx, tot);
        } else if (idx - NR <= r) {
          atomicAdd(corrQ + r * 16 + (idx - NR), tot);
        }
      }
    }
  }
}

}  // namespace kda
