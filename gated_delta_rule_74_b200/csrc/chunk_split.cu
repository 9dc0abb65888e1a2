// KDA prefill in two kernels on the sm_100a tensor cores, dk = dv = 128, bf16
// q/k/v, fp32 g/beta/state.
//
// Chunked form (miniKimiK3 model card, "Kimi Delta Attention" bullet: training
// and prefill run through a chunked parallel form; "Inside Kimi" outline,
// DeltaNet lesson: chunkwise prefill trades arithmetic for parallel hardware
// use).  For one chunk of L <= 64 tokens with initial state S (dk x dv) and
// G_r = g_0 + ... + g_r (per key channel, restarting at the chunk):
//     A[r,i]   = sum_c k_rc k_ic exp(G_rc - G_ic)        i <  r
//     Aqk[r,i] = sum_c q_rc k_ic exp(G_rc - G_ic)        i <= r
//     T        = (I + diag(beta) A)^-1
//     W = T diag(beta) Kbar,  U = T diag(beta) V,        Kbar_r = exp(G_r) k_r
//     Delta    = U - W S
//     O        = Qbar S + Aqk Delta,                     Qbar_r = exp(G_r) q_r
//     S_next   = Diag(exp(G_last)) S + Kend^T Delta,     Kend_i = exp(G_last - G_i) k_i
// Rows past the end of a sequence are zero (k = q = beta = g = 0) and so
// contribute nothing; G_last = G_63 then equals G at the last real row.
//
// Split.  Everything above except the last three lines depends on the chunk
// alone, so it is computed for all (chunk, head) pairs at once by the prep
// kernel (one CTA per pair, two CTAs per SM) and written out as a chunk record:
// the operands of the state update, stored as the exact shared-memory images
// the tensor cores read.  The state pass then walks each sequence's chunks in
// order doing only the state-dependent work,
//     [O^T | P]   [dv x 128] = S^T [Qbar^T | W^T]^T      (S^T bf16 copy in TMEM)
//     Delta^T = U^T - P
//     [S^T | O^T] [dv x 192] += Delta^T [Kend^T ; Aqk]^T  (after S^T <- S^T Diag(exp(G_last)))
// with one bulk copy per record, two records ahead.  The first product runs on bf16
// operands; the second on f16 ones (Delta, Kend and Aqk are bounded -- |Kend|,
// |Aqk| <= 1 for unit-norm keys -- and f16's 11-bit significand halves the
// output error against bf16's 8 bits; conversions saturate at the f16 range).
// S^T stays in TMEM in fp32 for the whole chain.  Packed documents restart the state from their own h0
// slot and restart chunking at the document start (Mini-K3-1H-mamba2 card,
// packed-document paragraph: state flow resets at every boundary).
//
// Decay factoring in the prep kernel (exp(G_r - G_i) split through reference
// points so no factor overflows): rows are grouped in 16-token blocks a with
// P_a = G at row 16a.
//   i, r in block a:   (k_r e^{G_r - P_a}) (k_i e^{P_a - G_i})
//       first factor <= 1; second <= e^{decay inside the block}
//   i in block b < a:  (k_r e^{G_r - P_a}) (k_i e^{P_a - G_i}),  e^{P_a - G_i} <= 1
// so the Gram of row block a is one product against R^(a) = [k_i e^{P_a - G_i}]
// over i < 16(a+1).  All four products (A and Aqk rows for all blocks) are one
// MMA of N = 160:
//   [D^(0) .. D^(3)] [128 x 160] = [Lk ; Lq] [R^(0); ..; R^(3)]^T
// A channel whose decay inside block a exceeds kUnsafeDecay (strong decay, or a
// gate that closes) has its within-block entries of R^(a) zeroed; those pairs are
// then added exactly by a CUDA-core pass (decay_pairs.cuh), and its other factors
// (R^(a') for a' > a, Kend) are formed directly, each <= 1.  Exponents are taken
// as differences of per-block sums, never of chunk-wide sums, so a closed gate
// (g -> -1e4) early in the chunk costs no precision later in it.
#include <cuda_fp16.h>

#include <algorithm>
#include <cstring>
#include <type_traits>

#include "chunk_record.cuh"
#include "decay_pairs.cuh"
#include "kda_common.cuh"
#include "segments.cuh"
#include "sm100.cuh"
#include "tma.cuh"

namespace kda {

// Set when a bounded wait of the split prefill gives up (diagnostic).
__device__ int g_chunk_split_timeout = 0;

namespace {
using namespace sm100;
using bf16 = __nv_bfloat16;

constexpr int C = kChunk;
constexpr int D = kHead;
constexpr int NT = 256;
constexpr uint32_t kWaitLimit = 1u << 22;

// ---- chunk record (one per (head, chunk)), byte offsets (chunk_record.cuh)
constexpr uint32_t REC_QW = rec::QW;    // [Qbar^T | W^T]: MN-major SW128, N = 128 (2 x 64 tokens,
                                        // 16 KB apart), K = dk
constexpr uint32_t REC_KA = rec::KA;    // [Kend^T ; Aqk] (f16): K-major SW128, 192 rows x 64 tokens
constexpr uint32_t REC_AQK = rec::AQK;
constexpr uint32_t REC_U = rec::U;      // U^T [dv][64 tokens] f16: 128-byte rows, 16-byte
                                        // chunks (8 tokens) XOR-swizzled with (row % 8)
constexpr uint32_t REC_DECAY = rec::DECAY;   // exp(G_last) per key channel, fp32 [dk]
constexpr uint32_t REC_BYTES = rec::BYTES;
// The backward's records (BWD instantiation): the same images, but Kend^T, Aqk and
// U^T in bf16 (gradients can be far below f16's normal range), followed by T as a bf16
// image and A in fp32.

// TMA maps of the prep kernel's tiles: q, k, g [rows, H, dk] and v [rows, H, dv]
// (3-D: channel, head, token row), boxes of 64 token rows of one head.
struct PrepMaps {
  CUtensorMap q, k, g, v;
};

// ---- prep kernel: shared memory (from a 1024-aligned base) and TMEM
constexpr uint32_t Q_V = 0;             // V: MN-major SW128 A operand of U^T (M = value, K = token)
constexpr uint32_t Q_KB = 16384;        // Kbar^T: K-major SW128 A operand of W^T
constexpr uint32_t Q_L = 32768;         // [Lk ; Lq]: MN-major SW128 A operand of the Gram
constexpr uint32_t Q_R = 65536;         // R^(0..3): MN-major SW32 B operand of the Gram, 40 KB
__host__ __device__ constexpr uint32_t q_r(int a) {
  return Q_R + (a == 0 ? 0u : a == 1 ? 4096u : a == 2 ? 12288u : 24576u);
}
// after the Gram has been read, the L / R region holds the solve
constexpr int LDA = 68;                 // fp32 row stride (16-byte rows)
constexpr uint32_t Q_B32 = 32768;       // diag(beta) A, fp32
constexpr uint32_t Q_T32 = Q_B32 + 17408;   // T, fp32
constexpr uint32_t Q_M32 = Q_T32 + 17408;   // T_aa B_am, 6 x 16 x 16 fp32
constexpr uint32_t Q_TB = 73728;        // T diag(beta): K-major SW128 B operand of W^T / U^T
// record images on their way out (bulk copies): Aqk after the Gram readout,
// then W^T and U^T over the dead solve scratch once their MMAs are done
constexpr uint32_t Q_OAQK = 81920, Q_OW = 32768, Q_OU = 49152;
// corrections of unsafe channels (8 KB, between the Gram readout and the solve)
constexpr uint32_t Q_CORR = 90112;
constexpr uint32_t PREP_SMEM = 106496 + 1024;
constexpr uint32_t PT_G = 0;            // Gram D^(0..3) at +0, +16, +48, +96 (160 columns)
constexpr uint32_t PT_W = 0;            // W^T [128 x 64] (after the Gram is read)
constexpr uint32_t PT_U = 64;           // U^T [128 x 64]
constexpr uint32_t kPrepTmemCols = 256;

// ---- state pass: shared memory and TMEM
constexpr uint32_t S_BUF = 74752;       // record buffer stride (two buffers)
constexpr uint32_t S_OUT = 2 * S_BUF;   // output tile [64 tokens][128] bf16
constexpr uint32_t S_GATE = S_OUT + 16384;   // output-gate tile [64 tokens][128] bf16
constexpr uint32_t STATE_SMEM = S_GATE + 16384 + 1024;
// [S^T | O^T] and [O^T | P] are each the accumulator of one MMA, so O^T sits
// between S^T and P.
constexpr uint32_t ST_S = 0;            // S^T fp32        [128 lanes x 128]
constexpr uint32_t ST_O = 128;          // O^T             [128 x 64]
constexpr uint32_t ST_P = 192;          // P               [128 x 64]
constexpr uint32_t ST_SB = 256;         // S^T bf16 (A)    [128 x 64]
constexpr uint32_t ST_D = 320;          // Delta^T f16 (A)  [128 x 32]
constexpr uint32_t ST_LO = 384;         // from a half point: bf16 lo part of S_start^T [128 x 64]
constexpr uint32_t kStateTmemCols = 512;

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}
__device__ __forceinline__ uint4 pack8(const float (&x)[8], float s) {
  return make_uint4(pack_bf16(x[0] * s, x[1] * s), pack_bf16(x[2] * s, x[3] * s),
                    pack_bf16(x[4] * s, x[5] * s), pack_bf16(x[6] * s, x[7] * s));
}
// the same as f16 (the [Kend^T ; Aqk] operand and Delta^T are f16: the second MMA
// of the state step runs in kind::f16 with f16 A and B)
__device__ __forceinline__ uint4 pack8_f16(const float (&x)[8], float s) {
  return make_uint4(pack_f16(x[0] * s, x[1] * s), pack_f16(x[2] * s, x[3] * s),
                    pack_f16(x[4] * s, x[5] * s), pack_f16(x[6] * s, x[7] * s));
}
__device__ __forceinline__ void sts16(uint8_t* base, uint32_t off, uint4 v) {
  *reinterpret_cast<uint4*>(base + off) = v;
}
__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }
__device__ __forceinline__ float h_lo(uint32_t w) {
  return __half2float(__ushort_as_half((unsigned short)(w & 0xffffu)));
}
__device__ __forceinline__ float h_hi(uint32_t w) {
  return __half2float(__ushort_as_half((unsigned short)(w >> 16)));
}

constexpr float kNormEps2 = 1e-24f;     // (1e-12)^2: L2 norm floor of the fused q/k prep

// Per-row values of one thread's two channels in its 16-row block a: x = G_r - P_a,
// k and q; per channel d[a2] = P_{a2} - P_a and tl = G_last - P_a.
struct UnsafeRows {
  float x[2][16], k[2][16], q[2][16], d[2][4], tl[2];
};

// Operands of this thread's unsafe channels (bit 0 / 1 of `uns`: c0, c0 + 1): no
// within-block entries in R^(a); R^(a2), a2 > a, and Kend formed directly as
// k e^{P_{a2} - G_i} and k e^{G_last - G_i} (exponents <= 0).  With conv, also
// stages the normalised k, q as bf16 [row][128] in the record's U^T and W^T areas
// for the exact pair pass (the record's own images overwrite them at the end).
__device__ __noinline__ void prep_unsafe_direct(uint8_t* sm, uint8_t* rc, int a, int c0, int uns,
                                                bool conv, bool bf, const UnsafeRows& ur) {
#pragma unroll 1
  for (int ch = 0; ch < 2; ++ch) {
    if (!((uns >> ch) & 1)) continue;
    const int c = c0 + ch;
#pragma unroll
    for (int gg = 0; gg < 2; ++gg) {
      const int g8 = 2 * a + gg;
      sts16(sm, q_r(a) + chunk_mnmajor_sw32(g8, c, D), make_uint4(0u, 0u, 0u, 0u));
      float v[8];
#pragma unroll 1
      for (int a2 = a + 1; a2 < 4; ++a2) {
#pragma unroll
        for (int e = 0; e < 8; ++e)
          v[e] = ur.k[ch][8 * gg + e] * __expf(fminf(ur.d[ch][a2] - ur.x[ch][8 * gg + e], 0.f));
        sts16(sm, q_r(a2) + chunk_mnmajor_sw32(g8, c, D), pack8(v, 1.f));
      }
#pragma unroll
      for (int e = 0; e < 8; ++e)
        v[e] = ur.k[ch][8 * gg + e] * __expf(fminf(ur.tl[ch] - ur.x[ch][8 * gg + e], 0.f));
      *reinterpret_cast<uint4*>(rc + REC_KA + chunk_kmajor_sw128(c, g8, D)) =
          bf ? pack8(v, 1.f) : pack8_f16(v, 1.f);
      if (conv) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int row = 16 * a + 8 * gg + e;
          reinterpret_cast<bf16*>(rc + REC_U)[row * D + c] = __float2bfloat16_rn(ur.k[ch][8 * gg + e]);
          reinterpret_cast<bf16*>(rc + REC_QW + 16384)[row * D + c] =
              __float2bfloat16_rn(ur.q[ch][8 * gg + e]);
        }
      }
    }
  }
}

// UnsafeRows of this thread's channel pair and block a, re-read from the inputs in
// global memory (other warps may already be overwriting the staged tiles), with
// the cumulative decay summed in the prep kernel's order; d1..d3, rel: P_{a2} - P_a
// + g_{16a} and the decay of blocks a..3 (per channel); gsh: one decay per group of
// 2^gsh channels.
__device__ __noinline__ void fill_unsafe_rows(UnsafeRows& ur, const float* __restrict__ g,
                                              const bf16* __restrict__ k,
                                              const bf16* __restrict__ q, long long rbase, int H,
                                              int h, int dk, int gsh, int L, int a, int c0,
                                              float2 d1, float2 d2, float2 d3, float2 rel) {
  float2 loc = make_float2(0.f, 0.f), first = make_float2(0.f, 0.f);
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    const int r = 16 * a + e;
    float2 gv = make_float2(0.f, 0.f);
    uint32_t kv = 0u, qv = 0u;
    if (r < L && c0 < dk) {
      const long long idx = ((rbase + r) * H + h) * dk + c0;
      kv = *reinterpret_cast<const uint32_t*>(k + idx);
      qv = *reinterpret_cast<const uint32_t*>(q + idx);
      if (gsh != 0) {                          // g [rows, H, dk >> gsh]
        const float t = g[((rbase + r) * H + h) * (dk >> gsh) + (c0 >> gsh)];
        gv = make_float2(t, t);
      } else {
        gv = *reinterpret_cast<const float2*>(g + idx);
      }
    }
    if (e == 0) {
      loc = gv;
      first = gv;
    } else {
      loc.x += gv.x;
      loc.y += gv.y;
    }
    ur.x[0][e] = loc.x - first.x;
    ur.x[1][e] = loc.y - first.y;
    ur.k[0][e] = bf_lo(kv);
    ur.k[1][e] = bf_hi(kv);
    ur.q[0][e] = bf_lo(qv);
    ur.q[1][e] = bf_hi(qv);
  }
  const float2 dd[4] = {make_float2(0.f, 0.f), d1, d2, d3};
#pragma unroll
  for (int a2 = 0; a2 < 4; ++a2) {
    ur.d[0][a2] = dd[a2].x - first.x;
    ur.d[1][a2] = dd[a2].y - first.y;
  }
  ur.tl[0] = rel.x - first.x;
  ur.tl[1] = rel.y - first.y;
}

// The exact within-block pair terms of this thread's unsafe channels (c0, c0 + 1;
// flags ux, uy) of one 16-row block, added to the block's corrections (A, Aqk:
// [r][i], row stride 16).  Warp-cooperative.  Reloads the block's rows: g (one
// value per channel, or per group of 2^gsh channels; `gst` apart), k and q (bf16
// channel pairs, `kst` apart); rows >= nrows are not read.  Out of line: it runs
// only for chunks with unsafe channels and keeps its registers to itself.
__device__ __noinline__ void prep_unsafe_pairs(const float* __restrict__ g, long long gix,
                                               long long gst, int gsh, const bf16* kp,
                                               const bf16* qp, long long kst, int nrows, bool ux,
                                               bool uy, float* corrA, float* corrQ, int lane) {
  if (!__any_sync(0xffffffffu, ux || uy)) return;
  float al[16][2], kv[16][2], qv[16][2];
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    float2 gg = make_float2(0.f, 0.f);
    uint32_t kw = 0u, qw = 0u;
    if (e < nrows && (ux || uy)) {
      if (gsh == 0) {
        gg = *reinterpret_cast<const float2*>(g + gix + e * gst);
      } else {
        const float t = g[gix + e * gst];
        gg = make_float2(t, t);
      }
      kw = *reinterpret_cast<const uint32_t*>(kp + e * kst);
      qw = *reinterpret_cast<const uint32_t*>(qp + e * kst);
    }
    al[e][0] = __expf(gg.x);
    al[e][1] = __expf(gg.y);
    kv[e][0] = ux ? bf_lo(kw) : 0.f;
    kv[e][1] = uy ? bf_hi(kw) : 0.f;
    qv[e][0] = ux ? bf_lo(qw) : 0.f;
    qv[e][1] = uy ? bf_hi(qw) : 0.f;
  }
  add_pair_terms<2, 16>(al, kv, qv, corrA, corrQ, lane);
}

// ============================================================================
// Prep kernel: one CTA per (chunk slot, head).  CONV: q and k are the raw
// projections; each is convolved causally per channel (width convW <= 4, history
// reset at the document start), L2-normalised per token, and q scaled by dk^-1/2.
// BWD: the backward's record (bf16 images, T as a bf16 image too, and A in fp32).
// ============================================================================
template <bool CONV, bool GRPD, bool BWD = false>
__global__ void __launch_bounds__(NT, 2)
kda_chunk_prep_kernel(const bf16* __restrict__ q, const bf16* __restrict__ k,
                      const bf16* __restrict__ v, const float* __restrict__ g,
                      const float* __restrict__ beta, const int32_t* __restrict__ cu_seqlens,
                      uint8_t* __restrict__ rec, int B, int T, int H, int dk, int dv, int gsh,
                      long long nslots, const float* __restrict__ conv_q,
                      const float* __restrict__ conv_k, int convW,
                      const __grid_constant__ PrepMaps maps, int tma) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1024(smem_raw);
  __shared__ uint64_t bar, in_bar;
  __shared__ uint32_t tmem_base_sh;
  __shared__ float s_beta[C];
  __shared__ float2 s_sum[4][64];       // per 16-row block: its total log-decay (channel pair)
  __shared__ float2 s_first[4][64];     // per 16-row block: g at its first row
  __shared__ float s_ss[CONV ? 4 * 2 * 2 * 16 : 1];   // [block][warp][k|q][row]: sums of squares
  __shared__ uint8_t s_uns[NT];         // per thread: bit 0 / 1 = channel c0 / c0 + 1 unsafe
  __shared__ long long s_rbase;
  __shared__ int s_L;

  const int tid = threadIdx.x, warp = tid >> 5;
  const long long slot = blockIdx.x;
  const int h = blockIdx.y;
  grid_dep_launch();          // the state pass may take SMs this grid no longer needs

  // which chunk of which sequence this slot is (uniform over the CTA)
  long long row0 = 0, t_beg = 0, t_end = 0, n = 0;
  if (!cu_seqlens) {
    const long long per = chunk_count(T);
    if (per == 0 || slot >= per * B) return;
    const int s = (int)(slot / per);
    n = slot - (long long)s * per;
    seq_range(nullptr, s, T, row0, t_beg, t_end);
  } else {
    long long base = 0;
    bool found = false;
    for (int d = 0; d < B && !found; ++d) {
      seq_range(cu_seqlens, d, T, row0, t_beg, t_end);
      const long long nc = chunk_count(t_end - t_beg);
      if (slot < base + nc) { n = slot - base; found = true; }
      base += nc;
    }
    if (!found) return;
  }
  const long long t0 = t_beg + n * C;
  const int L = (int)min((long long)C, t_end - t0);
  const long long rbase = row0 + t0;                   // first token row of the chunk
  uint8_t* rc = rec + ((size_t)h * (size_t)nslots + (size_t)slot) * (BWD ? rec::BYTES_BWD : REC_BYTES);

  // The chunk's tiles.  TMA (tma != 0; not with the fused convolution): v straight
  // into the MN-major operand of U^T (two 64-value boxes, 128-byte swizzle), q and k
  // row-major into the Gram operand area and g into the R area (both free until the
  // operand build), all on one mbarrier.  Otherwise v by cp.async and q, k, g by
  // per-thread loads below.  Rows >= L are never used from the staged tiles; the v
  // rows >= L are zeroed once the tile has landed.
  const bool use_tma = !CONV && tma != 0;
  if (use_tma) {
    if (tid == 0) {
      mbar_init(&in_bar, 1);
      mbar_init(&bar, 1);
      fence_mbar_init();
      const uint32_t bytes =
          (uint32_t)(C * dv * 2 + 2 * C * dk * 2 + (gsh == 0 ? C * dk * 4 : 0));
      mbar_arrive_expect_tx(&in_bar, bytes);
      const int row = (int)rbase;               // < 2^31 - 64 (checked on the host)
      tma_load_3d(sm + Q_V, &maps.v, 0, h, row, &in_bar);
      if (dv > 64) tma_load_3d(sm + Q_V + 8192, &maps.v, 64, h, row, &in_bar);
      tma_load_3d(sm + Q_L, &maps.q, 0, h, row, &in_bar);
      tma_load_3d(sm + Q_L + 16384, &maps.k, 0, h, row, &in_bar);
      if (gsh == 0) tma_load_3d(sm + Q_R, &maps.g, 0, h, row, &in_bar);
    }
  } else {
#pragma unroll
    for (int it = 0; it < 4; ++it) {
      const int idx = tid + it * NT;
      const int r = idx >> 4, ch = idx & 15;
      const long long e = ((rbase + min(r, L - 1)) * H + h) * dv + min(ch * 8, dv - 8);
      cp_async16(sm + Q_V + chunk_mnmajor_sw128(ch, r, C), v + e,
                 (r < L && ch * 8 < dv) ? 16u : 0u);
    }
    cp_async_commit();
  }
  if (tid < C) s_beta[tid] = tid < L ? beta[(rbase + tid) * H + h] : 0.f;
  // ---- P1: per thread a channel pair (2cp, 2cp+1) and a 16-row block a
  const int cp = tid & 63, a = tid >> 6, c0 = 2 * cp;
  float2 gq[16];
  if constexpr (GRPD) {                          // one decay per group of 2^gsh channels: its
#pragma unroll                                   // loads go out before the tiles are waited for
    for (int e = 0; e < 16; ++e) {
      const int r = 16 * a + e;
      float gg = 0.f;
      if (r < L && c0 < dk) gg = __ldg(g + ((rbase + r) * H + h) * (dk >> gsh) + (c0 >> gsh));
      gq[e] = make_float2(gg, gg);
    }
  }
  if (warp == 0) {
    tmem_alloc(&tmem_base_sh, kPrepTmemCols);
    tmem_relinquish();
  }
  if (!use_tma && tid == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  if (use_tma) {
    tc_fence_before();
    __syncthreads();                            // in_bar is initialised
    tc_fence_after();
    bool got = true;
    if (warp == 0) got = mbar_wait(&in_bar, 0, kWaitLimit);
    if (__syncthreads_or(!got)) {
      // the tiles never arrived: raise the flag, let the copies finish, free TMEM
      if (tid == 0) {
        atomicExch(&g_chunk_split_timeout, 1);
        mbar_wait(&in_bar, 0, kWaitLimit);
      }
      tc_fence_before();
      __syncthreads();
      if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem_base_sh, kPrepTmemCols);
      }
      return;
    }
    // v: rows >= L, and values >= dv, to zero
    if (L < C || dv < D) {
      for (int i = tid; i < C * 16; i += NT) {
        const int r = i >> 4, ch = i & 15;
        if (r >= L || ch * 8 >= dv) sts16(sm, Q_V + chunk_mnmajor_sw128(ch, r, C),
                                           make_uint4(0u, 0u, 0u, 0u));
      }
    }
  }

  uint32_t kw[16], qw[16];
  float2 kf[CONV ? 16 : 1], qf[CONV ? 16 : 1];   // CONV: fp32 convolution outputs
  // branch-free loops per source, so that all of a thread's loads issue back to back
  if (use_tma) {                                 // staged tiles: row stride dk
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const int r = 16 * a + e;
      const bool ok = r < L && c0 < dk;
      const int si = ok ? r * dk + c0 : 0;
      const uint32_t kv = *reinterpret_cast<const uint32_t*>(sm + Q_L + 16384 + 2 * si);
      const uint32_t qv = *reinterpret_cast<const uint32_t*>(sm + Q_L + 2 * si);
      if constexpr (!GRPD) {
        const float2 gv = *reinterpret_cast<const float2*>(sm + Q_R + 4 * si);
        gq[e] = ok ? gv : make_float2(0.f, 0.f);
      }
      kw[e] = ok ? kv : 0u;
      qw[e] = ok ? qv : 0u;
    }
  } else {
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const int r = 16 * a + e;
      if (r < L && c0 < dk) {
        const long long idx = ((rbase + r) * H + h) * dk + c0;
        if constexpr (!GRPD) gq[e] = __ldg(reinterpret_cast<const float2*>(g + idx));
        if constexpr (!CONV) {
          kw[e] = __ldg(reinterpret_cast<const unsigned int*>(k + idx));
          qw[e] = __ldg(reinterpret_cast<const unsigned int*>(q + idx));
        }
      } else {
        if constexpr (!GRPD) gq[e] = make_float2(0.f, 0.f);
        kw[e] = 0u;
        qw[e] = 0u;
      }
    }
  }
  if constexpr (CONV) {
    // x_conv[r] = sum_i w[i] x[r - (W-1) + i]: a 4-tap window whose first 4 - W taps
    // are zero; rows before the document start and at or after L read as zero.
    const long long doc0 = row0 + t_beg;
    auto conv = [&](const bf16* __restrict__ x, const float* __restrict__ w,
                    float2 (&o)[16], int which) {
      float2 wt[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int i = j - (4 - convW);
        wt[j] = make_float2(0.f, 0.f);
        if (i >= 0 && c0 < dk)
          wt[j] = make_float2(__ldg(w + ((long long)h * dk + c0) * convW + i),
                              __ldg(w + ((long long)h * dk + c0 + 1) * convW + i));
      }
      // rows 16 a - 3 .. 16 a + 15, all loads issued before any use; one pointer walks
      // the rows (stride H dk), rows outside [doc0 - rbase, L) read as zero
      uint32_t u[19];
      const int rlo = (int)max(doc0 - rbase, -3LL) - (16 * a - 3);   // first valid m
      const int rhi = L - (16 * a - 3);                              // first invalid m
      const long long stride = (long long)H * dk;
      const bf16* px = x + ((rbase + 16 * a - 3) * H + h) * dk + c0;
#pragma unroll
      for (int m = 0; m < 19; ++m) {
        const bool ok = c0 < dk && m >= rlo && m < rhi;
        u[m] = ok ? __ldg(reinterpret_cast<const unsigned int*>(px + m * stride)) : 0u;
      }
      auto raw = [&](int m) { return make_float2(bf_lo(u[m]), bf_hi(u[m])); };
      float2 w0 = raw(0), w1 = raw(1), w2 = raw(2);
      float ss[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const float2 cur = raw(e + 3);
        const float ox = fmaf(wt[3].x, cur.x, fmaf(wt[2].x, w2.x, fmaf(wt[1].x, w1.x, wt[0].x * w0.x)));
        const float oy = fmaf(wt[3].y, cur.y, fmaf(wt[2].y, w2.y, fmaf(wt[1].y, w1.y, wt[0].y * w0.y)));
        o[e] = 16 * a + e < L ? make_float2(ox, oy) : make_float2(0.f, 0.f);
        ss[e] = fmaf(o[e].x, o[e].x, o[e].y * o[e].y);
        w0 = w1; w1 = w2; w2 = cur;
      }
      const float tot = rowsum16(ss, tid & 31);
      if ((tid & 1) == 0) s_ss[((a * 2 + (warp & 1)) * 2 + which) * 16 + ((tid & 31) >> 1)] = tot;
    };
    conv(k, conv_k, kf, 0);
    conv(q, conv_q, qf, 1);
  }
#pragma unroll
  for (int e = 1; e < 16; ++e) {
    gq[e].x += gq[e - 1].x;
    gq[e].y += gq[e - 1].y;
  }
  s_sum[a][cp] = gq[15];
  s_first[a][cp] = gq[0];
  // a channel whose decay inside this block is too strong for the reference-point
  // split: its within-block pairs are added exactly after the Gram (decay_pairs.cuh)
  const bool ux = c0 < dk && gq[0].x - gq[15].x > kUnsafeDecay;
  const bool uy = c0 < dk && gq[0].y - gq[15].y > kUnsafeDecay;
  s_uns[tid] = (uint8_t)((ux ? 1 : 0) | (uy ? 2 : 0));
  if (tid == 0) {
    s_rbase = rbase;
    s_L = L;
  }
  tc_fence_before();
  const bool fix = __syncthreads_or(ux || uy) != 0;
  tc_fence_after();
  const uint32_t tb = tmem_base_sh;
  const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
  if constexpr (CONV) {                 // L2 norms of this block's rows (two warps' sums)
    // lane l < 16 forms row l's inverse norms; the other lanes take them by shuffle
    const int lr = (tid & 31) & 15;
    const float ik_l = rsqrtf(fmaxf(s_ss[((a * 2) * 2) * 16 + lr] +
                                        s_ss[((a * 2 + 1) * 2) * 16 + lr],
                                    kNormEps2));
    const float iq_l = rsqrtf(fmaxf(s_ss[((a * 2) * 2 + 1) * 16 + lr] +
                                        s_ss[((a * 2 + 1) * 2 + 1) * 16 + lr],
                                    kNormEps2) * (float)dk);
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const float ik = __shfl_sync(0xffffffffu, ik_l, e);
      const float iq = __shfl_sync(0xffffffffu, iq_l, e);
      kf[e].x *= ik; kf[e].y *= ik;
      qf[e].x *= iq; qf[e].y *= iq;
    }
  }

  // Per channel, from per-block sums only: off = P_a - g_{16a} (the blocks before
  // this one), rel = the decay of blocks a..3, d[a2] = P_{a2} - P_a + g_{16a}.
  float2 d[4], off = make_float2(0.f, 0.f), rel = make_float2(0.f, 0.f);
#pragma unroll
  for (int a2 = 0; a2 < 4; ++a2) {
    const float2 f = s_first[a2][cp], sm2 = s_sum[a2][cp];
    d[a2] = make_float2(rel.x + f.x, rel.y + f.y);
    if (a2 < a) {
      off.x += sm2.x;
      off.y += sm2.y;
    } else {
      rel.x += sm2.x;
      rel.y += sm2.y;
    }
  }
  const float2 fo = gq[0];                     // g at the block's first row
  auto kval = [&](int idx, int ch) -> float {
    if constexpr (!CONV) return ch ? bf_hi(kw[idx]) : bf_lo(kw[idx]);
    else return ch ? kf[idx].y : kf[idx].x;              // normalised above
  };
  auto qval = [&](int idx, int ch) -> float {
    if constexpr (!CONV) return ch ? bf_hi(qw[idx]) : bf_lo(qw[idx]);
    else return ch ? qf[idx].y : qf[idx].x;
  };

  if (!CONV && (ux || uy)) {
    // unsafe channels: their operands are formed out of line from the block's rows,
    // re-read from global memory (the loop below skips their R and Kend stores);
    // nothing of this stays in the common path
    UnsafeRows ur;
    fill_unsafe_rows(ur, g, k, q, rbase, H, h, dk, gsh, L, a, c0, d[1], d[2], d[3], rel);
    prep_unsafe_direct(sm, rc, a, c0, (ux ? 1 : 0) | (uy ? 2 : 0), false, BWD, ur);
  }
  if (CONV && (ux || uy)) {
    // fused convolution: the normalised q, k exist only in registers, so they go
    // over on the stack
    UnsafeRows ur;
#pragma unroll
    for (int ch = 0; ch < 2; ++ch) {
      const float first = ch ? fo.y : fo.x;
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        ur.x[ch][e] = (ch ? gq[e].y : gq[e].x) - first;
        ur.k[ch][e] = kval(e, ch);
        ur.q[ch][e] = qval(e, ch);
      }
#pragma unroll
      for (int a2 = 0; a2 < 4; ++a2) ur.d[ch][a2] = (ch ? d[a2].y : d[a2].x) - first;
      ur.tl[ch] = (ch ? rel.y : rel.x) - first;
    }
    prep_unsafe_direct(sm, rc, a, c0, (ux ? 1 : 0) | (uy ? 2 : 0), CONV, BWD, ur);
  }

  // the operand images of this thread's channel pair and 16-row block
  auto put_rows = [&](int ch, int g8, const float (&lk)[8], const float (&lq)[8],
                      const float (&kr)[8], float eP, float eE, const float (&f)[4]) {
    const int c = c0 + ch;
    const bool uns = ch ? uy : ux;
    if (c0 < dk) {
      // the Gram operands (its K loop covers channels < dk only)
      sts16(sm, Q_L + chunk_mnmajor_sw128(g8, c, D), pack8(lk, 1.f));
      sts16(sm, Q_L + chunk_mnmajor_sw128(8 + g8, c, D), pack8(lq, 1.f));
      if (!uns) {
#pragma unroll
        for (int a2 = 0; a2 < 4; ++a2)
          if (a2 >= a) sts16(sm, q_r(a2) + chunk_mnmajor_sw32(g8, c, D), pack8(kr, f[a2]));
      }
    }
    sts16(sm, Q_KB + chunk_kmajor_sw128(c, g8, D), pack8(lk, eP));
    // record: Qbar^T (MN-major, N = tokens, K = channels) and Kend^T (K-major)
    *reinterpret_cast<uint4*>(rc + REC_QW + chunk_mnmajor_sw128(g8, c, D)) = pack8(lq, eP);
    if (!uns)
      *reinterpret_cast<uint4*>(rc + REC_KA + chunk_kmajor_sw128(c, g8, D)) =
          BWD ? pack8(kr, eE) : pack8_f16(kr, eE);
  };
  if constexpr (GRPD) {
    // one decay per group of at least two channels: the pair's exponentials are shared
    const float first = fo.x;
    const float eP = __expf(off.x + first);   // Kbar, Qbar: e^{G_r} = e^{G_r - P_a} e^{P_a}
    const float eE = __expf(rel.x - first);   // Kend: e^{G_last - G_i} = e^{P_a - G_i} e^{G_last - P_a}
    float f[4];
#pragma unroll
    for (int a2 = 0; a2 < 4; ++a2) f[a2] = a2 > a ? __expf(d[a2].x - first) : 1.f;
#pragma unroll
    for (int gg = 0; gg < 2; ++gg) {
      const int g8 = 2 * a + gg;               // group of 8 rows
      float ell[8], rho[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float x = gq[8 * gg + e].x - first;                  // G_r - P_a
        ell[e] = __expf(x);
        rho[e] = __expf(fminf(-x, 80.f));
      }
#pragma unroll
      for (int ch = 0; ch < 2; ++ch) {
        float lk[8], lq[8], kr[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float kv = c0 < dk ? kval(8 * gg + e, ch) : 0.f;
          const float qv = c0 < dk ? qval(8 * gg + e, ch) : 0.f;
          lk[e] = kv * ell[e];
          lq[e] = qv * ell[e];
          kr[e] = kv * rho[e];                 // k_i e^{P_a - G_i}
        }
        put_rows(ch, g8, lk, lq, kr, eP, eE, f);
      }
    }
  } else {
#pragma unroll
    for (int ch = 0; ch < 2; ++ch) {
      const float first = ch ? fo.y : fo.x;
      const float eP = __expf((ch ? off.y : off.x) + first);
      const float eE = __expf((ch ? rel.y : rel.x) - first);
      float f[4];
#pragma unroll
      for (int a2 = 0; a2 < 4; ++a2)
        f[a2] = a2 > a ? __expf((ch ? d[a2].y : d[a2].x) - first) : 1.f;   // e^{P_{a2} - P_a}
#pragma unroll
      for (int gg = 0; gg < 2; ++gg) {
        const int g8 = 2 * a + gg;             // group of 8 rows
        float lk[8], lq[8], kr[8];
        if (c0 < dk) {
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int idx = 8 * gg + e;
            const float x = (ch ? gq[idx].y : gq[idx].x) - first;   // G_r - P_a
            const float ell = __expf(x);
            const float rho = __expf(fminf(-x, 80.f));
            const float kv = kval(idx, ch), qv = qval(idx, ch);
            lk[e] = kv * ell;
            lq[e] = qv * ell;
            kr[e] = kv * rho;                  // k_i e^{P_a - G_i}
          }
        } else {                       // padded channels (dk = 64; whole warps): zeros
#pragma unroll
          for (int e = 0; e < 8; ++e) lk[e] = lq[e] = kr[e] = 0.f;
        }
        put_rows(ch, g8, lk, lq, kr, eP, eE, f);
      }
    }
  }
  if (a == 3)                                  // exp(G_last), G_last = off + rel
    *reinterpret_cast<float2*>(rc + REC_DECAY + 4 * c0) =
        make_float2(__expf(off.x + rel.x), __expf(off.y + rel.y));
  cp_async_wait_all();
  fence_async_smem();
  tc_fence_before();
  __syncthreads();

  uint32_t phase = 0;
  // one warp polls the MMA barrier; the others sleep in the CTA barrier and
  // leave the issue slots to the SM's other CTA
  auto mma_wait = [&]() -> bool {
    bool good = true;
    if (warp == 0) good = mbar_wait(&bar, phase, kWaitLimit);
    phase ^= 1u;
    const bool ok = __syncthreads_or(!good) == 0;
    tc_fence_after();
    return ok;
  };
  bool alive = true;

  // ---- P2: Gram (one MMA per K step, N = 160)
  if (tid == 0) {
    tc_fence_after();
    const uint32_t idesc = idesc_bf16(128, 160, true, true);
    // K step kk: 2048 bytes further in L, 512 in R (descriptor address fields)
    const uint64_t a0 = desc_mnmajor_sw128(smem_u32(sm + Q_L), D, 0);
    const uint64_t b0 = desc_mnmajor_sw32(smem_u32(sm + q_r(0)), D, 0);
    const int nk = dk / 16;                    // channels < dk (64-wide heads: half the steps)
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk)
      if (kk < nk)
        mma_ss(tb + PT_G, a0 + (uint64_t)(kk * 128), b0 + (uint64_t)(kk * 32), idesc, kk > 0);
    mma_commit(&bar);
  }
  __syncwarp();
  if (!mma_wait()) alive = false;

  if (alive && fix) {
    // exact within-block pairs of the unsafe channels into the corrections (R^(3)'s
    // area, free once the Gram has completed): A at [block][r][i], Aqk 4 KB above
    float4* cz = reinterpret_cast<float4*>(sm + Q_CORR);
    cz[tid] = make_float4(0.f, 0.f, 0.f, 0.f);
    cz[tid + NT] = make_float4(0.f, 0.f, 0.f, 0.f);
    __syncthreads();
    // (rbase, L and the flags come back from shared memory: nothing of this stays
    // live in registers across the common path)
    const long long rb = s_rbase;
    const int u = s_uns[tid];
    const int ta = tid >> 6, tc0 = 2 * (tid & 63);
    const int nrows = max(0, min(16, s_L - 16 * ta));
    const long long gst = (long long)H * (dk >> gsh);
    const long long gix = ((rb + 16 * ta) * H + h) * (dk >> gsh) + (tc0 >> gsh);
    const bf16 *kp, *qp;
    long long kst;
    if constexpr (CONV) {
      kp = reinterpret_cast<const bf16*>(rc + REC_U) + 16 * ta * D + tc0;
      qp = reinterpret_cast<const bf16*>(rc + REC_QW + 16384) + 16 * ta * D + tc0;
      kst = D;
    } else {
      kp = k + ((rb + 16 * ta) * H + h) * dk + tc0;
      qp = q + ((rb + 16 * ta) * H + h) * dk + tc0;
      kst = (long long)H * dk;
    }
    float* corr = reinterpret_cast<float*>(sm + Q_CORR);
    prep_unsafe_pairs(g, gix, gst, gsh, kp, qp, kst, nrows, (u & 1) != 0, (u & 2) != 0,
                      corr + 256 * ta, corr + 1024 + 256 * ta, tid & 31);
    if constexpr (CONV) fence_async_global();   // the staged rows are overwritten by bulk copies
    __syncthreads();
  }

  float* B32 = reinterpret_cast<float*>(sm + Q_B32);
  float* T32 = reinterpret_cast<float*>(sm + Q_T32);
  float* M32 = reinterpret_cast<float*>(sm + Q_M32);
  if (alive) {
    // ---- P3: read A (beta-scaled, strictly lower, into B32) and Aqk (record)
    // warp w (mod 4) reads TMEM lanes 32w..32w+31: w%4 = 0,1 -> A rows, 2,3 -> Aqk rows.
    // Rows of a warp lie in blocks a0, a0+1; the lower warpgroup handles block a0
    // and the upper warpgroup block a0+1.
    const bool upper = tid >= 128;
    const int w4 = warp & 3;
    const int lane = tid & 31;
    const int r = (w4 & 1) * 32 + lane;
    const bool isA = w4 < 2;
    const int a0 = (w4 & 1) * 2;
    const int ab = a0 + (upper ? 1 : 0);
    const int colb = ab == 0 ? 0 : ab == 1 ? 16 : ab == 2 ? 48 : 96;
    const int nb = 16 * (ab + 1);
    const bool mine = (r >> 4) == ab;
    uint32_t tv[4][16];
#pragma unroll
    for (int q4 = 0; q4 < 4; ++q4) {
      if (16 * q4 < nb) tmem_ld16(tb + lane_base + PT_G + colb + 16 * q4, tv[q4]);
      else {
#pragma unroll
        for (int e = 0; e < 16; ++e) tv[q4][e] = 0u;
      }
    }
    tmem_wait_ld();
    if (fix && mine) {               // the exact within-block pairs of unsafe channels
      const float* cr = reinterpret_cast<const float*>(sm + Q_CORR) + (isA ? 0 : 1024) +
                        256 * ab + 16 * (r - 16 * ab);
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4)
        if (q4 == ab) {
#pragma unroll
          for (int e = 0; e < 16; ++e)
            tv[q4][e] = __float_as_uint(__uint_as_float(tv[q4][e]) + cr[e]);
        }
    }
    if (mine) {
      if (isA) {
        const float br = s_beta[r];
        if constexpr (BWD) {                 // A itself, strictly lower, for the backward
          float4* ar = reinterpret_cast<float4*>(rc + rec::AMAT) + 16 * r;
#pragma unroll
          for (int i4 = 0; i4 < 16; ++i4) {
            float4 w;
            w.x = (4 * i4 + 0 < r) ? __uint_as_float(tv[i4 >> 2][(4 * i4 + 0) & 15]) : 0.f;
            w.y = (4 * i4 + 1 < r) ? __uint_as_float(tv[i4 >> 2][(4 * i4 + 1) & 15]) : 0.f;
            w.z = (4 * i4 + 2 < r) ? __uint_as_float(tv[i4 >> 2][(4 * i4 + 2) & 15]) : 0.f;
            w.w = (4 * i4 + 3 < r) ? __uint_as_float(tv[i4 >> 2][(4 * i4 + 3) & 15]) : 0.f;
            ar[i4] = w;
          }
        }
#pragma unroll
        for (int i4 = 0; i4 < 16; ++i4) {
          float4 w;
          w.x = (4 * i4 + 0 < r) ? br * __uint_as_float(tv[i4 >> 2][(4 * i4 + 0) & 15]) : 0.f;
          w.y = (4 * i4 + 1 < r) ? br * __uint_as_float(tv[i4 >> 2][(4 * i4 + 1) & 15]) : 0.f;
          w.z = (4 * i4 + 2 < r) ? br * __uint_as_float(tv[i4 >> 2][(4 * i4 + 2) & 15]) : 0.f;
          w.w = (4 * i4 + 3 < r) ? br * __uint_as_float(tv[i4 >> 2][(4 * i4 + 3) & 15]) : 0.f;
          *reinterpret_cast<float4*>(B32 + r * LDA + 4 * i4) = w;
        }
      } else {
        // Aqk row r: rows 128.. of the K-major [Kend^T ; Aqk] record operand
#pragma unroll
        for (int c8 = 0; c8 < 8; ++c8) {
          float w[8];
#pragma unroll
          for (int e = 0; e < 8; ++e)
            w[e] = (c8 * 8 + e <= r) ? __uint_as_float(tv[c8 >> 1][(c8 & 1) * 8 + e]) : 0.f;
          sts16(sm, Q_OAQK + chunk_kmajor_sw128(r, c8, C), BWD ? pack8(w, 1.f) : pack8_f16(w, 1.f));
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();

  if (alive) {
    // ---- triangular inverse T = (I + B)^-1, B = diag(beta) A
    if (tid < 64) {                         // diagonal blocks: forward substitution
      const int ab = tid >> 4, jj = tid & 15, o = 16 * ab;
      float x[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) x[i] = (i == jj) ? 1.f : 0.f;
#pragma unroll
      for (int i = 1; i < 16; ++i) {
        float acc = 0.f;
#pragma unroll
        for (int m = 0; m < i; ++m) acc = fmaf(B32[(o + i) * LDA + o + m], x[m], acc);
        if (i > jj) x[i] = -acc;
      }
#pragma unroll
      for (int i = 0; i < 16; ++i) T32[(o + i) * LDA + o + jj] = x[i];
    }
    __syncthreads();
    // M_am = T_aa B_am for the 6 pairs a > m (p = a(a-1)/2 + m); 384 items of
    // 4 outputs, two accumulator chains each
#pragma unroll 1
    for (int w = tid; w < 384; w += NT) {
      const int p = w >> 6, i = (w >> 2) & 15, jq = w & 3;
      const int ar = p == 0 ? 1 : (p < 3 ? 2 : 3);
      const int m = p - ar * (ar - 1) / 2;
      const float* Ti = T32 + (16 * ar + i) * LDA + 16 * ar;
      const float* Bc = B32 + 16 * ar * LDA + 16 * m + 4 * jq;
      float4 s0 = make_float4(0.f, 0.f, 0.f, 0.f), s1 = s0;
#pragma unroll
      for (int l = 0; l < 16; l += 2) {
        const float4 b0 = *reinterpret_cast<const float4*>(Bc + l * LDA);
        const float4 b1 = *reinterpret_cast<const float4*>(Bc + (l + 1) * LDA);
        const float t0v = Ti[l], t1v = Ti[l + 1];
        s0.x = fmaf(t0v, b0.x, s0.x); s0.y = fmaf(t0v, b0.y, s0.y);
        s0.z = fmaf(t0v, b0.z, s0.z); s0.w = fmaf(t0v, b0.w, s0.w);
        s1.x = fmaf(t1v, b1.x, s1.x); s1.y = fmaf(t1v, b1.y, s1.y);
        s1.z = fmaf(t1v, b1.z, s1.z); s1.w = fmaf(t1v, b1.w, s1.w);
      }
      *reinterpret_cast<float4*>(M32 + p * 256 + i * 16 + 4 * jq) =
          make_float4(s0.x + s1.x, s0.y + s1.y, s0.z + s1.z, s0.w + s1.w);
    }
    __syncthreads();
    // block rows a = 1, 2, 3: T_ab = -sum_{m=b}^{a-1} M_am T_mb; thread (q, i, jq)
    // computes 4 columns of row i of block (a, q)
    auto mt = [&](int p, int m, int i, int col) -> float4 {   // (M_p T)[i][col..col+3] over block m
      const float* Mr = M32 + p * 256 + i * 16;
      const float* Tc = T32 + 16 * m * LDA + col;
      float4 s0 = make_float4(0.f, 0.f, 0.f, 0.f), s1 = s0;
#pragma unroll
      for (int l4 = 0; l4 < 4; ++l4) {
        const float4 m4 = *reinterpret_cast<const float4*>(Mr + 4 * l4);
        const float mv[4] = {m4.x, m4.y, m4.z, m4.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float4 t4 = *reinterpret_cast<const float4*>(Tc + (4 * l4 + e) * LDA);
          float4& sacc = (e & 1) ? s1 : s0;
          sacc.x = fmaf(mv[e], t4.x, sacc.x); sacc.y = fmaf(mv[e], t4.y, sacc.y);
          sacc.z = fmaf(mv[e], t4.z, sacc.z); sacc.w = fmaf(mv[e], t4.w, sacc.w);
        }
      }
      return make_float4(s0.x + s1.x, s0.y + s1.y, s0.z + s1.z, s0.w + s1.w);
    };
    auto put = [&](int row, int col, float4 x) {
      *reinterpret_cast<float4*>(T32 + row * LDA + col) = make_float4(-x.x, -x.y, -x.z, -x.w);
    };
    if (tid < 64) {                                            // T_10
      const int i = tid >> 2, jq = tid & 3;
      put(16 + i, 4 * jq, mt(0, 0, i, 4 * jq));
    }
    __syncthreads();
    if (tid < 128) {                                           // T_20, T_21
      const int qb = tid >> 6, i = (tid >> 2) & 15, jq = tid & 3;
      const int col = 16 * qb + 4 * jq;
      float4 x = mt(2, 1, i, col);                             // M_21 T_1q
      if (qb == 0) {
        const float4 y = mt(1, 0, i, col);                     // M_20 T_00
        x.x += y.x; x.y += y.y; x.z += y.z; x.w += y.w;
      }
      put(32 + i, col, x);
    }
    __syncthreads();
    if (tid < 192) {                                           // T_30, T_31, T_32
      const int qb = tid >> 6, i = (tid >> 2) & 15, jq = tid & 3;
      const int col = 16 * qb + 4 * jq;
      float4 x = mt(5, 2, i, col);                             // M_32 T_2q
      if (qb <= 1) {
        const float4 y = mt(4, 1, i, col);                     // M_31 T_1q
        x.x += y.x; x.y += y.y; x.z += y.z; x.w += y.w;
      }
      if (qb == 0) {
        const float4 y = mt(3, 0, i, col);                     // M_30 T_00
        x.x += y.x; x.y += y.y; x.z += y.z; x.w += y.w;
      }
      put(48 + i, col, x);
    }
    __syncthreads();
    if constexpr (BWD) {                       // T for the backward, as a bf16 image [r][i]
      // (the blocks above the diagonal were never written: zeros)
#pragma unroll
      for (int it = 0; it < 2; ++it) {
        const int idx = tid + it * NT, row = idx >> 3, c8 = idx & 7;
        const float4 x0 = *reinterpret_cast<const float4*>(T32 + row * LDA + 8 * c8);
        const float4 x1 = *reinterpret_cast<const float4*>(T32 + row * LDA + 8 * c8 + 4);
        const float xs[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
        float w[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) w[e] = 8 * c8 + e <= row ? xs[e] : 0.f;
        *reinterpret_cast<uint4*>(rc + rec::TMAT + off_kmajor_sw128((uint32_t)row, (uint32_t)(8 * c8), 64u)) =
            pack8(w, 1.f);
      }
    }
    // T diag(beta) as bf16: B operand of W^T / U^T, K-major SW128, N = 64 (r'), K = 64 (r)
#pragma unroll
    for (int it = 0; it < 2; ++it) {
      const int idx = tid + it * NT;
      const int rp = idx >> 3, c8 = idx & 7;
      float w[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const int rr = c8 * 8 + e;
        w[e] = (rr <= rp) ? T32[rp * LDA + rr] * s_beta[rr] : 0.f;
      }
      sts16(sm, Q_TB + chunk_kmajor_sw128(rp, c8, C), pack8(w, 1.f));
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();

    // ---- P4: W^T = Kbar^T (T beta)^T, U^T = V^T (T beta)^T
    if (tid == 0) {
      tc_fence_after();
      const uint32_t tb_base = smem_u32(sm + Q_TB);
      const uint32_t kb_base = smem_u32(sm + Q_KB);
      const uint32_t v_base = smem_u32(sm + Q_V);
      const uint32_t id_w = idesc_bf16(128, 64, false, false);
      const uint32_t id_u = idesc_bf16(128, 64, true, false);
      // K step kk: 32 bytes further along the K-major rows, 2048 in the MN-major V
      const uint64_t bt0 = desc_kmajor_sw128(tb_base, C, 0), kb0 = desc_kmajor_sw128(kb_base, D, 0);
      const uint64_t v0 = desc_mnmajor_sw128(v_base, C, 0);
#pragma unroll
      for (int kk = 0; kk < C / 16; ++kk) {
        const uint64_t bt = bt0 + (uint64_t)(kk * 2);
        mma_ss(tb + PT_W, kb0 + (uint64_t)(kk * 2), bt, id_w, kk > 0);
        mma_ss(tb + PT_U, v0 + (uint64_t)(kk * 128), bt, id_u, kk > 0);
      }
      mma_commit(&bar);
    }
    __syncwarp();
    if (!mma_wait()) alive = false;
  }

  if (alive) {
    // ---- P5: W^T (lower warpgroup) -> bf16 record image; U^T (upper) -> f16
    // record rows (Delta = U - W S is formed in fp32 by the state pass)
    const int j = tid & 127;
    uint32_t t[4][16];
    const uint32_t col = tid < 128 ? PT_W : PT_U;
#pragma unroll
    for (int q4 = 0; q4 < 4; ++q4) tmem_ld16(tb + lane_base + col + 16 * q4, t[q4]);
    tmem_wait_ld();
    if (tid < 128) {
#pragma unroll
      for (int g8 = 0; g8 < 8; ++g8) {
        const uint32_t* f = t[g8 >> 1] + 8 * (g8 & 1);
        const uint4 val = make_uint4(pack_bf16(__uint_as_float(f[0]), __uint_as_float(f[1])),
                                     pack_bf16(__uint_as_float(f[2]), __uint_as_float(f[3])),
                                     pack_bf16(__uint_as_float(f[4]), __uint_as_float(f[5])),
                                     pack_bf16(__uint_as_float(f[6]), __uint_as_float(f[7])));
        sts16(sm, Q_OW + chunk_mnmajor_sw128(g8, j, D), val);
      }
    } else {
#pragma unroll
      for (int c8 = 0; c8 < 8; ++c8) {
        const uint32_t* f = t[c8 >> 1] + 8 * (c8 & 1);
        float x[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) x[e] = __uint_as_float(f[e]);
        sts16(sm, Q_OU + j * 128 + (((uint32_t)c8 ^ (j & 7u)) << 4),
              BWD ? pack8(x, 1.f) : pack8_f16(x, 1.f));
      }
    }
    fence_async_smem();
    __syncthreads();
    if (tid == 0) {                          // the staged images go out as three bulk copies
      bulk_s2g(rc + REC_AQK, sm + Q_OAQK, 8192);
      bulk_s2g(rc + REC_QW + 16384, sm + Q_OW, 16384);
      bulk_s2g(rc + REC_U, sm + Q_OU, 16384);
      bulk_commit();
      bulk_wait_read<0>();                   // shared memory read out before the CTA ends
    }
  }

  if (!alive && tid == 0) {
    atomicExch(&g_chunk_split_timeout, 1);
    mbar_wait(&bar, phase ^ 1u, kWaitLimit);   // let an MMA still in flight finish
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tb, kPrepTmemCols);
  }
}

// ============================================================================
// State pass: one CTA per chain (sequence, head[, segment]), 512 threads.
// Thread (wq, j) with j = 32 (warp % 4) + lane owns TMEM lane j, i.e. row j of
// S^T, and the quarter wq = warp / 4 of every phase's columns.  Thread 0 issues
// the MMAs and the record copies (two records ahead).
// ============================================================================
constexpr int NT_S = 512;
constexpr int kStorePieces = (C * 16 + NT_S - 32 - 1) / (NT_S - 32);   // 16-byte pieces per thread

// hardware tanh approximation (one MUFU op; relative error about 2^-11)
__device__ __forceinline__ float tanh_fast(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// 8 bf16 outputs times sigmoid of the 8 bf16 gate values, rounded to bf16;
// o * sigmoid(z) = o/2 + (o/2) tanh(z/2)
__device__ __forceinline__ uint4 apply_gate(uint4 o, uint4 z) {
  uint32_t ow[4] = {o.x, o.y, o.z, o.w};
  const uint32_t zw[4] = {z.x, z.y, z.z, z.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float lo = 0.5f * bf_lo(ow[i]), hi = 0.5f * bf_hi(ow[i]);
    ow[i] = pack_bf16(fmaf(lo, tanh_fast(0.5f * bf_lo(zw[i])), lo),
                      fmaf(hi, tanh_fast(0.5f * bf_hi(zw[i])), hi));
  }
  return make_uint4(ow[0], ow[1], ow[2], ow[3]);
}

// A state in TMEM (this thread: columns [32 wq, 32 wq + 32) of row j of S^T, from
// taddr) -> dst.  A transition X (identity start) goes out as bf16 hi / lo images for
// pass C's hops (MN-major SW128 B operand, N = row of X, K = column; TMEM lane
// j holds column j of X); any other state as fp32 [dk][dv] rows.  Called once or
// twice per chain, out of line so the chunk loop keeps its registers.
__device__ __noinline__ void store_state_cols(float* dst, uint32_t taddr, bool ximg, int wq, int j,
                                              int dk, int dv) {
  uint32_t t[2][16];
  tmem_ld16(taddr, t[0]);
  tmem_ld16(taddr + 16, t[1]);
  tmem_wait_ld();
  if (ximg) {
    uint8_t* xb = reinterpret_cast<uint8_t*>(dst);
#pragma unroll
    for (int c8 = 0; c8 < 4; ++c8) {
      uint32_t hw[4], lw[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float x0 = __uint_as_float(t[c8 >> 1][(c8 & 1) * 8 + 2 * e]);
        const float x1 = __uint_as_float(t[c8 >> 1][(c8 & 1) * 8 + 2 * e + 1]);
        hw[e] = pack_bf16(x0, x1);
        lw[e] = pack_bf16(x0 - bf_lo(hw[e]), x1 - bf_hi(hw[e]));
      }
      const uint32_t o = chunk_mnmajor_sw128((uint32_t)(4 * wq + c8), (uint32_t)j, D);
      *reinterpret_cast<uint4*>(xb + o) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
      *reinterpret_cast<uint4*>(xb + 32768 + o) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
    }
  } else if (j < dv) {
#pragma unroll
    for (int e = 0; e < 32; ++e)
      if (32 * wq + e < dk) dst[(long long)(32 * wq + e) * dv + j] = __uint_as_float(t[e >> 4][e & 15]);
  }
}

// HALF: the split has half points (pass A keeps its half-way state, pass C's
// second-half chains form S_mid first); otherwise that code is compiled out.
template <bool HALF>
__global__ void __launch_bounds__(NT_S, 1)
kda_state_pass_kernel(const uint8_t* __restrict__ rec, const float* h0,
                      const int32_t* __restrict__ cu_seqlens, bf16* __restrict__ out, float* hT,
                      int T, int H, int dk, int dv, long long nslots, SegArgs sa,
                      const bf16* __restrict__ gate) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1024(smem_raw);
  __shared__ uint64_t full[2];
  __shared__ uint64_t mbar;
  __shared__ uint32_t tmem_base_sh;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = blockIdx.x, s = blockIdx.y;
  const int wq = warp >> 2, j = 32 * (warp & 3) + lane;
  const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;

  long long row0, t_beg, t_end;
  seq_range(cu_seqlens, s, T, row0, t_beg, t_end);
  const long long seq_t0 = t_beg;
  // what this chain computes: a token range, where its state starts, where it ends
  const long long hoff = ((long long)s * H + h) * dk * dv;
  const float* init = h0 ? h0 + hoff : nullptr;   // nullptr: zero state
  bool init_identity = false;
  float* fin = hT ? hT + hoff : nullptr;          // nullptr: final state not kept
  bool outputs = true, homog = false;
  int mid = 0;                                    // pass A: after `mid` chunks the state
  float* mid_dst = nullptr;                       // is also kept here
  int nhop = 0, hop_p = 0;                        // pass C: hops that form the start state
  const float* hop0 = nullptr;                    // (from hop0, see below)
  if (sa.pass != 0) {
    const int Ps = seg_count(t_end - t_beg, sa.G);
    const int z = blockIdx.z;
    const long long seg_tok = (long long)sa.G * C;
    auto slot_off = [&](int p) -> long long {
      const int sl = seg_slot_base(cu_seqlens, s, T, sa.G) + p;
      return sl < sa.slots ? ((long long)sl * H + h) * D * D : -1;
    };
    if (sa.pass == 1) {
      const bool xtype = z >= sa.P;
      const int p = xtype ? z - sa.P : z;
      if (Ps <= 1) {
        if (z != 0) return;                       // whole sequence in this one chain
      } else if (!xtype) {
        if (p > Ps - 2) return;
        const long long o = slot_off(p);
        if (o < 0) return;
        if (p > 0) {
          init = nullptr; outputs = false;
          if (HALF) { mid = sa.half; mid_dst = sa.sbuf_h + o; }
        }
        fin = sa.sbuf + o;
        t_beg += p * seg_tok;
        t_end = min(t_end, t_beg + seg_tok);
      } else {
        if (p < 1 || p > Ps - 2) return;
        const long long o = slot_off(p);
        if (o < 0) return;
        init = nullptr; init_identity = true; outputs = false; homog = true;
        fin = sa.xbuf + o;
        if (HALF) { mid = sa.half; mid_dst = sa.xbuf_h + o; }
        t_beg += p * seg_tok;
        t_end = min(t_end, t_beg + seg_tok);
      }
    } else {
      // z = p - 1 (one chain per segment), or 2 (p - 1) + q with half points: q = 0
      // runs the segment's first Gh chunks, q = 1 the rest from S_mid,p.  The chain
      // forms its own start state from pass A's results, hop by hop:
      //   S_start,1 = S_end,0 (= Sloc_0),  S_start,k+1 = X_k S_start,k + Sloc_k,
      //   and for q = 1  S_mid,p = X_half,p S_start,p + Sloc_half,p.
      const int p = (HALF ? z / 2 : z) + 1, q = HALF ? z % 2 : 0;
      if (Ps <= 1 || p > Ps - 1) return;
      const bool split = HALF && p <= Ps - 2;
      if (q == 1 && !split) return;
      if (slot_off(q == 1 ? p : p - 1) < 0) return;     // slots beyond the planned scratch
      nhop = p - 1 + q;
      hop0 = sa.sbuf + slot_off(0);
      init = nhop == 0 ? hop0 : nullptr;
      hop_p = p;
      if (p != Ps - 1) fin = nullptr;
      t_beg += p * seg_tok;
      const long long seg_end = min(t_end, t_beg + seg_tok);
      if (split) {
        const long long half_tok = (long long)sa.half * C;
        if (q == 0) t_end = min(seg_end, t_beg + half_tok);
        else { t_beg += half_tok; t_end = seg_end; }
      } else {
        t_end = seg_end;
      }
    }
  }
  const int nch = (int)chunk_count(t_end - t_beg);
  const long long cg0 = seq_chunk_base(cu_seqlens, s, T) + (t_beg - seq_t0) / C;
  const uint8_t* rec_h = rec + (size_t)h * (size_t)nslots * REC_BYTES;
  auto rec_ptr = [&](int i) { return rec_h + (size_t)(cg0 + i) * REC_BYTES; };

  if (warp == 0) {
    tmem_alloc(&tmem_base_sh, kStateTmemCols);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(&full[0], 1);
    mbar_init(&full[1], 1);
    mbar_init(&mbar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  // Hop h (pass C): X images and Sloc of the hop.  Loads go through the two record
  // buffers in one sequence -- the hops' X images first, then the records -- load li
  // into buffer li & 1 on barrier full[li & 1], phase (li >> 1) & 1.
  const long long seq_slot = seg_slot_base(cu_seqlens, s, T, sa.G);
  auto hop_off = [&](int hh) -> long long {
    return ((seq_slot + (hh < hop_p - 1 ? hh + 1 : hop_p)) * H + h) * D * D;
  };
  auto hop_x = [&](int hh) -> const uint8_t* {
    return reinterpret_cast<const uint8_t*>((hh < hop_p - 1 ? sa.xbuf : sa.xbuf_h) + hop_off(hh));
  };
  auto hop_l = [&](int hh) -> const float* {
    return (hh < hop_p - 1 ? sa.sbuf : sa.sbuf_h) + hop_off(hh);
  };
  const int nload = nhop + nch;
  auto issue_load = [&](int li) {                  // thread 0
    const uint32_t bytes = li < nhop ? 65536u : REC_BYTES;
    mbar_arrive_expect_tx(&full[li & 1], bytes);
    bulk_g2s(sm + (li & 1) * S_BUF, li < nhop ? hop_x(li) : rec_ptr(li - nhop), bytes,
             &full[li & 1]);
  };
  int issued = min(nload, 2);                      // loads requested (thread 0)
  int waited = 0;                                  // loads whose arrival thread 0 has seen
  // Launched right behind the kernel before it (programmatic stream serialization):
  // everything it reads from that kernel (prep's records, pass A's states and
  // transitions) is read after the wait.
  if (tid == 0) {
    grid_dep_wait();
    for (int li = 0; li < issued; ++li) issue_load(li);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tb = tmem_base_sh;
  const uint32_t tl = tb + lane_base;

  if (sa.pass == 2) grid_dep_wait();
  // ---- initial state: columns [32 wq, 32 wq + 32) of row j of S^T, and its bf16 copy
  if (nhop == 0) {
    const int c = 32 * wq;
    uint32_t f0[16], f1[16], pk[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      float x0 = init && c + e < dk && j < dv ? init[(long long)(c + e) * dv + j] : 0.f;
      float x1 = init && c + 16 + e < dk && j < dv ? init[(long long)(c + 16 + e) * dv + j] : 0.f;
      if (init_identity) { x0 = (c + e == j) ? 1.f : 0.f; x1 = (c + 16 + e == j) ? 1.f : 0.f; }
      f0[e] = __float_as_uint(x0);
      f1[e] = __float_as_uint(x1);
    }
    tmem_st16(tl + ST_S + c, f0);
    tmem_st16(tl + ST_S + c + 16, f1);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      pk[e] = pack_bf16(__uint_as_float(f0[2 * e]), __uint_as_float(f0[2 * e + 1]));
      pk[8 + e] = pack_bf16(__uint_as_float(f1[2 * e]), __uint_as_float(f1[2 * e + 1]));
    }
    tmem_st16(tl + ST_SB + c / 2, pk);
    tmem_wait_st();
  }
  bool good = true;
  uint32_t mphase = 0;
  // ---- pass C hops: S^T <- Sloc^T + S^T X^T (three bf16 products: hi hi, hi lo, lo hi;
  // fp32 accumulation onto Sloc^T in TMEM); X is the B operand (N = row of X, K =
  // column, MN-major images), S^T's hi / lo parts the A operands
#pragma unroll 1
  for (int hh = 0; hh < nhop && good; ++hh) {
    const float* lp = hop_l(hh);
#pragma unroll 1
    for (int hf = 0; hf < 2; ++hf) {                 // 16 of this thread's 32 columns at a time
      const int c = 32 * wq + 16 * hf;
      float cur[16];
      if (hh == 0) {
#pragma unroll
        for (int e = 0; e < 16; ++e)
          cur[e] = c + e < dk && j < dv ? hop0[(long long)(c + e) * dv + j] : 0.f;
      } else {
        uint32_t t[16];
        tmem_ld16(tl + ST_S + c, t);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 16; ++e) cur[e] = __uint_as_float(t[e]);
      }
      uint32_t hi[8], lo[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        hi[e] = pack_bf16(cur[2 * e], cur[2 * e + 1]);
        lo[e] = pack_bf16(cur[2 * e] - bf_lo(hi[e]), cur[2 * e + 1] - bf_hi(hi[e]));
      }
      tmem_st8(tl + ST_SB + c / 2, hi);
      tmem_st8(tl + ST_LO + c / 2, lo);
      uint32_t f[16];
#pragma unroll
      for (int e = 0; e < 16; ++e)
        f[e] = __float_as_uint(c + e < dk && j < dv ? lp[(long long)(c + e) * dv + j] : 0.f);
      tmem_st16(tl + ST_S + c, f);
      tmem_wait_st();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid == 0) {
      good = mbar_wait(&full[hh & 1], (hh >> 1) & 1, kWaitLimit);
      if (good) {
        waited = hh + 1;
        tc_fence_after();
        const uint32_t xh = smem_u32(sm + (hh & 1) * S_BUF), xl = xh + 32768u;
        const uint32_t id = idesc_bf16(128, 128, false, true);
        const uint64_t bh0 = desc_mnmajor_sw128(xh, D, 0), bl0 = desc_mnmajor_sw128(xl, D, 0);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {   // K step kk: 2048 bytes further
          const uint64_t bh = bh0 + (uint64_t)(kk * 128), bl = bl0 + (uint64_t)(kk * 128);
          mma_ts(tb + ST_S, tb + ST_SB + kk * 8, bh, id, 1);
          mma_ts(tb + ST_S, tb + ST_SB + kk * 8, bl, id, 1);
          mma_ts(tb + ST_S, tb + ST_LO + kk * 8, bh, id, 1);
        }
        mma_commit(&mbar);
      }
    }
    __syncwarp();
    if (__syncthreads_or(!good)) { good = false; break; }
    good = warp != 0 || mbar_wait(&mbar, mphase, kWaitLimit);
    mphase ^= 1u;
    if (__syncthreads_or(!good)) { good = false; break; }
    tc_fence_after();
    // this hop's buffer is consumed: the next load into it
    if (tid == 0 && issued < nload) {
      fence_async_smem();
      issue_load(issued);
      ++issued;
    }
  }
  if (nhop > 0 && good) {               // the bf16 copy of the start state for the first product
    uint32_t t[2][16], pk[16];
    tmem_ld16(tl + ST_S + 32 * wq, t[0]);
    tmem_ld16(tl + ST_S + 32 * wq + 16, t[1]);
    tmem_wait_ld();
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      pk[e] = pack_bf16(__uint_as_float(t[0][2 * e]), __uint_as_float(t[0][2 * e + 1]));
      pk[8 + e] = pack_bf16(__uint_as_float(t[1][2 * e]), __uint_as_float(t[1][2 * e + 1]));
    }
    tmem_st16(tl + ST_SB + 16 * wq, pk);
    tmem_wait_st();
  }
  if (good && nch > 0 && warp == 0) {
    good = mbar_wait(&full[nhop & 1], (nhop >> 1) & 1, kWaitLimit);
    if (good) waited = nhop + 1;
  }
  tc_fence_before();
  bool alive = __syncthreads_or(!good) == 0;
  tc_fence_after();

#pragma unroll 1
  for (int i = 0; i < nch && alive; ++i) {
    const int buf = (nhop + i) & 1;               // load nhop + i (see above)
    uint8_t* rb = sm + buf * S_BUF;
    const long long t0 = t_beg + (long long)i * C;
    const int L = (int)min((long long)C, t_end - t0);
    // the output gate's tile of this chunk: each thread fetches the pieces it stores
    if (gate && outputs && warp > 0) {
#pragma unroll
      for (int it = 0; it < kStorePieces; ++it) {
        const int idx = (tid - 32) + it * (NT_S - 32);
        const int r = idx >> 4, ch = idx & 15;
        if (idx < C * 16 && r < L && ch * 8 < dv)
          cp_async16(sm + S_GATE + r * 256 + ch * 16,
                     gate + ((row0 + t0 + r) * H + h) * dv + ch * 8, 16u);
      }
      cp_async_commit();
    }

    // ---- [O^T | P] = S^T [Qbar^T | W^T]^T   (P only when no outputs are kept)
    // The issue loop is kept to the MMA instructions alone: the descriptor of K step
    // kk is the first one plus kk * 2048 bytes in its address field.
    if (tid == 0) {
      tc_fence_after();
      const uint64_t b0 = desc_mnmajor_sw128(smem_u32(rb + REC_QW) + (outputs ? 0u : 16384u), D, 0);
      const uint32_t dst = tb + (outputs ? ST_O : ST_P);
      const uint32_t id = outputs ? idesc_bf16(128, 128, false, true) : idesc_bf16(128, 64, false, true);
      const int nk = dk / 16;                  // channels < dk
      mma_ts(dst, tb + ST_SB, b0, id, 0);
#pragma unroll
      for (int kk = 1; kk < D / 16; ++kk)
        if (kk < nk) mma_ts(dst, tb + ST_SB + kk * 8, b0 + (uint64_t)(kk * 128), id, 1);
      mma_commit(&mbar);
    }
    __syncwarp();
    // meanwhile S^T <- S^T Diag(exp(G_last)), columns [32 wq, 32 wq + 32)
    {
      const float* dec = reinterpret_cast<const float*>(rb + REC_DECAY) + 32 * wq;
      uint32_t t[2][16];
      tmem_ld16(tl + ST_S + 32 * wq, t[0]);
      tmem_ld16(tl + ST_S + 32 * wq + 16, t[1]);
      tmem_wait_ld();
#pragma unroll
      for (int q2 = 0; q2 < 2; ++q2) {
#pragma unroll
        for (int e = 0; e < 16; ++e)
          t[q2][e] = __float_as_uint(__uint_as_float(t[q2][e]) * dec[16 * q2 + e]);
        tmem_st16(tl + ST_S + 32 * wq + 16 * q2, t[q2]);
      }
      tmem_wait_st();
    }
    // warp 0 (whose thread 0 issued the MMAs) polls; the other warps wait in the CTA
    // barrier, so no spinning warp takes issue slots from the MMA issue
    tc_fence_before();
    good = warp != 0 || mbar_wait(&mbar, mphase, kWaitLimit);
    mphase ^= 1u;
    if (__syncthreads_or(!good)) { alive = false; break; }
    tc_fence_after();

    // ---- Delta^T = U^T - P for tokens [16 wq, 16 wq + 16) -> f16 TMEM
    {
      uint32_t tp[16];
      tmem_ld16(tl + ST_P + 16 * wq, tp);
      uint32_t uw[8];                  // U^T row j, tokens [16 wq, 16 wq + 16), f16 pairs
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const uint4 v4 = homog ? make_uint4(0u, 0u, 0u, 0u)
                               : *reinterpret_cast<const uint4*>(
                                     rb + REC_U + j * 128 + ((((uint32_t)(2 * wq + c)) ^ (j & 7u)) << 4));
        uw[4 * c] = v4.x; uw[4 * c + 1] = v4.y; uw[4 * c + 2] = v4.z; uw[4 * c + 3] = v4.w;
      }
      tmem_wait_ld();
      uint32_t dw[8];
#pragma unroll
      for (int e = 0; e < 8; ++e)
        dw[e] = pack_f16(h_lo(uw[e]) - __uint_as_float(tp[2 * e]),
                         h_hi(uw[e]) - __uint_as_float(tp[2 * e + 1]));
      tmem_st8(tl + ST_D + 8 * wq, dw);
      tmem_wait_st();
    }
    tc_fence_before();
    __syncthreads();

    // ---- [S^T | O^T] += Delta^T [Kend^T ; Aqk]^T
    if (tid == 0) {
      tc_fence_after();
      const int n = outputs ? D + C : D;
      const uint32_t id = idesc_f16(128, n, false, false);   // f16 A (Delta^T) and B
      // K step kk: 32 bytes further along the 128-byte rows
      const uint64_t b0 = desc_kmajor_sw128(smem_u32(rb + REC_KA), n, 0);
#pragma unroll
      for (int kk = 0; kk < C / 16; ++kk)
        mma_ts(tb + ST_S, tb + ST_D + kk * 8, b0 + (uint64_t)(kk * 2), id, 1);
      mma_commit(&mbar);
    }
    __syncwarp();
    good = warp != 0 || mbar_wait(&mbar, mphase, kWaitLimit);
    mphase ^= 1u;
    if (__syncthreads_or(!good)) { alive = false; break; }
    tc_fence_after();

    // the record in this buffer is consumed: fetch record i + 2 into it
    if (i + 2 < nch) {
      if (tid == 0) {
        fence_async_smem();
        mbar_arrive_expect_tx(&full[buf], REC_BYTES);
        bulk_g2s(rb, rec_ptr(i + 2), REC_BYTES, &full[buf]);
      }
      ++issued;
    }

    // ---- bf16 copy of the new state (columns [32 wq, +32)); O^T (tokens [16 wq, +16))
    {
      bf16* otile = reinterpret_cast<bf16*>(sm + S_OUT);
      uint32_t t[2][16], to[16];
      tmem_ld16(tl + ST_S + 32 * wq, t[0]);
      tmem_ld16(tl + ST_S + 32 * wq + 16, t[1]);
      if (outputs) tmem_ld16(tl + ST_O + 16 * wq, to);
      tmem_wait_ld();
      uint32_t pk[16];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        pk[e] = pack_bf16(__uint_as_float(t[0][2 * e]), __uint_as_float(t[0][2 * e + 1]));
        pk[8 + e] = pack_bf16(__uint_as_float(t[1][2 * e]), __uint_as_float(t[1][2 * e + 1]));
      }
      tmem_st16(tl + ST_SB + 16 * wq, pk);
      if (outputs) {
#pragma unroll
        for (int e = 0; e < 16; ++e)
          otile[(16 * wq + e) * D + j] = __float2bfloat16_rn(__uint_as_float(to[e]));
      }
      tmem_wait_st();
    }
    tc_fence_before();
    good = true;
    if (i + 1 < nch && warp == 0) {
      const int li = nhop + i + 1;
      good = mbar_wait(&full[li & 1], (li >> 1) & 1, kWaitLimit);
      if (good) waited = li + 1;
    }
    if (__syncthreads_or(!good)) { alive = false; break; }
    tc_fence_after();
    if (HALF && i + 1 == mid)           // the state after the first `mid` chunks (once)
      store_state_cols(mid_dst, tl + ST_S + 32 * wq, init_identity, wq, j, dk, dv);
    // coalesced 16-byte stores of the tile (overlap the next MMA)
    // (warps 1 .. 15: thread 0 is free to issue the next chunk's MMAs)
    if (outputs && warp > 0) {
      if (gate) cp_async_wait_all();
#pragma unroll
      for (int it = 0; it < kStorePieces; ++it) {
        const int idx = (tid - 32) + it * (NT_S - 32);
        const int r = idx >> 4, ch = idx & 15;
        if (idx < C * 16 && r < L && ch * 8 < dv) {
          uint4 val = *reinterpret_cast<const uint4*>(sm + S_OUT + r * 256 + ch * 16);
          if (gate)
            val = apply_gate(val, *reinterpret_cast<const uint4*>(sm + S_GATE + r * 256 + ch * 16));
          *reinterpret_cast<uint4*>(out + ((row0 + t0 + r) * H + h) * dv + ch * 8) = val;
        }
      }
    }
  }

  if (gate) cp_async_wait_all();          // no gate copy outlives the loop (early exit)

  // ---- final state
  if (alive && fin) {
    if (HALF) {
      store_state_cols(fin, tl + ST_S + 32 * wq, init_identity, wq, j, dk, dv);
    } else {
      uint32_t t[2][16];
      tmem_ld16(tl + ST_S + 32 * wq, t[0]);
      tmem_ld16(tl + ST_S + 32 * wq + 16, t[1]);
      tmem_wait_ld();
      if (init_identity) {
        // a transition X_p: bf16 hi / lo images for pass C's hops (MN-major SW128
        // B operand, N = row of X, K = column; TMEM lane j holds column j of X)
        uint8_t* xb = reinterpret_cast<uint8_t*>(fin);
#pragma unroll
        for (int c8 = 0; c8 < 4; ++c8) {
          uint32_t hw[4], lw[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float x0 = __uint_as_float(t[c8 >> 1][(c8 & 1) * 8 + 2 * e]);
            const float x1 = __uint_as_float(t[c8 >> 1][(c8 & 1) * 8 + 2 * e + 1]);
            hw[e] = pack_bf16(x0, x1);
            lw[e] = pack_bf16(x0 - bf_lo(hw[e]), x1 - bf_hi(hw[e]));
          }
          const uint32_t o = chunk_mnmajor_sw128((uint32_t)(4 * wq + c8), (uint32_t)j, D);
          *reinterpret_cast<uint4*>(xb + o) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
          *reinterpret_cast<uint4*>(xb + 32768 + o) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
        }
      } else if (j < dv) {
#pragma unroll
        for (int e = 0; e < 32; ++e)
          if (32 * wq + e < dk) fin[(long long)(32 * wq + e) * dv + j] = __uint_as_float(t[e >> 4][e & 15]);
      }
    }
  }
  if (!alive && tid == 0) {
    atomicExch(&g_chunk_split_timeout, 1);
    // let the MMA and the copies still in flight finish before the CTA exits
    mbar_wait(&mbar, mphase ^ 1u, kWaitLimit);
    for (int r = waited; r < issued; ++r) mbar_wait(&full[r & 1], (r >> 1) & 1, kWaitLimit);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tb, kStateTmemCols);
  }
}

// Dynamic shared memory of the kernels, set once per device.
bool set_attrs() {
  return once_per_device(kOnceSplit, []() {
    return cudaFuncSetAttribute(kda_chunk_prep_kernel<false, false>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, PREP_SMEM) == cudaSuccess &&
           cudaFuncSetAttribute(kda_chunk_prep_kernel<false, true>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, PREP_SMEM) == cudaSuccess &&
           cudaFuncSetAttribute(kda_chunk_prep_kernel<true, false>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, PREP_SMEM) == cudaSuccess &&
           cudaFuncSetAttribute(kda_chunk_prep_kernel<false, false, true>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, PREP_SMEM) == cudaSuccess &&
           cudaFuncSetAttribute(kda_chunk_prep_kernel<false, true, true>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, PREP_SMEM) == cudaSuccess &&
           cudaFuncSetAttribute(kda_state_pass_kernel<false>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, STATE_SMEM) == cudaSuccess &&
           cudaFuncSetAttribute(kda_state_pass_kernel<true>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, STATE_SMEM) == cudaSuccess;
  });
}

// Chunks per segment (G = 0: no split) and the half point of pass C (0: none).
// Cost model in units of one state-pass chunk step: pass A runs NH*(2P-3)
// chains, each G chunks long, in waves of one chain per SM; pass C runs NH*(P-1)
// chains of G chunks, or with half points NH*(2(P-2)+1) chains of at most
// max(Gh, last segment) chunks; chaining the segments' states (pass C's hops, about
// one chunk step each, on the deepest chain) is charged kCombine steps per segment
// and a second-half chain's extra hop (to S_mid) kMid steps.
constexpr double kCombine = 2.5;
constexpr double kMid = 1.0;
struct SplitPlan {
  int G, half;
};
SplitPlan plan_split(int B, int T, int H, bool varlen, int sms) {
  const long long NH = (long long)B * H;
  const long long nch = ((long long)T + C - 1) / C;
  if (NH >= sms || nch < 8) return {0, 0};
  if (varlen) return {nch >= 2 * 16 ? 16 : 0, 0};
  const long long w1 = (NH + sms - 1) / sms;
  double best = (double)(nch * w1);
  SplitPlan plan{0, 0};
  for (long long G = 2; G < nch; ++G) {
    const long long Pe = (nch + G - 1) / G;
    if (Pe < 2 || Pe > 64) continue;
    const long long wA = (NH * (2 * Pe - 3) + sms - 1) / sms;
    const long long wC = (NH * (Pe - 1) + sms - 1) / sms;
    const double cost = (double)G * (double)(wA + wC) + kCombine * (double)(Pe - 2) + 2.0;
    if (cost < best) { best = cost; plan = {(int)G, 0}; }
    if (Pe >= 3) {
      const long long Gh = (G + 1) / 2, last = nch - (Pe - 1) * G;
      const long long wCh = (NH * (2 * (Pe - 2) + 1) + sms - 1) / sms;
      const double costh = (double)G * (double)wA + (double)std::max(Gh, last) * (double)wCh +
                           kCombine * (double)(Pe - 2) + kMid + 2.0;
      if (costh < best) { best = costh; plan = {(int)G, (int)Gh}; }
    }
  }
  return plan;
}

}  // namespace

bool chunk_split_supported(int dk, int dv, int in_dtype) {
  return in_dtype == KDA_BF16 && (dk == 64 || dk == D) && (dv == 64 || dv == D);
}

void chunk_split_plan(int B, int T, int H, bool varlen, int sms, int* G, int* half) {
  const SplitPlan p = plan_split(B, T, H, varlen, sms);
  *G = p.G;
  *half = p.half;
}

namespace {
// TMA maps of the prep kernel's tiles (rows addressed by int32 coordinates); 0 when
// the tiles are loaded without TMA (the maps are then zeroed and not read).
int prep_maps(PrepMaps* maps, const bf16* qb, const bf16* kb, const bf16* vb, const float* g,
              long long rows, int H, int dk, int dv, int gsh) {
  int tma = 0;
  if (rows > 0 && rows < (1LL << 31) - 2 * C) {
    const uint64_t hh = (uint64_t)H, nr = (uint64_t)rows;
    tma = make_tile_map_3d(&maps->q, false, qb, dk, hh, nr, dk * 2ull, hh * dk * 2, dk, C,
                           false) &&
          make_tile_map_3d(&maps->k, false, kb, dk, hh, nr, dk * 2ull, hh * dk * 2, dk, C,
                           false) &&
          make_tile_map_3d(&maps->v, false, vb, dv, hh, nr, dv * 2ull, hh * dv * 2, 64, C,
                           true) &&
          (gsh != 0 || make_tile_map_3d(&maps->g, true, g, dk, hh, nr, dk * 4ull, hh * dk * 4,
                                        dk, C, false));
    if (gsh != 0) maps->g = maps->q;             // not read
  }
  if (!tma) memset(maps, 0, sizeof(*maps));
  return tma;
}

// Chunk records (nslots per head) and, when sequences are split, the segment
// states: the one layout both the size query and the launcher use.
struct SplitScratch {
  long long nslots;
  size_t rec_bytes, seg_bytes;
  SplitPlan plan;
  int P;
  long long slots;
};
SplitScratch split_scratch(int B, int T, int H, bool varlen, int sms) {
  SplitScratch r{};
  r.nslots = chunk_slots(B, T, varlen);
  r.rec_bytes = (size_t)r.nslots * H * REC_BYTES;
  r.plan = plan_split(B, T, H, varlen, sms);
  const long long nch_all = ((long long)T + C - 1) / C;
  if (r.plan.G > 0 && (nch_all + r.plan.G - 1) / r.plan.G >= 2) {
    r.P = (int)((nch_all + r.plan.G - 1) / r.plan.G);
    r.slots = varlen ? (long long)r.P + B : (long long)B * r.P;
    r.seg_bytes = (size_t)(r.plan.half > 0 ? 4 : 2) * r.slots * H * D * D * sizeof(float);
  }
  return r;
}

}  // namespace

size_t chunk_split_scratch_bytes(int B, int T, int H, bool varlen, int sms) {
  const SplitScratch r = split_scratch(B, T, H, varlen, sms);
  return r.rec_bytes + r.seg_bytes;
}

cudaError_t launch_chunk_split(const void* q, const void* k, const void* v, const float* g,
                               const float* beta, const float* h0, const int32_t* cu_seqlens,
                               void* out, float* hT, int B, int T, int H, int dk, int dv,
                               int gsh, cudaStream_t stream, const InputFusion* fz,
                               const Workspace* ws) {
  int sms = 148;
  cudaMemPool_t pool = nullptr;
  if (!device_ctx(&sms, ws ? nullptr : &pool) || !set_attrs()) return cudaErrorInvalidDevice;
  if (!ws && !pool) return cudaErrorMemoryAllocation;
  const bf16* qb = static_cast<const bf16*>(q);
  const bf16* kb = static_cast<const bf16*>(k);
  const bf16* vb = static_cast<const bf16*>(v);
  bf16* ob = static_cast<bf16*>(out);
  const bf16* gt = fz ? static_cast<const bf16*>(fz->gate) : nullptr;
  const bool varlen = cu_seqlens != nullptr;

  const SplitScratch sc = split_scratch(B, T, H, varlen, sms);
  const long long nslots = sc.nslots;
  const size_t rec_bytes = sc.rec_bytes, seg_bytes = sc.seg_bytes;
  const SplitPlan plan = sc.plan;
  const int G = plan.G, P = sc.P;
  const long long slots = sc.slots;
  void* scratch = nullptr;
  bool pooled = false;
  if (rec_bytes + seg_bytes > 0) {
    if (ws) {
      if (!ws->ptr || ws->bytes < rec_bytes + seg_bytes) return cudaErrorInvalidValue;
      scratch = ws->ptr;
    } else {
      const cudaError_t e = cudaMallocFromPoolAsync(&scratch, rec_bytes + seg_bytes, pool, stream);
      if (e != cudaSuccess) return e;
      pooled = true;
    }
  }
  uint8_t* rec = static_cast<uint8_t*>(scratch);
  float* segbuf = reinterpret_cast<float*>(rec + rec_bytes);

  cudaError_t e = cudaSuccess;
  if (nslots > 0) {
    PrepMaps maps;
    const long long rows = varlen ? (long long)T : (long long)B * T;
    const bool conv = fz && fz->conv_q;
    const int tma = conv ? 0 : prep_maps(&maps, qb, kb, vb, g, rows, H, dk, dv, gsh);
    if (conv) {
      KDA_TIMED(KDA_KERNEL_PREP, stream,
                kda_chunk_prep_kernel<true, false><<<dim3((unsigned)nslots, H), NT, PREP_SMEM, stream>>>(
                    qb, kb, vb, g, beta, cu_seqlens, rec, B, T, H, dk, dv, gsh, nslots,
                    fz->conv_q, fz->conv_k, fz->W, maps, 0));
    } else {
      auto prep = gsh != 0 ? kda_chunk_prep_kernel<false, true> : kda_chunk_prep_kernel<false, false>;
      KDA_TIMED(KDA_KERNEL_PREP, stream,
                prep<<<dim3((unsigned)nslots, H), NT, PREP_SMEM, stream>>>(
                    qb, kb, vb, g, beta, cu_seqlens, rec, B, T, H, dk, dv, gsh, nslots, nullptr,
                    nullptr, 0, maps, tma));
    }
    note_launches(1);
  }
  if (P == 0) {
    SegArgs sa{0, 1, 0, 0, nullptr, nullptr};
    KDA_TIMED(KDA_KERNEL_STATE, stream,
              e = launch_after(kda_state_pass_kernel<false>, dim3(H, B, 1), dim3(NT_S), STATE_SMEM,
                               stream, rec, h0, cu_seqlens, ob, hT, T, H, dk, dv, nslots, sa, gt));
    note_launches(1);
  } else {
    const size_t per = (size_t)slots * H * D * D;
    SegArgs sa{G, P, 1, (int)slots, segbuf, segbuf + per};
    if (plan.half > 0) {
      sa.half = plan.half;
      sa.sbuf_h = segbuf + 2 * per;
      sa.xbuf_h = segbuf + 3 * per;
    }
    auto state_pass = [&](dim3 grid) {
      return launch_after(sa.half > 0 ? kda_state_pass_kernel<true> : kda_state_pass_kernel<false>,
                          grid, dim3(NT_S), STATE_SMEM, stream, rec, h0, cu_seqlens, ob, hT, T, H, dk,
                          dv, nslots, sa, gt);
    };
    // pass A, then pass C, whose chains chain the segments' states themselves
    cudaError_t es = cudaSuccess;
    KDA_TIMED(KDA_KERNEL_STATE, stream, es = state_pass(dim3(H, B, 2 * P)));
    sa.pass = 2;
    const unsigned zc = (unsigned)(sa.half > 0 ? 2 * (P - 1) : P - 1);
    const cudaError_t es2 = es;
    KDA_TIMED(KDA_KERNEL_STATE, stream, es = state_pass(dim3(H, B, zc)));
    note_launches(2);
    if (es2 != cudaSuccess) e = es2;
    if (es != cudaSuccess) e = es;
  }
  const cudaError_t el = cudaGetLastError();
  if (e == cudaSuccess) e = el;
  if (pooled) cudaFreeAsync(scratch, stream);
  return e;
}

// The prep kernel for the backward (dk = dv = 128): nslots records of
// rec::BYTES_BWD bytes per head at `rec`, numbered as the prefill numbers them.
cudaError_t launch_chunk_prep_bwd(const void* q, const void* k, const void* v, const float* g,
                                  const float* beta, const int32_t* cu_seqlens, uint8_t* rec,
                                  int B, int T, int H, int gsh, long long nslots,
                                  cudaStream_t stream) {
  if (!set_attrs()) return cudaErrorInvalidDevice;
  if (nslots == 0) return cudaSuccess;
  const bf16* qb = static_cast<const bf16*>(q);
  const bf16* kb = static_cast<const bf16*>(k);
  const bf16* vb = static_cast<const bf16*>(v);
  PrepMaps maps;
  const long long rows = cu_seqlens ? (long long)T : (long long)B * T;
  const int tma = prep_maps(&maps, qb, kb, vb, g, rows, H, D, D, gsh);
  auto prep = gsh != 0 ? kda_chunk_prep_kernel<false, true, true>
                       : kda_chunk_prep_kernel<false, false, true>;
  KDA_TIMED(KDA_KERNEL_BWD_PREP, stream,
            prep<<<dim3((unsigned)nslots, H), NT, PREP_SMEM, stream>>>(
                qb, kb, vb, g, beta, cu_seqlens, rec, B, T, H, D, D, gsh, nslots, nullptr,
                nullptr, 0, maps, tma));
  note_launches(1);
  return cudaGetLastError();
}

// Reads (and with reset clears) g_chunk_split_timeout; host side of kda_device_status.
cudaError_t take_split_timeout(int* flag, bool reset) {
  int v = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, g_chunk_split_timeout, sizeof(int));
  if (e == cudaSuccess && reset && v != 0) {
    const int zero = 0;
    e = cudaMemcpyToSymbol(g_chunk_split_timeout, &zero, sizeof(int));
  }
  *flag = v;
  return e;
}

}  // namespace kda
