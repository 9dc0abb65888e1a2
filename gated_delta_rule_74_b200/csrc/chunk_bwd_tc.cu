// KDA prefill backward in the chunked form on the tensor cores (bf16 q/k/v/dout,
// dk = dv = 128, fp32 g/beta/states/gradients).
//
// Chunked form (miniKimiK3 model card, "Kimi Delta Attention" bullet: KDA trains
// through a chunked parallel form).  Per chunk of 64 tokens with start state S and
// the chunk quantities of the forward (Gamma = cumsum g, Qbar, Kbar, Kend, A, Aqk,
// T = (I + diag(beta) A)^-1, W, U; see chunk_split.cu):
//     Delta = U - W S,  O = Qbar S + Aqk Delta,  S' = Diag(e^Gamma_last) S + Kend^T Delta.
// For L = sum(O * dO) + sum(S_final * dS_final), with dS the gradient of the state
// after the chunk, the chain rule through those lines (last first) gives
//     dDelta   = Aqk^T dO + Kend dS
//     dS_start = Diag(e^Gamma_last) dS + Qbar^T dO - W^T dDelta
//     dQbar = dO S^T,  dAqk = tril(dO Delta^T),  dKend = Delta dS^T,  dW = -dDelta S^T
//     [dVb | dKb] = T^T [dDelta | dW]           (Vb = diag(beta) V, Kb = diag(beta) Kbar)
//     dT = dDelta Vb^T + dW Kb^T,  dM = -T^T dT T^T (strictly lower),  dA = diag(beta) dM
// and from there to q, k, v, beta and Gamma through their definitions; dg is the
// reverse cumulative sum of dGamma inside the chunk.
//
// Three launches after the prep kernel's backward form (per (chunk, head): the
// record images in bf16, T as a bf16 image too, and A in fp32; chunk_split.cu):
//   chains    the state and its gradient move across a sequence's chunks column
//             block by column block (every column of S, and of dS, evolves on its
//             own): per (column block, head, sequence) one CTA walks the chunks
//             forward, writing S at every chunk start and Delta, and one walks them
//             backward, writing dS after every chunk and dDelta; both in one grid.
//   gradients per (chunk, head), everything else, all chunks in parallel.
// The matrix products run on the tensor cores as warp-level tiles (m16n8k16, bf16
// operands, fp32 accumulation) read from 128-byte-swizzled shared-memory images.
// In the gradient kernel each warp owns one 16-token row block -- one of the
// chunk's decay blocks -- and 64 channels, so every product that lands on
// (token, channel) accumulates in that warp's registers.
//
// The decay-weighted Gram products (dA and dAqk against k and q with the pairwise
// factors exp(Gamma_rc - Gamma_ic)) are split through per-block reference points as
// in the prefill: row side against R^(a)_ic = k_ic e^{Gamma_16a,c - Gamma_ic}
// (i < 16(a+1)), column side against R'^(b)_rc = x_rc e^{Gamma_rc - Gamma_16b+15,c}
// (r >= 16b), so every factor outside the diagonal block is <= 1.  A channel whose
// decay inside a block exceeds kUnsafeDecay has that block's entries zeroed and its
// within-block pairs added exactly on the CUDA cores.
#include <cuda_bf16.h>

#include "chunk_record.cuh"
#include "decay_pairs.cuh"
#include "kda_common.cuh"
#include "segments.cuh"
#include "sm100.cuh"

namespace kda {

// Set when a bounded wait of the chunked backward gives up (diagnostic).
__device__ int g_bwd_tc_timeout = 0;

cudaError_t launch_chunk_prep_bwd(const void* q, const void* k, const void* v, const float* g,
                                  const float* beta, const int32_t* cu_seqlens, uint8_t* rec,
                                  int B, int T, int H, int gsh, long long nslots,
                                  cudaStream_t stream);

namespace {
using namespace sm100;
using bf16 = __nv_bfloat16;

constexpr int C = kChunk;
constexpr int D = kHead;
constexpr int NTC = 256;               // threads of the chain kernel
constexpr uint32_t kImgS = 32768;      // S / dS image per (chunk, head): [128 j][128 c] bf16
constexpr uint32_t kImgD = 16384;      // Delta / dDelta image: [64 t][128 j] bf16
constexpr uint32_t kWaitLimit = 1u << 22;

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// ------------------------------------------------------------ warp-level tiles
__device__ __forceinline__ void ldsm4(uint32_t a, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(a)
               : "memory");
}
__device__ __forceinline__ void ldsm4t(uint32_t a, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(a)
               : "memory");
}
__device__ __forceinline__ void ldsm2(uint32_t a, uint32_t (&r)[2]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];"
               : "=r"(r[0]), "=r"(r[1])
               : "r"(a)
               : "memory");
}
__device__ __forceinline__ void ldsm2t(uint32_t a, uint32_t (&r)[2]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0,%1}, [%2];"
               : "=r"(r[0]), "=r"(r[1])
               : "r"(a)
               : "memory");
}
__device__ __forceinline__ void stsm4(uint32_t a, const uint32_t (&r)[4]) {
  asm volatile("stmatrix.sync.aligned.m8n8.x4.shared.b16 [%0], {%1,%2,%3,%4};" ::"r"(a),
               "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3])
               : "memory");
}
__device__ __forceinline__ void stsm4t(uint32_t a, const uint32_t (&r)[4]) {
  asm volatile("stmatrix.sync.aligned.m8n8.x4.trans.shared.b16 [%0], {%1,%2,%3,%4};" ::"r"(a),
               "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3])
               : "memory");
}
__device__ __forceinline__ void stsm2(uint32_t a, const uint32_t (&r)[2]) {
  asm volatile("stmatrix.sync.aligned.m8n8.x2.shared.b16 [%0], {%1,%2};" ::"r"(a), "r"(r[0]),
               "r"(r[1])
               : "memory");
}
// d += a b (16 x 8 x 16, bf16 in, fp32 accumulate)
__device__ __forceinline__ void mma(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                    uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// byte offset of element (row, col) of an image with `rows` rows (chunk_record.cuh)
__device__ __forceinline__ uint32_t io(int row, int col, int rows) {
  return off_kmajor_sw128((uint32_t)row, (uint32_t)col, (uint32_t)rows);
}

// Fragment of the 16 x 16 block (rows m0.., columns k0..) of an operand A stored
// as an image [m][k] (a_mk) or [k][m] (a_km, transposed on load).
__device__ __forceinline__ void a_mk(uint32_t img, int rows, int m0, int k0, int lane,
                                     uint32_t (&a)[4]) {
  ldsm4(img + io(m0 + (lane & 15), k0 + ((lane >> 4) << 3), rows), a);
}
__device__ __forceinline__ void a_km(uint32_t img, int rows, int m0, int k0, int lane,
                                     uint32_t (&a)[4]) {
  ldsm4t(img + io(k0 + (lane & 7) + ((lane >> 4) << 3), m0 + (((lane >> 3) & 1) << 3), rows), a);
}
// Fragments of operand B for the k16 step k0 and two n8 tiles (n0.. in b[0..1],
// n0+8.. in b[2..3]), stored as an image [n][k] (b_nk) or [k][n] (b_kn); *1: one tile.
__device__ __forceinline__ void b_nk(uint32_t img, int rows, int n0, int k0, int lane,
                                     uint32_t (&b)[4]) {
  ldsm4(img + io(n0 + (lane & 7) + ((lane >> 4) << 3), k0 + (((lane >> 3) & 1) << 3), rows), b);
}
__device__ __forceinline__ void b_kn(uint32_t img, int rows, int n0, int k0, int lane,
                                     uint32_t (&b)[4]) {
  ldsm4t(img + io(k0 + (lane & 7) + (((lane >> 3) & 1) << 3), n0 + ((lane >> 4) << 3), rows), b);
}
__device__ __forceinline__ void b_nk1(uint32_t img, int rows, int n0, int k0, int lane,
                                      uint32_t (&b)[2]) {
  ldsm2(img + io(n0 + (lane & 7), k0 + (((lane >> 3) & 1) << 3), rows), b);
}
__device__ __forceinline__ void b_kn1(uint32_t img, int rows, int n0, int k0, int lane,
                                      uint32_t (&b)[2]) {
  ldsm2t(img + io(k0 + (lane & 7) + (((lane >> 3) & 1) << 3), n0, rows), b);
}
// bf16 image stores of an m16 x n16 accumulator pair (c0: columns n0.., c1: n0+8..)
// times s, as [m][n] (st_mn) or transposed as [n][m] (st_nm); st_mn1: one m16 x n8.
__device__ __forceinline__ void st_mn(uint32_t img, int rows, int m0, int n0, int lane,
                                      const float (&c0)[4], const float (&c1)[4], float s) {
  const uint32_t r[4] = {pack_bf16(c0[0] * s, c0[1] * s), pack_bf16(c0[2] * s, c0[3] * s),
                         pack_bf16(c1[0] * s, c1[1] * s), pack_bf16(c1[2] * s, c1[3] * s)};
  stsm4(img + io(m0 + (lane & 7) + (((lane >> 3) & 1) << 3), n0 + ((lane >> 4) << 3), rows), r);
}
__device__ __forceinline__ void st_nm(uint32_t img, int rows, int m0, int n0, int lane,
                                      const float (&c0)[4], const float (&c1)[4], float s) {
  const uint32_t r[4] = {pack_bf16(c0[0] * s, c0[1] * s), pack_bf16(c0[2] * s, c0[3] * s),
                         pack_bf16(c1[0] * s, c1[1] * s), pack_bf16(c1[2] * s, c1[3] * s)};
  stsm4t(img + io(n0 + (lane & 7) + ((lane >> 4) << 3), m0 + (((lane >> 3) & 1) << 3), rows), r);
}
__device__ __forceinline__ void st_mn1(uint32_t img, int rows, int m0, int n0, int lane,
                                       const float (&c)[4], float s) {
  const uint32_t r[2] = {pack_bf16(c[0] * s, c[1] * s), pack_bf16(c[2] * s, c[3] * s)};
  stsm2(img + io(m0 + (lane & 7) + (((lane >> 3) & 1) << 3), n0, rows), r);
}
__device__ __forceinline__ float bf_at(const uint8_t* p) {
  return __bfloat162float(*reinterpret_cast<const bf16*>(p));
}
__device__ __forceinline__ float2 bf2_at(const uint8_t* p) {
  const uint32_t w = *reinterpret_cast<const uint32_t*>(p);
  return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

// ============================================================================
// Chains: per (column block, head, sequence) one CTA of 8 warps walks the chunks forward
// (S at every chunk start, Delta) or backward (dS after every chunk, dDelta, dh0).
// Warp w keeps rows 16w .. 16w + 15 of the state (or of its gradient) for the
// block's columns as m16n8 accumulators: lane (g, qd) holds rows 16w + g (+8),
// columns 8 nt + 2 qd (+1).
// ============================================================================
template <int NB>
struct Chain {
  static constexpr int NJ = NB / 8;        // n8 tiles of the column block
  static constexpr int STG = 3;            // record stages in flight
  // forward stage: W^T (16 KB), Kend^T (16 KB), U^T rows of the block, exp(Gamma_last)
  static constexpr uint32_t F_W = 0, F_K = 16384, F_U = 32768, F_DEC = F_U + NB * 128,
                            F_STAGE = F_DEC + 512, F_BYTES = F_STAGE;
  static constexpr uint32_t F_S = STG * F_STAGE;        // S tile [NB j][128 c]
  static constexpr uint32_t F_DL = F_S + NB * 256;      // Delta tile [64 t][NB j] (64-column panel)
  static constexpr uint32_t F_SMEM = F_DL + 8192;
  // reverse stage: [Qbar^T | W^T] (32 KB), [Kend^T ; Aqk] (24 KB), exp(Gamma_last), dO tile
  static constexpr uint32_t R_QW = 0, R_KA = 32768, R_DEC = 57344, R_DO = 57856,
                            R_STAGE = R_DO + 8192, R_BYTES = R_DO;
  static constexpr uint32_t R_Y = STG * R_STAGE;        // dS tile [NB j][128 c]
  static constexpr uint32_t R_DD = R_Y + NB * 256;      // -dDelta tile [64 t][NB j]
  static constexpr uint32_t R_SMEM = R_DD + 8192;
  static constexpr uint32_t SMEM = (F_SMEM > R_SMEM ? F_SMEM : R_SMEM) + 1024;
  static_assert(F_STAGE % 128 == 0 && R_STAGE % 128 == 0, "tiles stay 128-byte aligned");
};

// Shared setup of one chain CTA: the sequence's chunk range and its slots.
struct ChainCtx {
  const uint8_t* rec;
  const bf16* dout;
  uint8_t* sm;
  uint32_t sb;
  uint64_t* full;
  size_t base, st_off;
  long long row0, t_beg, t_end;
  int nch, j0, h, H, tid, w, lane, g, qd;
};

// The state (or its gradient) of one CTA: warp w holds rows cr = 16 w .. cr + 15 and the
// block's NB / 8 n8 tiles of columns.  Returns the first chain step's state loaded from init.
template <int NB>
__device__ __forceinline__ void chain_load(const ChainCtx& x, const float* init,
                                           float (&X)[NB / 8][4]) {
#pragma unroll
  for (int nt = 0; nt < NB / 8; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int c = 16 * x.w + x.g + ((e >> 1) << 3), j = x.j0 + 8 * nt + 2 * x.qd + (e & 1);
      X[nt][e] = init ? init[x.st_off + (size_t)c * D + j] : 0.f;
    }
}

// The state tile as bf16 [j][c]; each warp then copies its own 16 channels of the tile's
// NB rows j out to rows j0.. of the chunk's image (no barrier needed).
template <int NB>
__device__ __forceinline__ void chain_put(const ChainCtx& x, const float (&X)[NB / 8][4],
                                          uint32_t tile_off, uint8_t* img) {
  const int cr = 16 * x.w;
#pragma unroll
  for (int p = 0; p < NB / 16; ++p)
    st_nm(x.sb + tile_off, NB, cr, 16 * p, x.lane, X[2 * p], X[2 * p + 1], 1.f);
  __syncwarp();
#pragma unroll
  for (int i = x.lane; i < 2 * NB; i += 32) {
    const int rr = i >> 1, ck = (cr >> 3) + (i & 1);          // row j, 16-byte chunk
    const uint32_t sw = (uint32_t)(((ck & 7) ^ (rr & 7)) << 4);
    *reinterpret_cast<uint4*>(img + (ck >> 3) * 16384 + (x.j0 + rr) * 128 + sw) =
        *reinterpret_cast<const uint4*>(x.sm + tile_off + (ck >> 3) * NB * 128 + rr * 128 + sw);
  }
}

// One K step (16 tokens) of A B added into the state X (set 0) or a partial sum Y:
// A a [c][t] image (the warp's 16 rows), B a [t][j] tile of the block's NB columns.
template <int NB>
__device__ __forceinline__ void chain_update(const ChainCtx& x, uint32_t a_img, uint32_t b_img,
                                             float (&X)[NB / 8][4], float (&Y)[NB / 8][4],
                                             int ks, bool into_y) {
  uint32_t a[4];
  a_mk(a_img, 128, 16 * x.w, 16 * ks, x.lane, a);
#pragma unroll
  for (int p = 0; p < NB / 16; ++p) {
    uint32_t b[4];
    b_kn(b_img, 64, 16 * p, 16 * ks, x.lane, b);
    float (&u0)[4] = into_y ? Y[2 * p] : X[2 * p];
    float (&u1)[4] = into_y ? Y[2 * p + 1] : X[2 * p + 1];
    mma(u0, a, b[0], b[1]);
    mma(u1, a, b[2], b[3]);
  }
}

// A bounded wait for a stage failed: raise the flag and let the copies in flight land.
template <int STG>
__device__ void chain_give_up(const ChainCtx& x, int n_first, int n_last, bool ascending) {
  if (x.tid == 0) {
    atomicExch(&g_bwd_tc_timeout, 1);
    for (int m = n_first; ascending ? m <= n_last : m >= n_last; m += ascending ? 1 : -1) {
      const uint32_t use = ascending ? (uint32_t)(m / STG) : (uint32_t)((x.nch - 1 - m) / STG);
      mbar_wait(&x.full[m % STG], use & 1u, kWaitLimit);
    }
  }
  cp_async_wait_all();
}

// Forward chain: S at every chunk start and Delta of every chunk.
template <int NB>
__device__ __forceinline__ void chain_forward(const ChainCtx& x, const float* h0, uint8_t* simg,
                                              uint8_t* dlimg) {
  using CF = Chain<NB>;
  constexpr int NJ = NB / 8, NH = NB / 16, STG = CF::STG;
  const int tb = x.w & 3, jh = x.w >> 2, g = x.g, qd = x.qd, lane = x.lane;
  float X[NJ][4];
  chain_load<NB>(x, h0, X);
  auto issue = [&](int n) {
    if (x.tid == NTC - 32 && n < x.nch) {
      const uint8_t* rc = x.rec + (x.base + n) * rec::BYTES_BWD;
      uint8_t* st = x.sm + (n % STG) * CF::F_STAGE;
      uint64_t* bar = &x.full[n % STG];
      fence_async_smem();
      mbar_arrive_expect_tx(bar, CF::F_BYTES);
      bulk_g2s(st + CF::F_W, rc + rec::QW + 16384, 16384, bar);
      bulk_g2s(st + CF::F_K, rc + rec::KA, 16384, bar);
      bulk_g2s(st + CF::F_U, rc + rec::U + x.j0 * 128, NB * 128, bar);
      bulk_g2s(st + CF::F_DEC, rc + rec::DECAY, 512, bar);
    }
  };
  const uint32_t uS = x.sb + CF::F_S, uDL = x.sb + CF::F_DL;
#pragma unroll 1
  for (int n = 0; n < STG - 1; ++n) issue(n);
#pragma unroll 1
  for (int n = 0; n < x.nch; ++n) {
    const uint32_t so = (uint32_t)(n % STG) * CF::F_STAGE;
    chain_put<NB>(x, X, CF::F_S, simg + (x.base + n) * kImgS);   // S at the start of chunk n
    const bool ok = mbar_wait(&x.full[n % STG], (uint32_t)(n / STG) & 1u, kWaitLimit);
    if (__syncthreads_or(!ok)) {
      chain_give_up<STG>(x, n, min(n + STG - 2, x.nch - 1), true);
      return;
    }
    // Delta = U - W S: token block tb, n8 tiles jh * NH .. (two accumulators each)
    float acc[NH][2][4] = {};
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      uint32_t a[4];
      a_km(x.sb + so + CF::F_W, 128, 16 * tb, 16 * ks, lane, a);       // W [t][c] from W^T
      if constexpr (NH == 2) {
        uint32_t b[4];
        b_nk(uS, NB, 16 * jh, 16 * ks, lane, b);                       // S [c][j] from [j][c]
        mma(acc[0][ks & 1], a, b[0], b[1]);
        mma(acc[1][ks & 1], a, b[2], b[3]);
      } else {
        uint32_t b[2];
        b_nk1(uS, NB, 8 * jh, 16 * ks, lane, b);
        mma(acc[0][ks & 1], a, b[0], b[1]);
      }
    }
    uint8_t* gD = dlimg + (x.base + n) * kImgD;
#pragma unroll
    for (int p = 0; p < NH; ++p) {
      const int n0 = 8 * (jh * NH + p), jl = n0 + 2 * qd;
      float dl[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int t = 16 * tb + g + ((e >> 1) << 3);
        dl[e] = bf_at(x.sm + so + CF::F_U + io(jl + (e & 1), t, NB)) - acc[p][0][e] - acc[p][1][e];
      }
      st_mn1(uDL, 64, 16 * tb, n0, lane, dl, 1.f);
#pragma unroll
      for (int hf = 0; hf < 2; ++hf)
        *reinterpret_cast<uint32_t*>(gD + io(16 * tb + g + 8 * hf, x.j0 + jl, 64)) =
            pack_bf16(dl[2 * hf], dl[2 * hf + 1]);
    }
    __syncthreads();
    // S <- Diag(exp(Gamma_last)) S + Kend^T Delta
    const float* dec = reinterpret_cast<const float*>(x.sm + so + CF::F_DEC);
    const float d0 = dec[16 * x.w + g], d1 = dec[16 * x.w + g + 8];
    float Y[NJ][4] = {};
#pragma unroll
    for (int nt = 0; nt < NJ; ++nt) {
      X[nt][0] *= d0; X[nt][1] *= d0; X[nt][2] *= d1; X[nt][3] *= d1;
    }
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) chain_update<NB>(x, x.sb + so + CF::F_K, uDL, X, Y, ks, ks & 1);
#pragma unroll
    for (int nt = 0; nt < NJ; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) X[nt][e] += Y[nt][e];
    issue(n + STG - 1);                 // into chunk n - 1's stage, read before this step's barrier
  }
}

// Reverse chain: dS after every chunk, dDelta of every chunk, and dh0.
template <int NB>
__device__ __forceinline__ void chain_reverse(const ChainCtx& x, const float* dhT, float* dh0,
                                              uint8_t* dsimg, uint8_t* ddimg, uint8_t* ddlo) {
  using CF = Chain<NB>;
  constexpr int NJ = NB / 8, NH = NB / 16, STG = CF::STG;
  const int tb = x.w & 3, jh = x.w >> 2, g = x.g, qd = x.qd, lane = x.lane;
  float X[NJ][4];
  chain_load<NB>(x, dhT, X);
  auto issue = [&](int n) {
    if (n >= 0) {
      const uint8_t* rc = x.rec + (x.base + n) * rec::BYTES_BWD;
      uint8_t* st = x.sm + (n % STG) * CF::R_STAGE;
      if (x.tid == NTC - 32) {
        uint64_t* bar = &x.full[n % STG];
        fence_async_smem();
        mbar_arrive_expect_tx(bar, CF::R_BYTES);
        bulk_g2s(st + CF::R_QW, rc + rec::QW, 32768, bar);
        bulk_g2s(st + CF::R_KA, rc + rec::KA, 24576, bar);
        bulk_g2s(st + CF::R_DEC, rc + rec::DECAY, 512, bar);
      }
      const long long t0 = x.t_beg + (long long)n * C;
      const int L = (int)min((long long)C, x.t_end - t0);
      for (int i = x.tid; i < 64 * NJ; i += NTC) {
        const int t = i / NJ, ck = i % NJ;
        const bf16* src = x.dout + ((x.row0 + t0 + min(t, L - 1)) * x.H + x.h) * D + x.j0 + 8 * ck;
        cp_async16(st + CF::R_DO + io(t, 8 * ck, 64), src, t < L ? 16u : 0u);
      }
    }
    cp_async_commit();
  };
  const uint32_t uY = x.sb + CF::R_Y, uDD = x.sb + CF::R_DD;
#pragma unroll 1
  for (int i = 0; i < STG - 1; ++i) issue(x.nch - 1 - i);
#pragma unroll 1
  for (int n = x.nch - 1; n >= 0; --n) {
    const uint32_t so = (uint32_t)(n % STG) * CF::R_STAGE;
    chain_put<NB>(x, X, CF::R_Y, dsimg + (x.base + n) * kImgS);   // dS after chunk n
    cp_async_wait_group<STG - 2>();
    const bool ok =
        mbar_wait(&x.full[n % STG], (uint32_t)((x.nch - 1 - n) / STG) & 1u, kWaitLimit);
    if (__syncthreads_or(!ok)) {
      chain_give_up<STG>(x, n, max(n - (STG - 2), 0), false);
      return;
    }
    // dDelta = Kend dS + Aqk^T dO: token block tb, n8 tiles jh * NH ..
    float acc[NH][2][4] = {};
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      uint32_t a[4];
      a_km(x.sb + so + CF::R_KA, 128, 16 * tb, 16 * ks, lane, a);          // Kend [t][c] from Kend^T
      if constexpr (NH == 2) {
        uint32_t b[4];
        b_nk(uY, NB, 16 * jh, 16 * ks, lane, b);                           // dS [c][j] from [j][c]
        mma(acc[0][ks & 1], a, b[0], b[1]);
        mma(acc[1][ks & 1], a, b[2], b[3]);
      } else {
        uint32_t b[2];
        b_nk1(uY, NB, 8 * jh, 16 * ks, lane, b);
        mma(acc[0][ks & 1], a, b[0], b[1]);
      }
    }
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
      uint32_t a[4];
      a_km(x.sb + so + CF::R_KA + 16384, 64, 16 * tb, 16 * ks, lane, a);   // Aqk^T [t][r] from Aqk
      if constexpr (NH == 2) {
        uint32_t b[4];
        b_kn(x.sb + so + CF::R_DO, 64, 16 * jh, 16 * ks, lane, b);         // dO [r][j]
        mma(acc[0][ks & 1], a, b[0], b[1]);
        mma(acc[1][ks & 1], a, b[2], b[3]);
      } else {
        uint32_t b[2];
        b_kn1(x.sb + so + CF::R_DO, 64, 8 * jh, 16 * ks, lane, b);
        mma(acc[0][ks & 1], a, b[0], b[1]);
      }
    }
    uint8_t* gD = ddimg + (x.base + n) * kImgD;
    uint8_t* gDl = ddlo + (x.base + n) * kImgD;
#pragma unroll
    for (int p = 0; p < NH; ++p) {
      const int n0 = 8 * (jh * NH + p), jl = n0 + 2 * qd;
      float dd[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) dd[e] = acc[p][0][e] + acc[p][1][e];
      st_mn1(uDD, 64, 16 * tb, n0, lane, dd, -1.f);
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        // dDelta as a bf16 pair: hi, and lo = dDelta - hi (the gradient kernel's
        // T^T dDelta for dv and dbeta takes both)
        const uint32_t o = io(16 * tb + g + 8 * hf, x.j0 + jl, 64);
        const uint32_t hi = pack_bf16(dd[2 * hf], dd[2 * hf + 1]);
        *reinterpret_cast<uint32_t*>(gD + o) = hi;
        *reinterpret_cast<uint32_t*>(gDl + o) =
            pack_bf16(dd[2 * hf] - __uint_as_float(hi << 16),
                      dd[2 * hf + 1] - __uint_as_float(hi & 0xffff0000u));
      }
    }
    __syncthreads();
    // dS <- Diag(exp(Gamma_last)) dS + Qbar^T dO - W^T dDelta
    const float* dec = reinterpret_cast<const float*>(x.sm + so + CF::R_DEC);
    const float d0 = dec[16 * x.w + g], d1 = dec[16 * x.w + g + 8];
    float Y[NJ][4] = {};
#pragma unroll
    for (int nt = 0; nt < NJ; ++nt) {
      X[nt][0] *= d0; X[nt][1] *= d0; X[nt][2] *= d1; X[nt][3] *= d1;
    }
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
      chain_update<NB>(x, x.sb + so + CF::R_QW, x.sb + so + CF::R_DO, X, Y, ks, ks & 1);  // Qbar^T dO
      chain_update<NB>(x, x.sb + so + CF::R_QW + 16384, uDD, X, Y, ks, !(ks & 1));     // W^T (-dDelta)
    }
#pragma unroll
    for (int nt = 0; nt < NJ; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) X[nt][e] += Y[nt][e];
    issue(n - (STG - 1));               // into chunk n + 1's stage, read before this step's barrier
  }
  cp_async_wait_all();
  if (dh0) {
#pragma unroll
    for (int nt = 0; nt < NJ; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int c = 16 * x.w + g + ((e >> 1) << 3), j = x.j0 + 8 * nt + 2 * qd + (e & 1);
        dh0[x.st_off + (size_t)c * D + j] = X[nt][e];
      }
  }
}

// Chain kernel: CTA (xb, h, s) with xb < D / NBF walks sequence s of head h forward for the
// value columns [NBF xb, NBF xb + NBF); the others walk it backward, NBR columns each (the
// reverse step reads more operands, so it takes narrower blocks; both directions fit one wave
// at the headline shape).
template <int NBF, int NBR>
__global__ void __launch_bounds__(NTC, 1)
kda_bwd_chain_kernel(const uint8_t* __restrict__ rec, const float* __restrict__ h0,
                     const int32_t* __restrict__ cu_seqlens, const bf16* __restrict__ dout,
                     const float* __restrict__ dhT, float* __restrict__ dh0,
                     uint8_t* __restrict__ simg, uint8_t* __restrict__ dlimg,
                     uint8_t* __restrict__ dsimg, uint8_t* __restrict__ ddimg,
                     uint8_t* __restrict__ ddlo, int T, int H, long long nslots) {
  constexpr int STG = Chain<NBF>::STG;
  static_assert(Chain<NBR>::STG == STG, "one stage count");
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t full[STG];           // record stage landed (bulk copies)
  ChainCtx x;
  x.sm = align1024(smem_raw);
  x.sb = smem_u32(x.sm);
  x.full = full;
  x.rec = rec;
  x.dout = dout;
  x.tid = threadIdx.x;
  x.w = x.tid >> 5;
  x.lane = x.tid & 31;
  x.g = x.lane >> 2;
  x.qd = x.lane & 3;
  constexpr int NF = D / NBF;
  const bool fwd = (int)blockIdx.x < NF;
  x.j0 = fwd ? (int)blockIdx.x * NBF : ((int)blockIdx.x - NF) * NBR;
  x.h = blockIdx.y;
  x.H = H;
  const int s = blockIdx.z;
  seq_range(cu_seqlens, s, T, x.row0, x.t_beg, x.t_end);
  x.nch = (int)chunk_count(x.t_end - x.t_beg);
  x.base = (size_t)x.h * (size_t)nslots + (size_t)seq_chunk_base(cu_seqlens, s, T);
  x.st_off = ((size_t)s * H + x.h) * D * D;
  if (x.tid == 0) {
#pragma unroll
    for (int i = 0; i < STG; ++i) mbar_init(&full[i], 1);
    fence_mbar_init();
  }
  grid_dep_launch();                       // the gradient kernel may start preloading its inputs
  __syncthreads();                         // the barriers are initialised
  grid_dep_wait();                         // the records are complete
  if (fwd) chain_forward<NBF>(x, h0, simg, dlimg);
  else chain_reverse<NBR>(x, dhT, dh0, dsimg, ddimg, ddlo);
}

// ============================================================================
// Gradient kernel: one CTA per (chunk slot, head), 16 warps.  Warp w owns token
// rows r0 = 16 tb .. r0 + 15 (tb = w % 4: one decay block) and channels
// c0 = 32 cq .. c0 + 31 (cq = w / 4) of dq, dk and dGamma in registers: lane
// (g, qd) holds rows r0 + g + 8 hf (hf = 0, 1) and channels c0 + 8 nt + 2 qd + e1
// (nt = 0..3, e1 = 0, 1), element [nt][2 hf + e1] -- the m16n8 accumulator layout.
// ============================================================================
constexpr int NTG = 512;                       // threads of the gradient kernel
constexpr int LDG = 136;                       // Gamma / dGamma row stride (floats)
constexpr uint32_t G_Q = 0;                    // q image [t][c]
constexpr uint32_t G_K = 16384;                // k image [t][c]
constexpr uint32_t G_G = 32768;                // Gamma fp32 [64][LDG]
constexpr uint32_t G_S0 = 67584;               // S image [j][c]  | dDelta lo image, A fp32 [64][64] | R images
constexpr uint32_t G_DS = 100352;              // dS image [j][c] | Kb, Vb images | X fp32 [64][68]
constexpr uint32_t G_DO = 133120;              // dO image [t][j] | V image | dT^T fp32 [64][68]
constexpr uint32_t G_DL = 149504;              // Delta image     | T image (bf16)
constexpr uint32_t G_DD = 165888;              // dDelta image    | T^T fp32 [64][68]
constexpr uint32_t G_DW = 182272;              // dW image [t][c]
constexpr uint32_t G_AQK = 198656;             // dAqk image [r][i]
constexpr uint32_t G_DA = 206848;              // dA image [r][i]
constexpr uint32_t GRAD_SMEM = 215040 + 1024;
// R images (phase 4), from G_S0: R^(a) rows i < 16(a+1); R'k^(b), R'q^(b) rows r >= 16b
__host__ __device__ constexpr uint32_t r_row(int a) {
  return a == 0 ? 0u : a == 1 ? 4096u : a == 2 ? 12288u : 24576u;
}
__host__ __device__ constexpr uint32_t r_col(int b) {
  return b == 0 ? 0u : b == 1 ? 16384u : b == 2 ? 28672u : 36864u;
}
constexpr uint32_t G_RR = G_S0, G_RK = G_S0 + 40960, G_RQ = G_S0 + 81920;
// factors between the blocks' reference points, fp32 [6][128] each (after the R images)
constexpr uint32_t G_F1 = G_S0 + 122880, G_F2 = G_F1 + 3072;
// exact within-block corrections of unsafe channels (phase 4, after the products):
// fp32 [64][128] each
constexpr uint32_t G_CYA = G_S0, G_CYQ = G_S0 + 32768, G_CZ = G_S0 + 65536;

template <bool GRPD>
__global__ void __launch_bounds__(NTG, 1)
kda_bwd_grad_kernel(const bf16* __restrict__ q, const bf16* __restrict__ k,
                    const bf16* __restrict__ v, const float* __restrict__ g,
                    const float* __restrict__ beta, const bf16* __restrict__ dout,
                    const int32_t* __restrict__ cu_seqlens, const uint8_t* __restrict__ rec,
                    const uint8_t* __restrict__ simg, const uint8_t* __restrict__ dlimg,
                    const uint8_t* __restrict__ dsimg, const uint8_t* __restrict__ ddimg,
                    const uint8_t* __restrict__ ddlo,
                    float* __restrict__ dq, float* __restrict__ dk, float* __restrict__ dv,
                    float* __restrict__ dg, float* __restrict__ dbeta, int B, int T, int H,
                    int gsh, long long nslots) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1024(smem_raw);
  const uint32_t sb = smem_u32(sm);
  __shared__ float s_beta[C], s_dbeta[C], s_dgl[D], s_part[4][D], s_daqk[C];
  __shared__ __align__(16) uint8_t s_uns[4][D];
  __shared__ uint64_t s_img_bar;               // the chains' four images landed

  const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31, g8 = lane >> 2, qd = lane & 3;
  const long long slot = blockIdx.x;
  const int h = blockIdx.y;

  // which chunk of which sequence this slot is (numbered as the prep kernel numbers them)
  long long row0 = 0, t_beg = 0, t_end = 0, n = 0;
  if (!cu_seqlens) {
    const long long per = chunk_count(T);
    if (per == 0 || slot >= per * B) return;
    const int s = (int)(slot / per);
    n = slot - (long long)s * per;
    seq_range(nullptr, s, T, row0, t_beg, t_end);
  } else {
    long long bse = 0;
    bool found = false;
    for (int d = 0; d < B && !found; ++d) {
      seq_range(cu_seqlens, d, T, row0, t_beg, t_end);
      const long long nc = chunk_count(t_end - t_beg);
      if (slot < bse + nc) { n = slot - bse; found = true; }
      bse += nc;
    }
    if (!found) return;
  }
  const long long t0 = t_beg + n * C;
  const int L = (int)min((long long)C, t_end - t0);
  const long long rb = row0 + t0;                      // first token row of the chunk
  const size_t ix = (size_t)h * (size_t)nslots + (size_t)slot;
  const uint8_t* rc = rec + ix * rec::BYTES_BWD;
  float* G = reinterpret_cast<float*>(sm + G_G);

  // ---- phase 0: loads (the inputs first; the chains' images once the chains are done)
  if (tid == 0) {
    mbar_init(&s_img_bar, 1);
    fence_mbar_init();
  }
  for (int i = tid; i < 1024; i += NTG) {
    const int t = i >> 4, c8 = i & 15;
    const long long src = ((rb + min(t, L - 1)) * H + h) * D + 8 * c8;
    const uint32_t ok = t < L ? 16u : 0u;
    cp_async16(sm + G_DO + io(t, 8 * c8, 64), dout + src, ok);
    cp_async16(sm + G_Q + io(t, 8 * c8, 64), q + src, ok);
    cp_async16(sm + G_K + io(t, 8 * c8, 64), k + src, ok);
  }
  if constexpr (!GRPD) {
    for (int i = tid; i < 2048; i += NTG) {
      const int t = i >> 5, c4 = i & 31;
      cp_async16(G + t * LDG + 4 * c4, g + ((rb + min(t, L - 1)) * H + h) * D + 4 * c4,
                 t < L ? 16u : 0u);
    }
  }
  cp_async_commit();
  grid_dep_wait();
  if (tid == 0) {                       // the images: four bulk copies on one barrier
    mbar_arrive_expect_tx(&s_img_bar, 2 * kImgS + 2 * kImgD);
    bulk_g2s(sm + G_S0, simg + ix * kImgS, kImgS, &s_img_bar);
    bulk_g2s(sm + G_DS, dsimg + ix * kImgS, kImgS, &s_img_bar);
    bulk_g2s(sm + G_DL, dlimg + ix * kImgD, kImgD, &s_img_bar);
    bulk_g2s(sm + G_DD, ddimg + ix * kImgD, kImgD, &s_img_bar);
  }
  if (tid < C) {
    s_beta[tid] = tid < L ? beta[(rb + tid) * H + h] : 0.f;
    s_dbeta[tid] = 0.f;
  }
  if (tid < D) s_dgl[tid] = 0.f;
  if constexpr (GRPD) {
    const int ng = D >> gsh;
    for (int i = tid; i < C * D; i += NTG) {
      const int t = i >> 7, c = i & 127;
      G[t * LDG + c] = t < L ? g[((rb + t) * H + h) * ng + (c >> gsh)] : 0.f;
    }
  }
  cp_async_wait_all();                  // the inputs (the images may still be in flight)
  __syncthreads();
  // Gamma = cumsum g per channel: four threads per channel, 16 rows each
  {
    const int c = tid & 127, part = tid >> 7;
    float x[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) x[e] = G[(16 * part + e) * LDG + c];
#pragma unroll
    for (int e = 1; e < 16; ++e) x[e] += x[e - 1];
    s_part[part][c] = x[15];
    __syncthreads();
    float add = 0.f;
    for (int p2 = 0; p2 < part; ++p2) add += s_part[p2][c];
#pragma unroll
    for (int e = 0; e < 16; ++e) G[(16 * part + e) * LDG + c] = x[e] + add;
  }
  {
    bool ok = true;
    if (w == 0) ok = mbar_wait(&s_img_bar, 0, kWaitLimit);
    if (__syncthreads_or(!ok)) {        // the images never arrived: flag, let them land, leave
      if (tid == 0) {
        atomicExch(&g_bwd_tc_timeout, 1);
        mbar_wait(&s_img_bar, 0, kWaitLimit);
      }
      return;
    }
  }
  // unsafe (block, channel) pairs; dGamma_last's state term e^Gamma_last sum_j S dS
  bool any_uns = false, far = false;
  {
    const int c = tid & 127, a = tid >> 7;
    const bool u = G[16 * a * LDG + c] - G[(16 * a + 15) * LDG + c] > kUnsafeDecay;
    s_uns[a][c] = u ? 1 : 0;
    any_uns = u;
    // the mid-chunk reference (row 32) serves all pairs when neither half decays by more
    // than kUnsafeDecay on this channel
    if (a == 0)
      far = G[c] - G[32 * LDG + c] > kUnsafeDecay || G[32 * LDG + c] - G[63 * LDG + c] > kUnsafeDecay;
    const int c8 = tid & 15, jg = tid >> 4;           // 32 groups of 4 rows j
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
      const int j = 4 * jg + jj;
      const uint4 a4 = *reinterpret_cast<const uint4*>(sm + G_S0 + io(j, 8 * c8, 128));
      const uint4 b4 = *reinterpret_cast<const uint4*>(sm + G_DS + io(j, 8 * c8, 128));
      const uint32_t aw[4] = {a4.x, a4.y, a4.z, a4.w}, bw[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        acc[2 * e] = fmaf(__uint_as_float(aw[e] << 16), __uint_as_float(bw[e] << 16), acc[2 * e]);
        acc[2 * e + 1] = fmaf(__uint_as_float(aw[e] & 0xffff0000u),
                              __uint_as_float(bw[e] & 0xffff0000u), acc[2 * e + 1]);
      }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], 16);
    if (lane < 16) {
#pragma unroll
      for (int e = 0; e < 8; ++e)
        atomicAdd(&s_dgl[8 * c8 + e], acc[e] * __expf(G[63 * LDG + 8 * c8 + e]));
    }
  }
  const bool fix = __syncthreads_or(any_uns) != 0;
  const bool mid = __syncthreads_or(far) == 0;

  const int tb = w & 3, cq = w >> 2, r0 = 16 * tb, c0 = 32 * cq;
  float dQ[4][4], dK[4][4], dG[4][4];
#pragma unroll
  for (int nt = 0; nt < 4; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) dQ[nt][e] = dK[nt][e] = dG[nt][e] = 0.f;
  // The element pair (e = 2 hf, 2 hf + 1) of n8 tile nt: row r0 + g8 + 8 hf, columns
  // c0 + 8 nt + 2 qd (+1).  Its values in a [t][c] image and in Gamma:
  const uint32_t prow = (uint32_t)(cq >> 1) * 8192u + (uint32_t)(r0 + g8) * 128u + (uint32_t)qd * 4u;
  const int cb = 4 * (cq & 1);                 // the tile's first 16-byte chunk in its panel
  auto img2 = [&](uint32_t img, int hf, int nt) -> float2 {
    return bf2_at(sm + img + prow + hf * 1024 + (((cb + nt) ^ g8) << 4));
  };
  auto gam2 = [&](int row, int nt) -> float2 {
    return *reinterpret_cast<const float2*>(G + row * LDG + c0 + 8 * nt + 2 * qd);
  };

  // ---- phase 1: dQbar and dW (against S^T), dKend (dS^T), dAqk
#pragma unroll
  for (int np = 0; np < 2; ++np) {
    float aq[2][4] = {}, aw[2][4] = {};
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      uint32_t a1[4], a2[4], b[4];
      a_mk(sb + G_DO, 64, r0, 16 * ks, lane, a1);
      a_mk(sb + G_DD, 64, r0, 16 * ks, lane, a2);
      b_kn(sb + G_S0, 128, c0 + 16 * np, 16 * ks, lane, b);       // S^T [j][c]
      mma(aq[0], a1, b[0], b[1]);
      mma(aq[1], a1, b[2], b[3]);
      mma(aw[0], a2, b[0], b[1]);
      mma(aw[1], a2, b[2], b[3]);
    }
#pragma unroll
    for (int sub = 0; sub < 2; ++sub) {
      const int nt = 2 * np + sub;
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const float2 gp = gam2(r0 + g8 + 8 * hf, nt), qv = img2(G_Q, hf, nt);
        const float e0 = __expf(gp.x), e1 = __expf(gp.y);
        const float x0 = aq[sub][2 * hf], x1 = aq[sub][2 * hf + 1];
        dQ[nt][2 * hf] = fmaf(x0, e0, dQ[nt][2 * hf]);
        dQ[nt][2 * hf + 1] = fmaf(x1, e1, dQ[nt][2 * hf + 1]);
        dG[nt][2 * hf] = fmaf(x0 * qv.x, e0, dG[nt][2 * hf]);
        dG[nt][2 * hf + 1] = fmaf(x1 * qv.y, e1, dG[nt][2 * hf + 1]);
      }
    }
    st_mn(sb + G_DW, 64, r0, c0 + 16 * np, lane, aw[0], aw[1], -1.f);   // dW = -dDelta S^T
  }
  __syncthreads();                      // S image no longer read: dDelta's lo image and A go there
  for (int i = tid; i < 1024; i += NTG) {
    cp_async16(sm + G_S0 + 16 * i, ddlo + ix * kImgD + 16 * i, 16u);
    cp_async16(sm + G_S0 + 16384 + 16 * i, rc + rec::AMAT + 16 * i, 16u);
  }
  cp_async_commit();
#pragma unroll
  for (int np = 0; np < 2; ++np) {
    float ak[2][4] = {};
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      uint32_t a[4], b[4];
      a_mk(sb + G_DL, 64, r0, 16 * ks, lane, a);
      b_kn(sb + G_DS, 128, c0 + 16 * np, 16 * ks, lane, b);       // dS^T [j][c]
      mma(ak[0], a, b[0], b[1]);
      mma(ak[1], a, b[2], b[3]);
    }
#pragma unroll
    for (int sub = 0; sub < 2; ++sub) {
      const int nt = 2 * np + sub;
      const float2 gl = gam2(63, nt);
      float cs0 = 0.f, cs1 = 0.f;
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const float2 gp = gam2(r0 + g8 + 8 * hf, nt), kv = img2(G_K, hf, nt);
        const float e0 = __expf(gl.x - gp.x), e1 = __expf(gl.y - gp.y);
        const float x0 = ak[sub][2 * hf], x1 = ak[sub][2 * hf + 1];
        dK[nt][2 * hf] = fmaf(x0, e0, dK[nt][2 * hf]);
        dK[nt][2 * hf + 1] = fmaf(x1, e1, dK[nt][2 * hf + 1]);
        const float t0v = x0 * kv.x * e0, t1v = x1 * kv.y * e1;
        dG[nt][2 * hf] -= t0v;
        dG[nt][2 * hf + 1] -= t1v;
        cs0 += t0v;
        cs1 += t1v;
      }
#pragma unroll
      for (int m = 4; m < 32; m <<= 1) {
        cs0 += __shfl_xor_sync(0xffffffffu, cs0, m);
        cs1 += __shfl_xor_sync(0xffffffffu, cs1, m);
      }
      if (g8 == 0) {
        atomicAdd(&s_dgl[c0 + 8 * nt + 2 * qd], cs0);
        atomicAdd(&s_dgl[c0 + 8 * nt + 2 * qd + 1], cs1);
      }
    }
  }
  {   // dAqk (rows r0.., columns 16 cq ..), lower triangle
    float aa[2][4] = {};
    if (cq <= tb) {
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        uint32_t a[4], b[4];
        a_mk(sb + G_DO, 64, r0, 16 * ks, lane, a);
        b_nk(sb + G_DL, 64, 16 * cq, 16 * ks, lane, b);             // Delta^T from Delta [i][j]
        mma(aa[0], a, b[0], b[1]);
        mma(aa[1], a, b[2], b[3]);
      }
#pragma unroll
      for (int sub = 0; sub < 2; ++sub)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int r = r0 + g8 + ((e >> 1) << 3);
          const int i = 16 * cq + 8 * sub + 2 * qd + (e & 1);
          if (i > r) aa[sub][e] = 0.f;
          // the diagonal (i = r, decay factor e^0): kept apart in fp32 and left out of the
          // image, so that the decay-weighted products below never form its dGamma terms,
          // which cancel exactly (row side + q k dAqk, column side - q k dAqk); its dq and
          // dk terms are added in phase 5
          if (i == r) {
            s_daqk[r] = aa[sub][e];
            aa[sub][e] = 0.f;
          }
        }
    }
    st_mn(sb + G_AQK, 64, r0, 16 * cq, lane, aa[0], aa[1], 1.f);
  }
  __syncthreads();                      // dO, Delta, dS no longer read
  for (int i = tid; i < 1024; i += NTG) {
    const int t = i >> 4, c8 = i & 15;
    cp_async16(sm + G_DO + io(t, 8 * c8, 64), v + ((rb + min(t, L - 1)) * H + h) * D + 8 * c8,
               t < L ? 16u : 0u);
  }
  // the T image (bf16 [r][i], as the record holds it) to G_DL
  for (int i = tid; i < 512; i += NTG) cp_async16(sm + G_DL + 16 * i, rc + rec::TMAT + 16 * i, 16u);
  cp_async_commit();
  // Kb = diag(beta) Kbar = beta k e^Gamma (image [i][c] at G_DS)
  for (int i = tid; i < 1024; i += NTG) {
    const int t = i >> 4, c8 = i & 15;
    const float bt = s_beta[t];
    const float4 ga = *reinterpret_cast<const float4*>(G + t * LDG + 8 * c8);
    const float4 gb = *reinterpret_cast<const float4*>(G + t * LDG + 8 * c8 + 4);
    const uint4 kw = *reinterpret_cast<const uint4*>(sm + G_K + io(t, 8 * c8, 64));
    const float gv[8] = {ga.x, ga.y, ga.z, ga.w, gb.x, gb.y, gb.z, gb.w};
    const uint32_t kk[4] = {kw.x, kw.y, kw.z, kw.w};
    float x[8];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      x[2 * e] = bt * __uint_as_float(kk[e] << 16) * __expf(gv[2 * e]);
      x[2 * e + 1] = bt * __uint_as_float(kk[e] & 0xffff0000u) * __expf(gv[2 * e + 1]);
    }
    *reinterpret_cast<uint4*>(sm + G_DS + io(t, 8 * c8, 64)) =
        make_uint4(pack_bf16(x[0], x[1]), pack_bf16(x[2], x[3]), pack_bf16(x[4], x[5]),
                   pack_bf16(x[6], x[7]));
  }
  cp_async_wait_all();
  __syncthreads();
  const float* Am = reinterpret_cast<const float*>(sm + G_S0 + 16384);   // A [r][i]
  // Vb = diag(beta) V (image [i][j] at G_DS + 16384)
  for (int i = tid; i < 1024; i += NTG) {
    const int t = i >> 4, c8 = i & 15;
    const float bt = s_beta[t];
    const uint4 vw = *reinterpret_cast<const uint4*>(sm + G_DO + io(t, 8 * c8, 64));
    const uint32_t vv[4] = {vw.x, vw.y, vw.z, vw.w};
    uint32_t o[4];
#pragma unroll
    for (int e = 0; e < 4; ++e)
      o[e] = pack_bf16(bt * __uint_as_float(vv[e] << 16), bt * __uint_as_float(vv[e] & 0xffff0000u));
    *reinterpret_cast<uint4*>(sm + G_DS + 16384 + io(t, 8 * c8, 64)) =
        make_uint4(o[0], o[1], o[2], o[3]);
  }
  __syncthreads();

  // ---- phase 2: [dVb | dKb] = T^T [dDelta | dW] for token rows i in block tb
  {
    float dbp[2] = {0.f, 0.f};                 // dbeta parts of rows r0 + g8 (+8)
#pragma unroll
    for (int np = 0; np < 2; ++np) {
      float av[2][4] = {}, ak[2][4] = {};
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        if (ks < tb) continue;                 // T[r][i] = 0 for r < i
        uint32_t a[4], bv[4], bk[4];
        a_km(sb + G_DL, 64, r0, 16 * ks, lane, a);                  // T^T [i][r] from T [r][i]
        b_kn(sb + G_DD, 64, c0 + 16 * np, 16 * ks, lane, bv);      // dDelta [r][j] (hi)
        b_kn(sb + G_DW, 64, c0 + 16 * np, 16 * ks, lane, bk);      // dW [r][c]
        mma(av[0], a, bv[0], bv[1]);
        mma(av[1], a, bv[2], bv[3]);
        b_kn(sb + G_S0, 64, c0 + 16 * np, 16 * ks, lane, bv);      // dDelta (lo)
        mma(av[0], a, bv[0], bv[1]);
        mma(av[1], a, bv[2], bv[3]);
        mma(ak[0], a, bk[0], bk[1]);
        mma(ak[1], a, bk[2], bk[3]);
      }
#pragma unroll
      for (int sub = 0; sub < 2; ++sub) {
        const int nt = 2 * np + sub;
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          const int i = r0 + g8 + 8 * hf, c = c0 + 8 * nt + 2 * qd;
          const float bi = s_beta[i];
          const float2 vv = img2(G_DO, hf, nt), kv = img2(G_K, hf, nt), gp = gam2(i, nt);
          const float x0 = av[sub][2 * hf], x1 = av[sub][2 * hf + 1];
          if (i < L)
            *reinterpret_cast<float2*>(dv + ((rb + i) * H + h) * D + c) =
                make_float2(bi * x0, bi * x1);
          const float e0 = __expf(gp.x), e1 = __expf(gp.y);
          const float kb0 = kv.x * e0, kb1 = kv.y * e1;             // Kbar
          const float y0 = ak[sub][2 * hf], y1 = ak[sub][2 * hf + 1];
          dK[nt][2 * hf] = fmaf(bi * y0, e0, dK[nt][2 * hf]);
          dK[nt][2 * hf + 1] = fmaf(bi * y1, e1, dK[nt][2 * hf + 1]);
          dG[nt][2 * hf] = fmaf(bi * y0, kb0, dG[nt][2 * hf]);
          dG[nt][2 * hf + 1] = fmaf(bi * y1, kb1, dG[nt][2 * hf + 1]);
          dbp[hf] += x0 * vv.x + x1 * vv.y + y0 * kb0 + y1 * kb1;
        }
      }
    }
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      float x = dbp[hf];
      x += __shfl_xor_sync(0xffffffffu, x, 1);
      x += __shfl_xor_sync(0xffffffffu, x, 2);
      if (qd == 0) atomicAdd(&s_dbeta[r0 + g8 + 8 * hf], x);
    }
  }
  __syncthreads();                      // V no longer read

  // ---- phase 3: dT = dDelta Vb^T + dW Kb^T, X = dT T^T, dM = -T^T X (strictly lower),
  // on the tensor cores: dT and X as bf16 images [r][i], [r][b] at G_DO, G_DO + 8192
  {                                     // dT tile: rows r0 .., columns i = 16 cq ..
    float at[2][2][4] = {};             // two accumulator pairs: even / odd K steps
    if (cq <= tb) {                     // (tiles above the diagonal are never read: zeros)
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        uint32_t a[4], b[4];
        a_mk(sb + G_DD, 64, r0, 16 * ks, lane, a);
        b_nk(sb + G_DS + 16384, 64, 16 * cq, 16 * ks, lane, b);   // Vb^T from Vb [i][j]
        mma(at[ks & 1][0], a, b[0], b[1]);
        mma(at[ks & 1][1], a, b[2], b[3]);
      }
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        uint32_t a[4], b[4];
        a_mk(sb + G_DW, 64, r0, 16 * ks, lane, a);
        b_nk(sb + G_DS, 64, 16 * cq, 16 * ks, lane, b);           // Kb^T from Kb [i][c]
        mma(at[ks & 1][0], a, b[0], b[1]);
        mma(at[ks & 1][1], a, b[2], b[3]);
      }
#pragma unroll
      for (int sub = 0; sub < 2; ++sub)
#pragma unroll
        for (int e = 0; e < 4; ++e) at[0][sub][e] += at[1][sub][e];
    }
    st_mn(sb + G_DO, 64, r0, 16 * cq, lane, at[0][0], at[0][1], 1.f);
  }
  __syncthreads();
  {                                     // X tile: rows r0 .., columns b = 16 cq .. (r > b only)
    float ax[2][4] = {};
    if (cq <= tb) {
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        if (ks > cq) continue;          // T[b][i] = 0 for i > b
        uint32_t a[4], b[4];
        a_mk(sb + G_DO, 64, r0, 16 * ks, lane, a);                  // dT [r][i]
        b_nk(sb + G_DL, 64, 16 * cq, 16 * ks, lane, b);             // T^T from T [b][i]
        mma(ax[0], a, b[0], b[1]);
        mma(ax[1], a, b[2], b[3]);
      }
#pragma unroll
      for (int sub = 0; sub < 2; ++sub)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int r = r0 + g8 + ((e >> 1) << 3), bb = 16 * cq + 8 * sub + 2 * qd + (e & 1);
          if (r <= bb) ax[sub][e] = 0.f;
        }
    }
    st_mn(sb + G_DO + 8192, 64, r0, 16 * cq, lane, ax[0], ax[1], 1.f);
  }
  __syncthreads();
  {                                     // dM tile: rows a = r0 .., columns b = 16 cq ..
    float am[2][4] = {};
    if (cq <= tb) {
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        if (ks < tb) continue;          // T[r][a] = 0 for r < a
        uint32_t a[4], b[4];
        a_km(sb + G_DL, 64, r0, 16 * ks, lane, a);                  // T^T [a][r] from T [r][a]
        b_kn(sb + G_DO + 8192, 64, 16 * cq, 16 * ks, lane, b);      // X [r][b]
        mma(am[0], a, b[0], b[1]);
        mma(am[1], a, b[2], b[3]);
      }
    }
    float dbp[2] = {0.f, 0.f};
#pragma unroll
    for (int sub = 0; sub < 2; ++sub)
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const int ra = r0 + g8 + 8 * hf, bb = 16 * cq + 8 * sub + 2 * qd;
        const float m0 = ra > bb ? -am[sub][2 * hf] : 0.f;
        const float m1 = ra > bb + 1 ? -am[sub][2 * hf + 1] : 0.f;
        const float2 a2 = *reinterpret_cast<const float2*>(Am + ra * 64 + bb);
        dbp[hf] += m0 * a2.x + m1 * a2.y;
        am[sub][2 * hf] = s_beta[ra] * m0;
        am[sub][2 * hf + 1] = s_beta[ra] * m1;
      }
    st_mn(sb + G_DA, 64, r0, 16 * cq, lane, am[0], am[1], 1.f);   // dA = diag(beta) dM
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      float x = dbp[hf];
      x += __shfl_xor_sync(0xffffffffu, x, 1);
      x += __shfl_xor_sync(0xffffffffu, x, 2);
      if (qd == 0) atomicAdd(&s_dbeta[r0 + g8 + 8 * hf], x);
    }
  }
  __syncthreads();                      // T, A, dT, X no longer read

  // ---- phase 4: the decay-weighted Gram products
  // R^(a)[i][c] = k_ic e^{G_16a,c - G_ic}, i < 16(a+1) (block a's own rows zero where
  // unsafe); R'x^(b)[r - 16b][c] = x_rc e^{G_rc - G_16b+15,c}, r >= 16b (likewise).
  // One item: 8 channels of one row of one image.
  auto build_r = [&](bool flags) {
    for (int i = tid; i < 160 * 16; i += NTG) {
      const int x = i >> 4, c8 = i & 15;
      const int a = x >= 96 ? 3 : x >= 48 ? 2 : x >= 16 ? 1 : 0;
      const int ii = x - 8 * a * (a + 1);
      const float* gi = G + ii * LDG + 8 * c8;
      const float* ga = G + 16 * a * LDG + 8 * c8;
      const float4 i0 = *reinterpret_cast<const float4*>(gi), i1 = *reinterpret_cast<const float4*>(gi + 4);
      const float4 a0 = *reinterpret_cast<const float4*>(ga), a1 = *reinterpret_cast<const float4*>(ga + 4);
      const uint4 kw = *reinterpret_cast<const uint4*>(sm + G_K + io(ii, 8 * c8, 64));
      const float dgv[8] = {a0.x - i0.x, a0.y - i0.y, a0.z - i0.z, a0.w - i0.w,
                            a1.x - i1.x, a1.y - i1.y, a1.z - i1.z, a1.w - i1.w};
      const uint32_t kk[4] = {kw.x, kw.y, kw.z, kw.w};
      uint32_t zm = 0;                  // channels whose within-block entries are zero
      if (flags && ii >= 16 * a) {
        const uint2 un = *reinterpret_cast<const uint2*>(&s_uns[a][8 * c8]);
#pragma unroll
        for (int e = 0; e < 8; ++e) zm |= (((e < 4 ? un.x : un.y) >> (8 * (e & 3))) & 1u) << e;
      }
      uint32_t o[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float v0 = __uint_as_float(kk[e] << 16) * __expf(fminf(dgv[2 * e], 80.f));
        const float v1 = __uint_as_float(kk[e] & 0xffff0000u) * __expf(fminf(dgv[2 * e + 1], 80.f));
        o[e] = pack_bf16(((zm >> (2 * e)) & 1u) ? 0.f : v0, ((zm >> (2 * e + 1)) & 1u) ? 0.f : v1);
      }
      *reinterpret_cast<uint4*>(sm + G_RR + r_row(a) + io(ii, 8 * c8, 16 * (a + 1))) =
          make_uint4(o[0], o[1], o[2], o[3]);
    }
    for (int i = tid; i < 160 * 16; i += NTG) {
      const int x = i >> 4, c8 = i & 15;
      const int b = x >= 144 ? 3 : x >= 112 ? 2 : x >= 64 ? 1 : 0;
      const int start = b == 0 ? 0 : b == 1 ? 64 : b == 2 ? 112 : 144;
      const int rr = x - start, r = 16 * b + rr, nrows = 64 - 16 * b;
      const float* gr = G + r * LDG + 8 * c8;
      const float* gb = G + (16 * b + 15) * LDG + 8 * c8;
      const float4 r0v = *reinterpret_cast<const float4*>(gr), r1v = *reinterpret_cast<const float4*>(gr + 4);
      const float4 b0v = *reinterpret_cast<const float4*>(gb), b1v = *reinterpret_cast<const float4*>(gb + 4);
      const uint4 kw = *reinterpret_cast<const uint4*>(sm + G_K + io(r, 8 * c8, 64));
      const uint4 qw = *reinterpret_cast<const uint4*>(sm + G_Q + io(r, 8 * c8, 64));
      const float dgv[8] = {r0v.x - b0v.x, r0v.y - b0v.y, r0v.z - b0v.z, r0v.w - b0v.w,
                            r1v.x - b1v.x, r1v.y - b1v.y, r1v.z - b1v.z, r1v.w - b1v.w};
      const uint32_t kk[4] = {kw.x, kw.y, kw.z, kw.w}, qq[4] = {qw.x, qw.y, qw.z, qw.w};
      uint32_t zm = 0;
      if (flags && rr < 16) {
        const uint2 un = *reinterpret_cast<const uint2*>(&s_uns[b][8 * c8]);
#pragma unroll
        for (int e = 0; e < 8; ++e) zm |= (((e < 4 ? un.x : un.y) >> (8 * (e & 3))) & 1u) << e;
      }
      uint32_t ok_[4], oq[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float f0 = ((zm >> (2 * e)) & 1u) ? 0.f : __expf(fminf(dgv[2 * e], 80.f));
        const float f1 = ((zm >> (2 * e + 1)) & 1u) ? 0.f : __expf(fminf(dgv[2 * e + 1], 80.f));
        ok_[e] = pack_bf16(__uint_as_float(kk[e] << 16) * f0, __uint_as_float(kk[e] & 0xffff0000u) * f1);
        oq[e] = pack_bf16(__uint_as_float(qq[e] << 16) * f0, __uint_as_float(qq[e] & 0xffff0000u) * f1);
      }
      const uint32_t o = r_col(b) + io(rr, 8 * c8, nrows);
      *reinterpret_cast<uint4*>(sm + G_RK + o) = make_uint4(ok_[0], ok_[1], ok_[2], ok_[3]);
      *reinterpret_cast<uint4*>(sm + G_RQ + o) = make_uint4(oq[0], oq[1], oq[2], oq[3]);
    }
  };
  if (mid) {
    // one reference point for the whole chunk, P = Gamma at row 32 (every factor within
    // e^{+-kUnsafeDecay}): R = k e^{P - G}, R'k = k e^{G - P}, R'q = q e^{G - P}, 64 rows each
    for (int i = tid; i < C * 16; i += NTG) {
      const int x = i >> 4, c8 = i & 15;
      const float* gx = G + x * LDG + 8 * c8;
      const float* gp = G + 32 * LDG + 8 * c8;
      const float4 x0 = *reinterpret_cast<const float4*>(gx), x1 = *reinterpret_cast<const float4*>(gx + 4);
      const float4 p0 = *reinterpret_cast<const float4*>(gp), p1 = *reinterpret_cast<const float4*>(gp + 4);
      const uint4 kw = *reinterpret_cast<const uint4*>(sm + G_K + io(x, 8 * c8, 64));
      const uint4 qw = *reinterpret_cast<const uint4*>(sm + G_Q + io(x, 8 * c8, 64));
      const float dv8[8] = {p0.x - x0.x, p0.y - x0.y, p0.z - x0.z, p0.w - x0.w,
                            p1.x - x1.x, p1.y - x1.y, p1.z - x1.z, p1.w - x1.w};
      const uint32_t kk[4] = {kw.x, kw.y, kw.z, kw.w}, qq[4] = {qw.x, qw.y, qw.z, qw.w};
      uint32_t orr[4], ork[4], orq[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float up0 = __expf(dv8[2 * e]), up1 = __expf(dv8[2 * e + 1]);
        const float dn0 = __expf(-dv8[2 * e]), dn1 = __expf(-dv8[2 * e + 1]);
        const float k0 = __uint_as_float(kk[e] << 16), k1 = __uint_as_float(kk[e] & 0xffff0000u);
        const float q0 = __uint_as_float(qq[e] << 16), q1 = __uint_as_float(qq[e] & 0xffff0000u);
        orr[e] = pack_bf16(k0 * up0, k1 * up1);
        ork[e] = pack_bf16(k0 * dn0, k1 * dn1);
        orq[e] = pack_bf16(q0 * dn0, q1 * dn1);
      }
      const uint32_t o = io(x, 8 * c8, 64);
      *reinterpret_cast<uint4*>(sm + G_RR + o) = make_uint4(orr[0], orr[1], orr[2], orr[3]);
      *reinterpret_cast<uint4*>(sm + G_RK + o) = make_uint4(ork[0], ork[1], ork[2], ork[3]);
      *reinterpret_cast<uint4*>(sm + G_RQ + o) = make_uint4(orq[0], orq[1], orq[2], orq[3]);
    }
  } else if (fix) {
    build_r(true);
  } else {
    // No unsafe channel: each row's within-block factor is formed once and scaled by
    // factors between block references (all <= 1):
    //   R^(a)[x]  = k_x e^{G_16i - G_x} F1(a, i),        F1(a, i) = e^{G_16a - G_16i},  a > i
    //   R'^(b)[x] = x_x e^{G_x - G_16i+15} F2(i, b),     F2(i, b) = e^{G_16i+15 - G_16b+15}, b < i
    // (i = block of row x; pair index hi (hi - 1) / 2 + lo).
    float* F1 = reinterpret_cast<float*>(sm + G_F1);
    float* F2 = reinterpret_cast<float*>(sm + G_F2);
    for (int i = tid; i < 6 * D; i += NTG) {
      const int pr = i >> 7, c = i & 127;
      const int hi = pr == 0 ? 1 : pr < 3 ? 2 : 3, lo = pr - hi * (hi - 1) / 2;
      F1[i] = __expf(G[16 * hi * LDG + c] - G[16 * lo * LDG + c]);
      F2[i] = __expf(G[(16 * hi + 15) * LDG + c] - G[(16 * lo + 15) * LDG + c]);
    }
    __syncthreads();
    for (int i = tid; i < C * 16; i += NTG) {
      const int x = i >> 4, c8 = i & 15, blk = x >> 4;
      const float* gx = G + x * LDG + 8 * c8;
      const float* gs = G + 16 * blk * LDG + 8 * c8;
      const float* ge = G + (16 * blk + 15) * LDG + 8 * c8;
      const float4 x0 = *reinterpret_cast<const float4*>(gx), x1 = *reinterpret_cast<const float4*>(gx + 4);
      const float4 s0 = *reinterpret_cast<const float4*>(gs), s1 = *reinterpret_cast<const float4*>(gs + 4);
      const float4 e0 = *reinterpret_cast<const float4*>(ge), e1 = *reinterpret_cast<const float4*>(ge + 4);
      const uint4 kw = *reinterpret_cast<const uint4*>(sm + G_K + io(x, 8 * c8, 64));
      const uint4 qw = *reinterpret_cast<const uint4*>(sm + G_Q + io(x, 8 * c8, 64));
      const float gxv[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
      const float gsv[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
      const float gev[8] = {e0.x, e0.y, e0.z, e0.w, e1.x, e1.y, e1.z, e1.w};
      const uint32_t kk[4] = {kw.x, kw.y, kw.z, kw.w}, qq[4] = {qw.x, qw.y, qw.z, qw.w};
      float rk[8], ck[8], cqv[8];                // k e^{G_16i - G_x}; k, q e^{G_x - G_16i+15}
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float kv = __uint_as_float((e & 1) ? (kk[e >> 1] & 0xffff0000u) : (kk[e >> 1] << 16));
        const float qv = __uint_as_float((e & 1) ? (qq[e >> 1] & 0xffff0000u) : (qq[e >> 1] << 16));
        const float up = __expf(fminf(gsv[e] - gxv[e], 80.f)), dn = __expf(fminf(gxv[e] - gev[e], 80.f));
        rk[e] = kv * up;
        ck[e] = kv * dn;
        cqv[e] = qv * dn;
      }
      auto put8 = [&](uint32_t off, const float (&v)[8], const float* f) {
        float y[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) y[e] = f ? v[e] * f[8 * c8 + e] : v[e];
        *reinterpret_cast<uint4*>(sm + off) =
            make_uint4(pack_bf16(y[0], y[1]), pack_bf16(y[2], y[3]), pack_bf16(y[4], y[5]),
                       pack_bf16(y[6], y[7]));
      };
#pragma unroll
      for (int a = 0; a < 4; ++a)              // row x of R^(a), a >= blk
        if (a >= blk)
          put8(G_RR + r_row(a) + io(x, 8 * c8, 16 * (a + 1)), rk,
               a == blk ? nullptr : F1 + (a * (a - 1) / 2 + blk) * D);
#pragma unroll
      for (int b = 0; b < 4; ++b)              // row x - 16 b of R'k^(b), R'q^(b), b <= blk
        if (b <= blk) {
          const float* f = b == blk ? nullptr : F2 + (blk * (blk - 1) / 2 + b) * D;
          const uint32_t o = r_col(b) + io(x - 16 * b, 8 * c8, 64 - 16 * b);
          put8(G_RK + o, ck, f);
          put8(G_RQ + o, cqv, f);
        }
    }
  }
  __syncthreads();
  // row side: [YA | YQ] = [dA | dAqk] R^(tb) for rows r0.. (times e^{G_r - G_16tb})
#pragma unroll
  for (int np = 0; np < 2; ++np) {
    float ya[2][4] = {}, yq[2][4] = {};
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
      if (ks > tb) continue;
      uint32_t aa[4], aq[4], b[4];
      a_mk(sb + G_DA, 64, r0, 16 * ks, lane, aa);
      a_mk(sb + G_AQK, 64, r0, 16 * ks, lane, aq);
      b_kn(sb + G_RR + (mid ? 0u : r_row(tb)), mid ? 64 : 16 * (tb + 1), c0 + 16 * np, 16 * ks,
           lane, b);
      mma(ya[0], aa, b[0], b[1]);
      mma(ya[1], aa, b[2], b[3]);
      mma(yq[0], aq, b[0], b[1]);
      mma(yq[1], aq, b[2], b[3]);
    }
#pragma unroll
    for (int sub = 0; sub < 2; ++sub) {
      const int nt = 2 * np + sub;
      const float2 gref = gam2(mid ? 32 : r0, nt);
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const float2 gp = gam2(r0 + g8 + 8 * hf, nt);
        const float2 kv = img2(G_K, hf, nt), qv = img2(G_Q, hf, nt);
        const float f0 = __expf(fminf(gp.x - gref.x, 80.f)), f1 = __expf(fminf(gp.y - gref.y, 80.f));
        const float yA0 = ya[sub][2 * hf] * f0, yA1 = ya[sub][2 * hf + 1] * f1;
        const float yQ0 = yq[sub][2 * hf] * f0, yQ1 = yq[sub][2 * hf + 1] * f1;
        dK[nt][2 * hf] += yA0;
        dK[nt][2 * hf + 1] += yA1;
        dQ[nt][2 * hf] += yQ0;
        dQ[nt][2 * hf + 1] += yQ1;
        dG[nt][2 * hf] += yA0 * kv.x + yQ0 * qv.x;
        dG[nt][2 * hf + 1] += yA1 * kv.y + yQ1 * qv.y;
      }
    }
  }
  // column side: Z = dA^T R'k^(tb) + dAqk^T R'q^(tb) for rows i = r0.. (times e^{G_16tb+15 - G_i})
#pragma unroll
  for (int np = 0; np < 2; ++np) {
    float z[2][4] = {};
#pragma unroll
    for (int rho = 0; rho < 4; ++rho) {
      if (rho < tb) continue;
      uint32_t aa[4], aq[4], bk[4], bq[4];
      a_km(sb + G_DA, 64, r0, 16 * rho, lane, aa);
      a_km(sb + G_AQK, 64, r0, 16 * rho, lane, aq);
      const uint32_t co = mid ? 0u : r_col(tb);
      const int crows = mid ? 64 : 64 - 16 * tb, ck0 = mid ? 16 * rho : 16 * (rho - tb);
      b_kn(sb + G_RK + co, crows, c0 + 16 * np, ck0, lane, bk);
      b_kn(sb + G_RQ + co, crows, c0 + 16 * np, ck0, lane, bq);
      mma(z[0], aa, bk[0], bk[1]);
      mma(z[1], aa, bk[2], bk[3]);
      mma(z[0], aq, bq[0], bq[1]);
      mma(z[1], aq, bq[2], bq[3]);
    }
#pragma unroll
    for (int sub = 0; sub < 2; ++sub) {
      const int nt = 2 * np + sub;
      const float2 gref = gam2(mid ? 32 : r0 + 15, nt);
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const float2 gp = gam2(r0 + g8 + 8 * hf, nt), kv = img2(G_K, hf, nt);
        const float z0 = z[sub][2 * hf] * __expf(fminf(gref.x - gp.x, 80.f));
        const float z1 = z[sub][2 * hf + 1] * __expf(fminf(gref.y - gp.y, 80.f));
        dK[nt][2 * hf] += z0;
        dK[nt][2 * hf + 1] += z1;
        dG[nt][2 * hf] -= z0 * kv.x;
        dG[nt][2 * hf + 1] -= z1 * kv.y;
      }
    }
  }
  if (fix) {
    // exact within-block pairs of unsafe (block, channel) pairs, by running products
    // of alpha_j = e^{g_j} (exponents from the block's own g, never from Gamma)
    auto qk = [&](uint32_t img, int r, int c) { return bf_at(sm + img + io(r, c, 64)); };
    __syncthreads();                    // R images no longer read
    float* cya = reinterpret_cast<float*>(sm + G_CYA);
    float* cyq = reinterpret_cast<float*>(sm + G_CYQ);
    float* cz = reinterpret_cast<float*>(sm + G_CZ);
    for (int i = tid; i < 3 * 64 * 128; i += NTG) cya[i] = 0.f;   // the three are contiguous
    __syncthreads();
    for (int item = tid; item < 4 * D; item += NTG) {
      const int a = item >> 7, c = item & 127;
      if (!s_uns[a][c]) continue;
      const int ra = 16 * a;
      float al[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const int r = ra + e;
        float gv = 0.f;
        if (r < L) gv = GRPD ? g[((rb + r) * H + h) * (D >> gsh) + (c >> gsh)]
                             : g[((rb + r) * H + h) * D + c];
        al[e] = __expf(gv);
      }
#pragma unroll 1
      for (int e = 0; e < 16; ++e) {        // row r = ra + e: pairs i <= r inside the block
        const int r = ra + e;
        float p = 1.f, ya = 0.f, yq = 0.f;
        const float kr = qk(G_K, r, c), qr = qk(G_Q, r, c);
#pragma unroll 1
        for (int f = e; f >= 0; --f) {     // i = ra + f; p = prod_{j=i+1..r} alpha_j
          const int i = ra + f;
          if (f < e) p *= al[f + 1];
          const float ki = qk(G_K, i, c);
          const float da = bf_at(sm + G_DA + io(r, i, 64));
          const float dq2 = bf_at(sm + G_AQK + io(r, i, 64));
          ya = fmaf(da * p, ki, ya);
          yq = fmaf(dq2 * p, ki, yq);
          // column side of pair (r, i): into row i's Z
          cz[i * 128 + c] += (da * kr + dq2 * qr) * p;
        }
        cya[r * 128 + c] = ya;
        cyq[r * 128 + c] = yq;
      }
    }
    __syncthreads();
#pragma unroll
    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int r = r0 + g8 + ((e >> 1) << 3), c = c0 + 8 * nt + 2 * qd + (e & 1);
        if (!s_uns[tb][c]) continue;
        const float yA = cya[r * 128 + c], yQ = cyq[r * 128 + c], zz = cz[r * 128 + c];
        const float kv = qk(G_K, r, c), qv = qk(G_Q, r, c);
        dK[nt][e] += yA + zz;
        dQ[nt][e] += yQ;
        dG[nt][e] += yA * kv + yQ * qv - zz * kv;
      }
  }

  // ---- phase 5: outputs.  dq and dk straight from the accumulators (each lane's pairs of
  // channels: eight rows of 32 contiguous bytes per store); dg = the reverse cumulative sum
  // of dGamma over the chunk's rows plus dGamma_last's state term: within the warp's 16 rows
  // by shuffles, across the four row blocks through the block totals.
  __syncthreads();                      // s_dgl and s_dbeta are complete; s_part is free
#pragma unroll
  for (int nt = 0; nt < 4; ++nt)
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      const int r = r0 + g8 + 8 * hf;
      {                                 // A_qk's diagonal: dq_r += dAqk_rr k_r, dk_r += dAqk_rr q_r
        const float dd = s_daqk[r];
        const float2 kv = img2(G_K, hf, nt), qv = img2(G_Q, hf, nt);
        dQ[nt][2 * hf] = fmaf(dd, kv.x, dQ[nt][2 * hf]);
        dQ[nt][2 * hf + 1] = fmaf(dd, kv.y, dQ[nt][2 * hf + 1]);
        dK[nt][2 * hf] = fmaf(dd, qv.x, dK[nt][2 * hf]);
        dK[nt][2 * hf + 1] = fmaf(dd, qv.y, dK[nt][2 * hf + 1]);
      }
      if (r < L) {
        const long long o = ((rb + r) * H + h) * D + c0 + 8 * nt + 2 * qd;
        *reinterpret_cast<float2*>(dq + o) = make_float2(dQ[nt][2 * hf], dQ[nt][2 * hf + 1]);
        *reinterpret_cast<float2*>(dk + o) = make_float2(dK[nt][2 * hf], dK[nt][2 * hf + 1]);
      }
    }
  // suffix sums over the rows g8 (+8) of each half (lanes 4 apart are adjacent rows)
#pragma unroll
  for (int nt = 0; nt < 4; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
#pragma unroll
      for (int s = 4; s < 32; s <<= 1) {
        const float y = __shfl_down_sync(0xffffffffu, dG[nt][e], s);
        if (lane + s < 32) dG[nt][e] += y;
      }
    }
  // the lower half (rows 8..15) adds to every row of the upper one; lanes 0..3 then hold
  // the block's totals
#pragma unroll
  for (int nt = 0; nt < 4; ++nt)
#pragma unroll
    for (int e1 = 0; e1 < 2; ++e1) {
      const float lower = __shfl_sync(0xffffffffu, dG[nt][2 + e1], qd);
      dG[nt][e1] += lower;
      if (g8 == 0) s_part[tb][c0 + 8 * nt + 2 * qd + e1] = dG[nt][e1];
    }
  __syncthreads();
#pragma unroll
  for (int nt = 0; nt < 4; ++nt)
#pragma unroll
    for (int e1 = 0; e1 < 2; ++e1) {
      const int c = c0 + 8 * nt + 2 * qd + e1;
      float add = s_dgl[c];
      for (int b2 = tb + 1; b2 < 4; ++b2) add += s_part[b2][c];
      dG[nt][e1] += add;
      dG[nt][2 + e1] += add;
    }
  if constexpr (!GRPD) {
#pragma unroll
    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const int r = r0 + g8 + 8 * hf;
        if (r < L)
          *reinterpret_cast<float2*>(dg + ((rb + r) * H + h) * D + c0 + 8 * nt + 2 * qd) =
              make_float2(dG[nt][2 * hf], dG[nt][2 * hf + 1]);
      }
  } else {
    // one decay per group of 1 << gsh channels: the group's sum, through shared memory
    float* dGs = reinterpret_cast<float*>(sm + G_S0);
#pragma unroll
    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
      for (int hf = 0; hf < 2; ++hf)
        *reinterpret_cast<float2*>(dGs + (r0 + g8 + 8 * hf) * LDG + c0 + 8 * nt + 2 * qd) =
            make_float2(dG[nt][2 * hf], dG[nt][2 * hf + 1]);
    __syncthreads();
    const int ng = D >> gsh, gs = 1 << gsh;
    for (int i = tid; i < C * ng; i += NTG) {
      const int r = i / ng, m = i % ng;
      if (r < L) {
        float acc = 0.f;
        for (int e = 0; e < gs; ++e) acc += dGs[r * LDG + m * gs + e];
        dg[((rb + r) * H + h) * ng + m] = acc;
      }
    }
  }
  if (tid < L) dbeta[(rb + tid) * H + h] = s_dbeta[tid];
}

constexpr int kChainF = 32, kChainR = 16;      // value columns per forward / reverse chain
constexpr uint32_t kChainSmem = Chain<kChainF>::SMEM > Chain<kChainR>::SMEM ? Chain<kChainF>::SMEM
                                                                          : Chain<kChainR>::SMEM;

bool set_attrs() {
  return once_per_device(kOnceBwdTc, []() {
    return cudaFuncSetAttribute(kda_bwd_chain_kernel<kChainF, kChainR>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                kChainSmem) == cudaSuccess &&
           cudaFuncSetAttribute(kda_bwd_grad_kernel<false>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, GRAD_SMEM) == cudaSuccess &&
           cudaFuncSetAttribute(kda_bwd_grad_kernel<true>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, GRAD_SMEM) == cudaSuccess;
  });
}

struct BwdTcScratch {
  long long nslots;
  size_t rec, simg, dlimg, dsimg, ddimg, ddlo, total;
};
BwdTcScratch bwd_tc_scratch(int B, int T, int H, bool varlen) {
  BwdTcScratch r{};
  r.nslots = chunk_slots(B, T, varlen);
  const size_t per = (size_t)r.nslots * H;
  r.rec = 0;
  r.simg = r.rec + per * rec::BYTES_BWD;
  r.dlimg = r.simg + per * kImgS;
  r.dsimg = r.dlimg + per * kImgD;
  r.ddimg = r.dsimg + per * kImgS;
  r.ddlo = r.ddimg + per * kImgD;
  r.total = r.ddlo + per * kImgD;
  return r;
}

}  // namespace

bool chunk_bwd_tc_supported(int dk, int dv, int in_dtype) {
  return in_dtype == KDA_BF16 && dk == D && dv == D;
}

size_t chunk_bwd_tc_scratch_bytes(int B, int T, int H, bool varlen) {
  return bwd_tc_scratch(B, T, H, varlen).total;
}

cudaError_t launch_chunk_bwd_tc(const void* q, const void* k, const void* v, const float* g,
                                const float* beta, const float* h0, const int32_t* cu_seqlens,
                                const void* dout, const float* dhT, float* dq, float* dk,
                                float* dv, float* dg, float* dbeta, float* dh0, int B, int T,
                                int H, int gsh, cudaStream_t stream, const Workspace* ws) {
  int sms = 148;
  cudaMemPool_t pool = nullptr;
  if (!device_ctx(&sms, ws ? nullptr : &pool) || !set_attrs()) return cudaErrorInvalidDevice;
  if (!ws && !pool) return cudaErrorMemoryAllocation;
  const bool varlen = cu_seqlens != nullptr;
  const BwdTcScratch sc = bwd_tc_scratch(B, T, H, varlen);
  void* scratch = nullptr;
  bool pooled = false;
  if (sc.total > 0) {
    if (ws) {
      if (!ws->ptr || ws->bytes < sc.total) return cudaErrorInvalidValue;
      scratch = ws->ptr;
    } else {
      const cudaError_t e = cudaMallocFromPoolAsync(&scratch, sc.total, pool, stream);
      if (e != cudaSuccess) return e;
      pooled = true;
    }
  }
  uint8_t* base = static_cast<uint8_t*>(scratch);
  uint8_t* rec = base + sc.rec;
  cudaError_t e = launch_chunk_prep_bwd(q, k, v, g, beta, cu_seqlens, rec, B, T, H, gsh,
                                        sc.nslots, stream);
  if (e == cudaSuccess) {
    KDA_TIMED(KDA_KERNEL_BWD_CHAIN, stream,
              e = launch_after(kda_bwd_chain_kernel<kChainF, kChainR>,
                               dim3(D / kChainF + D / kChainR, H, B), dim3(NTC), kChainSmem,
                               stream, rec, h0, cu_seqlens,
                               static_cast<const bf16*>(dout), dhT, dh0, base + sc.simg,
                               base + sc.dlimg, base + sc.dsimg, base + sc.ddimg,
                               base + sc.ddlo, T, H, sc.nslots));
    note_launches(1);
  }
  if (e == cudaSuccess && sc.nslots > 0) {
    auto grad = gsh != 0 ? kda_bwd_grad_kernel<true> : kda_bwd_grad_kernel<false>;
    KDA_TIMED(KDA_KERNEL_BWD_GRAD, stream,
              e = launch_after(grad, dim3((unsigned)sc.nslots, H), dim3(NTG), GRAD_SMEM, stream,
                               static_cast<const bf16*>(q), static_cast<const bf16*>(k),
                               static_cast<const bf16*>(v), g, beta,
                               static_cast<const bf16*>(dout), cu_seqlens,
                               static_cast<const uint8_t*>(rec), static_cast<const uint8_t*>(base + sc.simg),
                               static_cast<const uint8_t*>(base + sc.dlimg),
                               static_cast<const uint8_t*>(base + sc.dsimg),
                               static_cast<const uint8_t*>(base + sc.ddimg),
                               static_cast<const uint8_t*>(base + sc.ddlo), dq, dk, dv, dg,
                               dbeta, B, T, H, gsh, sc.nslots));
    note_launches(1);
  }
  if (pooled) cudaFreeAsync(scratch, stream);
  return e;
}

// Reads (and with reset clears) g_bwd_tc_timeout; host side of kda_device_status.
cudaError_t take_bwd_tc_timeout(int* flag, bool reset) {
  int v = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, g_bwd_tc_timeout, sizeof(int));
  if (e == cudaSuccess && reset && v != 0) {
    const int zero = 0;
    e = cudaMemcpyToSymbol(g_bwd_tc_timeout, &zero, sizeof(int));
  }
  *flag = v;
  return e;
}

}  // namespace kda
