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
// record images in bf16, plus T and A in fp32; chunk_split.cu):
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

cudaError_t launch_chunk_prep_bwd(const void* q, const void* k, const void* v, const float* g,
                                  const float* beta, const int32_t* cu_seqlens, uint8_t* rec,
                                  int B, int T, int H, int gsh, long long nslots,
                                  cudaStream_t stream);

namespace {
using namespace sm100;
using bf16 = __nv_bfloat16;

constexpr int C = kChunk;
constexpr int D = kHead;
constexpr int NTH = 256;
constexpr uint32_t kImgS = 32768;      // S / dS image per (chunk, head): [128 j][128 c] bf16
constexpr uint32_t kImgD = 16384;      // Delta / dDelta image: [64 t][128 j] bf16

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
// Chains.  CTA (x, h, s): x < NJB walks sequence s of head h forward for the
// value columns [NB x, NB x + NB); x >= NJB walks it backward for block x - NJB.
// Warp w keeps rows 16w .. 16w + 15 of the state (or of its gradient) for the
// block's columns as m16n8 accumulators: lane (g, qd) holds rows 16w + g (+8),
// columns 8 nt + 2 qd (+1).
// ============================================================================
template <int NB>
struct Chain {
  static constexpr int NJ = NB / 8;        // n8 tiles of the column block
  static constexpr int NJB = D / NB;       // column blocks per head
  static constexpr int STG = 3;            // record stages in flight
  // forward stage: W^T (16 KB), Kend^T (16 KB), U^T rows of the block, exp(Gamma_last)
  static constexpr uint32_t F_W = 0, F_K = 16384, F_U = 32768, F_DEC = F_U + NB * 128,
                            F_STAGE = F_DEC + 512;
  static constexpr uint32_t F_S = STG * F_STAGE;        // S tile [NB j][128 c]
  static constexpr uint32_t F_DL = F_S + NB * 256;      // Delta tile [64 t][NB j] (64-column panel)
  static constexpr uint32_t F_SMEM = F_DL + 8192;
  // reverse stage: [Qbar^T | W^T] (32 KB), [Kend^T ; Aqk] (24 KB), exp(Gamma_last), dO tile
  static constexpr uint32_t R_QW = 0, R_KA = 32768, R_DEC = 57344, R_DO = 57856,
                            R_STAGE = R_DO + 8192;
  static constexpr uint32_t R_Y = STG * R_STAGE;        // dS tile [NB j][128 c]
  static constexpr uint32_t R_DD = R_Y + NB * 256;      // -dDelta tile [64 t][NB j]
  static constexpr uint32_t R_SMEM = R_DD + 8192;
  static constexpr uint32_t SMEM = (F_SMEM > R_SMEM ? F_SMEM : R_SMEM) + 1024;
};

template <int NB>
__global__ void __launch_bounds__(NTH, 1)
kda_bwd_chain_kernel(const uint8_t* __restrict__ rec, const float* __restrict__ h0,
                     const int32_t* __restrict__ cu_seqlens, const bf16* __restrict__ dout,
                     const float* __restrict__ dhT, float* __restrict__ dh0,
                     uint8_t* __restrict__ simg, uint8_t* __restrict__ dlimg,
                     uint8_t* __restrict__ dsimg, uint8_t* __restrict__ ddimg, int T, int H,
                     long long nslots) {
  using CF = Chain<NB>;
  constexpr int NJ = CF::NJ, STG = CF::STG;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1024(smem_raw);
  const uint32_t sb = smem_u32(sm);
  const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31, g = lane >> 2, qd = lane & 3;
  const bool fwd = (int)blockIdx.x < CF::NJB;
  const int jb = fwd ? (int)blockIdx.x : (int)blockIdx.x - CF::NJB;
  const int j0 = jb * NB, h = blockIdx.y, s = blockIdx.z;
  long long row0, t_beg, t_end;
  seq_range(cu_seqlens, s, T, row0, t_beg, t_end);
  const int nch = (int)chunk_count(t_end - t_beg);
  const size_t base = (size_t)h * (size_t)nslots + (size_t)seq_chunk_base(cu_seqlens, s, T);
  const size_t st_off = ((size_t)s * H + h) * D * D;

  float X[NJ][4];
  {
    const float* init = fwd ? h0 : dhT;
#pragma unroll
    for (int nt = 0; nt < NJ; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int c = 16 * w + g + ((e >> 1) << 3), j = j0 + 8 * nt + 2 * qd + (e & 1);
        X[nt][e] = init ? init[st_off + (size_t)c * D + j] : 0.f;
      }
  }
  const int tb = w & 3, jh = w >> 2;       // Delta / dDelta tiles: token block, half of the n8 tiles
  constexpr int NH = NJ / 2;

  // the S (or dS) tile as bf16 [j][c], then copied out as rows j0.. of the chunk's image
  auto put_state = [&](uint32_t tile) {
#pragma unroll
    for (int p = 0; p < NH; ++p) st_nm(tile, NB, 16 * w, 16 * p, lane, X[2 * p], X[2 * p + 1], 1.f);
  };
  auto copy_state = [&](uint32_t tile_off, uint8_t* img) {
    for (int i = tid; i < NB * 16; i += NTH) {
      const int pnl = i / (NB * 8), rr = (i >> 3) % NB, ck = i & 7;
      *reinterpret_cast<uint4*>(img + pnl * 16384 + (j0 + rr) * 128 + ck * 16) =
          *reinterpret_cast<const uint4*>(sm + tile_off + pnl * NB * 128 + rr * 128 + ck * 16);
    }
  };

  if (fwd) {
    auto issue = [&](int n) {
      if (n < nch) {
        const uint8_t* rc = rec + (base + n) * rec::BYTES_BWD;
        uint8_t* st = sm + (n % STG) * CF::F_STAGE;
        constexpr int NP = 2048 + NB * 8 + 32;
        for (int i = tid; i < NP; i += NTH) {
          uint32_t d, o;
          if (i < 1024) { d = CF::F_W + 16 * i; o = rec::QW + 16384 + 16 * i; }
          else if (i < 2048) { d = CF::F_K + 16 * (i - 1024); o = rec::KA + 16 * (i - 1024); }
          else if (i < 2048 + NB * 8) { d = CF::F_U + 16 * (i - 2048); o = rec::U + j0 * 128 + 16 * (i - 2048); }
          else { d = CF::F_DEC + 16 * (i - 2048 - NB * 8); o = rec::DECAY + 16 * (i - 2048 - NB * 8); }
          cp_async16(st + d, rc + o, 16u);
        }
      }
      cp_async_commit();
    };
    const uint32_t uS = sb + CF::F_S, uDL = sb + CF::F_DL;
#pragma unroll 1
    for (int n = 0; n < STG - 1; ++n) issue(n);
#pragma unroll 1
    for (int n = 0; n < nch; ++n) {
      const uint32_t so = (uint32_t)(n % STG) * CF::F_STAGE;
      put_state(uS);                                   // S at the start of chunk n
      cp_async_wait_group<STG - 2>();
      __syncthreads();
      issue(n + STG - 1);
      copy_state(CF::F_S, simg + (base + n) * kImgS);
      // Delta = U - W S: token block tb, n8 tiles jh * NH ..
      float acc[NH][4];
#pragma unroll
      for (int p = 0; p < NH; ++p)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[p][e] = 0.f;
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        uint32_t a[4];
        a_km(sb + so + CF::F_W, 128, 16 * tb, 16 * ks, lane, a);      // W [t][c] from W^T
#pragma unroll
        for (int p = 0; p < NH; ++p) {
          uint32_t b[2];
          b_nk1(uS, NB, 8 * (jh * NH + p), 16 * ks, lane, b);           // S [c][j] from [j][c]
          mma(acc[p], a, b[0], b[1]);
        }
      }
      uint8_t* gD = dlimg + (base + n) * kImgD;
#pragma unroll
      for (int p = 0; p < NH; ++p) {
        const int n0 = 8 * (jh * NH + p), jl = n0 + 2 * qd;
        float dl[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int t = 16 * tb + g + ((e >> 1) << 3);
          dl[e] = bf_at(sm + so + CF::F_U + io(jl + (e & 1), t, NB)) - acc[p][e];
        }
        st_mn1(uDL, 64, 16 * tb, n0, lane, dl, 1.f);
#pragma unroll
        for (int hf = 0; hf < 2; ++hf)
          *reinterpret_cast<uint32_t*>(gD + io(16 * tb + g + 8 * hf, j0 + jl, 64)) =
              pack_bf16(dl[2 * hf], dl[2 * hf + 1]);
      }
      __syncthreads();
      // S <- Diag(exp(Gamma_last)) S + Kend^T Delta
      const float* dec = reinterpret_cast<const float*>(sm + so + CF::F_DEC);
      const float d0 = dec[16 * w + g], d1 = dec[16 * w + g + 8];
#pragma unroll
      for (int nt = 0; nt < NJ; ++nt) {
        X[nt][0] *= d0; X[nt][1] *= d0; X[nt][2] *= d1; X[nt][3] *= d1;
      }
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        uint32_t a[4];
        a_mk(sb + so + CF::F_K, 128, 16 * w, 16 * ks, lane, a);       // Kend^T [c][t]
#pragma unroll
        for (int p = 0; p < NH; ++p) {
          uint32_t b[4];
          b_kn(uDL, 64, 16 * p, 16 * ks, lane, b);                    // Delta [t][j]
          mma(X[2 * p], a, b[0], b[1]);
          mma(X[2 * p + 1], a, b[2], b[3]);
        }
      }
    }
    cp_async_wait_all();
    return;
  }

  // ---- reverse chain
  auto issue = [&](int n) {
    if (n >= 0) {
      const uint8_t* rc = rec + (base + n) * rec::BYTES_BWD;
      uint8_t* st = sm + (n % STG) * CF::R_STAGE;
      const long long t0 = t_beg + (long long)n * C;
      const int L = (int)min((long long)C, t_end - t0);
      constexpr int NP = 2048 + 1536 + 32 + 64 * NJ;
      for (int i = tid; i < NP; i += NTH) {
        if (i < 2048) {
          cp_async16(st + CF::R_QW + 16 * i, rc + rec::QW + 16 * i, 16u);
        } else if (i < 3584) {
          cp_async16(st + CF::R_KA + 16 * (i - 2048), rc + rec::KA + 16 * (i - 2048), 16u);
        } else if (i < 3616) {
          cp_async16(st + CF::R_DEC + 16 * (i - 3584), rc + rec::DECAY + 16 * (i - 3584), 16u);
        } else {
          const int kk = i - 3616, t = kk / NJ, ck = kk % NJ;
          const bf16* src = dout + ((row0 + t0 + min(t, L - 1)) * H + h) * D + j0 + 8 * ck;
          cp_async16(st + CF::R_DO + io(t, 8 * ck, 64), src, t < L ? 16u : 0u);
        }
      }
    }
    cp_async_commit();
  };
  const uint32_t uY = sb + CF::R_Y, uDD = sb + CF::R_DD;
#pragma unroll 1
  for (int i = 0; i < STG - 1; ++i) issue(nch - 1 - i);
#pragma unroll 1
  for (int n = nch - 1; n >= 0; --n) {
    const uint32_t so = (uint32_t)(n % STG) * CF::R_STAGE;
    put_state(uY);                                       // dS after chunk n
    cp_async_wait_group<STG - 2>();
    __syncthreads();
    issue(n - (STG - 1));
    copy_state(CF::R_Y, dsimg + (base + n) * kImgS);
    // dDelta = Kend dS + Aqk^T dO
    float acc[NH][4];
#pragma unroll
    for (int p = 0; p < NH; ++p)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[p][e] = 0.f;
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      uint32_t a[4];
      a_km(sb + so + CF::R_KA, 128, 16 * tb, 16 * ks, lane, a);          // Kend [t][c] from Kend^T
#pragma unroll
      for (int p = 0; p < NH; ++p) {
        uint32_t b[2];
        b_nk1(uY, NB, 8 * (jh * NH + p), 16 * ks, lane, b);               // dS [c][j] from [j][c]
        mma(acc[p], a, b[0], b[1]);
      }
    }
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
      uint32_t a[4];
      a_km(sb + so + CF::R_KA + 16384, 64, 16 * tb, 16 * ks, lane, a);   // Aqk^T [t][r] from Aqk
#pragma unroll
      for (int p = 0; p < NH; ++p) {
        uint32_t b[2];
        b_kn1(sb + so + CF::R_DO, 64, 8 * (jh * NH + p), 16 * ks, lane, b);   // dO [r][j]
        mma(acc[p], a, b[0], b[1]);
      }
    }
    uint8_t* gD = ddimg + (base + n) * kImgD;
#pragma unroll
    for (int p = 0; p < NH; ++p) {
      const int n0 = 8 * (jh * NH + p), jl = n0 + 2 * qd;
      st_mn1(uDD, 64, 16 * tb, n0, lane, acc[p], -1.f);
#pragma unroll
      for (int hf = 0; hf < 2; ++hf)
        *reinterpret_cast<uint32_t*>(gD + io(16 * tb + g + 8 * hf, j0 + jl, 64)) =
            pack_bf16(acc[p][2 * hf], acc[p][2 * hf + 1]);
    }
    __syncthreads();
    // dS <- Diag(exp(Gamma_last)) dS + Qbar^T dO - W^T dDelta
    const float* dec = reinterpret_cast<const float*>(sm + so + CF::R_DEC);
    const float d0 = dec[16 * w + g], d1 = dec[16 * w + g + 8];
#pragma unroll
    for (int nt = 0; nt < NJ; ++nt) {
      X[nt][0] *= d0; X[nt][1] *= d0; X[nt][2] *= d1; X[nt][3] *= d1;
    }
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
      uint32_t a[4], a2[4];
      a_mk(sb + so + CF::R_QW, 128, 16 * w, 16 * ks, lane, a);            // Qbar^T [c][t]
      a_mk(sb + so + CF::R_QW + 16384, 128, 16 * w, 16 * ks, lane, a2);   // W^T [c][t]
#pragma unroll
      for (int p = 0; p < NH; ++p) {
        uint32_t b[4], b2[4];
        b_kn(sb + so + CF::R_DO, 64, 16 * p, 16 * ks, lane, b);           // dO [t][j]
        b_kn(uDD, 64, 16 * p, 16 * ks, lane, b2);                         // -dDelta [t][j]
        mma(X[2 * p], a, b[0], b[1]);
        mma(X[2 * p + 1], a, b[2], b[3]);
        mma(X[2 * p], a2, b2[0], b2[1]);
        mma(X[2 * p + 1], a2, b2[2], b2[3]);
      }
    }
  }
  cp_async_wait_all();
  if (dh0) {
#pragma unroll
    for (int nt = 0; nt < NJ; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int c = 16 * w + g + ((e >> 1) << 3), j = j0 + 8 * nt + 2 * qd + (e & 1);
        dh0[st_off + (size_t)c * D + j] = X[nt][e];
      }
  }
}

// ============================================================================
// Gradient kernel: one CTA per (chunk slot, head), 8 warps.  Warp w owns token
// rows r0 = 16 tb .. r0 + 15 (tb = w % 4: one decay block) and channels
// c0 = 64 ch .. c0 + 63 (ch = w / 4) of dq, dk and dGamma in registers: lane
// (g, qd) holds rows r0 + g + 8 hf (hf = 0, 1) and channels c0 + 8 nt + 2 qd + e1
// (nt = 0..7, e1 = 0, 1), element [nt][2 hf + e1] -- the m16n8 accumulator layout.
// ============================================================================
constexpr int LDG = 136;                       // Gamma / dGamma row stride (floats)
constexpr uint32_t G_Q = 0;                    // q image [t][c]
constexpr uint32_t G_K = 16384;                // k image [t][c]
constexpr uint32_t G_G = 32768;                // Gamma fp32 [64][LDG]
constexpr uint32_t G_S0 = 67584;               // S image [j][c]  | T, A fp32 [64][64] | R images
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
// exact within-block corrections of unsafe channels (phase 4, after the products):
// fp32 [64][128] each
constexpr uint32_t G_CYA = G_S0, G_CYQ = G_S0 + 32768, G_CZ = G_S0 + 65536;

template <bool GRPD>
__global__ void __launch_bounds__(NTH, 1)
kda_bwd_grad_kernel(const bf16* __restrict__ q, const bf16* __restrict__ k,
                    const bf16* __restrict__ v, const float* __restrict__ g,
                    const float* __restrict__ beta, const bf16* __restrict__ dout,
                    const int32_t* __restrict__ cu_seqlens, const uint8_t* __restrict__ rec,
                    const uint8_t* __restrict__ simg, const uint8_t* __restrict__ dlimg,
                    const uint8_t* __restrict__ dsimg, const uint8_t* __restrict__ ddimg,
                    float* __restrict__ dq, float* __restrict__ dk, float* __restrict__ dv,
                    float* __restrict__ dg, float* __restrict__ dbeta, int B, int T, int H,
                    int gsh, long long nslots) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1024(smem_raw);
  const uint32_t sb = smem_u32(sm);
  __shared__ float s_beta[C], s_dbeta[C], s_dgl[D], s_half[D];
  __shared__ uint8_t s_uns[4][D];

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

  // ---- phase 0: loads
  for (int i = tid; i < 2048; i += NTH) {
    cp_async16(sm + G_S0 + 16 * i, simg + ix * kImgS + 16 * i, 16u);
    cp_async16(sm + G_DS + 16 * i, dsimg + ix * kImgS + 16 * i, 16u);
  }
  for (int i = tid; i < 1024; i += NTH) {
    cp_async16(sm + G_DL + 16 * i, dlimg + ix * kImgD + 16 * i, 16u);
    cp_async16(sm + G_DD + 16 * i, ddimg + ix * kImgD + 16 * i, 16u);
    const int t = i >> 4, c8 = i & 15;
    const long long src = ((rb + min(t, L - 1)) * H + h) * D + 8 * c8;
    const uint32_t ok = t < L ? 16u : 0u;
    cp_async16(sm + G_DO + io(t, 8 * c8, 64), dout + src, ok);
    cp_async16(sm + G_Q + io(t, 8 * c8, 64), q + src, ok);
    cp_async16(sm + G_K + io(t, 8 * c8, 64), k + src, ok);
  }
  if constexpr (!GRPD) {
    for (int i = tid; i < 2048; i += NTH) {
      const int t = i >> 5, c4 = i & 31;
      cp_async16(G + t * LDG + 4 * c4, g + ((rb + min(t, L - 1)) * H + h) * D + 4 * c4,
                 t < L ? 16u : 0u);
    }
  }
  cp_async_commit();
  if (tid < C) {
    s_beta[tid] = tid < L ? beta[(rb + tid) * H + h] : 0.f;
    s_dbeta[tid] = 0.f;
  }
  if (tid < D) s_dgl[tid] = 0.f;
  if constexpr (GRPD) {
    const int ng = D >> gsh;
    for (int i = tid; i < C * D; i += NTH) {
      const int t = i >> 7, c = i & 127;
      G[t * LDG + c] = t < L ? g[((rb + t) * H + h) * ng + (c >> gsh)] : 0.f;
    }
  }
  cp_async_wait_all();
  __syncthreads();
  // Gamma = cumsum g per channel: two threads per channel, 32 rows each
  {
    const int c = tid & 127, part = tid >> 7;
    float x[32];
#pragma unroll
    for (int e = 0; e < 32; ++e) x[e] = G[(32 * part + e) * LDG + c];
#pragma unroll
    for (int e = 1; e < 32; ++e) x[e] += x[e - 1];
    if (part == 0) s_half[c] = x[31];
    __syncthreads();
    const float add = part ? s_half[c] : 0.f;
#pragma unroll
    for (int e = 0; e < 32; ++e) G[(32 * part + e) * LDG + c] = x[e] + add;
  }
  __syncthreads();
  // unsafe (block, channel) pairs; and dGamma_last's state term e^Gamma_last sum_j S dS
  bool any_uns = false;
  {
    const int c = tid & 127, part = tid >> 7;
#pragma unroll
    for (int a2 = 0; a2 < 2; ++a2) {
      const int a = 2 * part + a2;
      const bool u = G[16 * a * LDG + c] - G[(16 * a + 15) * LDG + c] > kUnsafeDecay;
      s_uns[a][c] = u ? 1 : 0;
      any_uns |= u;
    }
    float acc = 0.f;
#pragma unroll 8
    for (int j = 64 * part; j < 64 * part + 64; ++j)
      acc = fmaf(bf_at(sm + G_S0 + io(j, c, 128)), bf_at(sm + G_DS + io(j, c, 128)), acc);
    atomicAdd(&s_dgl[c], acc * __expf(G[63 * LDG + c]));
  }
  const bool fix = __syncthreads_or(any_uns) != 0;

  const int tb = w & 3, ch = w >> 2, r0 = 16 * tb, c0 = 64 * ch;
  float dQ[8][4], dK[8][4], dG[8][4];
#pragma unroll
  for (int nt = 0; nt < 8; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) dQ[nt][e] = dK[nt][e] = dG[nt][e] = 0.f;
  // element helpers: row, column of accumulator element e of n8 tile nt (this warp's tile)
  auto erow = [&](int e) { return r0 + g8 + ((e >> 1) << 3); };
  auto ecol = [&](int nt, int e) { return c0 + 8 * nt + 2 * qd + (e & 1); };
  auto qk = [&](uint32_t img, int r, int c) { return bf_at(sm + img + io(r, c, 64)); };

  // ---- phase 1: dQbar and dW (against S^T), dKend (dS^T), dAqk
#pragma unroll
  for (int np = 0; np < 4; ++np) {
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
      for (int e = 0; e < 4; ++e) {
        const int r = erow(e), c = ecol(nt, e);
        const float eg = __expf(G[r * LDG + c]);
        dQ[nt][e] = fmaf(aq[sub][e], eg, dQ[nt][e]);
        dG[nt][e] = fmaf(aq[sub][e] * qk(G_Q, r, c), eg, dG[nt][e]);
      }
    }
    st_mn(sb + G_DW, 64, r0, c0 + 16 * np, lane, aw[0], aw[1], -1.f);   // dW = -dDelta S^T
  }
  __syncthreads();                      // S image no longer read: T and A go there
  for (int i = tid; i < 2048; i += NTH) cp_async16(sm + G_S0 + 16 * i, rc + rec::TMAT + 16 * i, 16u);
  cp_async_commit();
#pragma unroll
  for (int np = 0; np < 4; ++np) {
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
      float cs[2] = {0.f, 0.f};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int r = erow(e), c = ecol(nt, e);
        const float ee = __expf(G[63 * LDG + c] - G[r * LDG + c]);
        dK[nt][e] = fmaf(ak[sub][e], ee, dK[nt][e]);
        const float tk = ak[sub][e] * qk(G_K, r, c) * ee;
        dG[nt][e] -= tk;
        cs[e & 1] += tk;
      }
#pragma unroll
      for (int e1 = 0; e1 < 2; ++e1) {
        float x = cs[e1];
        x += __shfl_xor_sync(0xffffffffu, x, 4);
        x += __shfl_xor_sync(0xffffffffu, x, 8);
        x += __shfl_xor_sync(0xffffffffu, x, 16);
        if (g8 == 0) atomicAdd(&s_dgl[c0 + 8 * nt + 2 * qd + e1], x);
      }
    }
  }
  {   // dAqk (rows r0.., columns 32 ch ..), lower triangle
    const bool live = ch == 0 || tb >= 2;
#pragma unroll
    for (int np = 0; np < 2; ++np) {
      float aa[2][4] = {};
      if (live) {
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          uint32_t a[4], b[4];
          a_mk(sb + G_DO, 64, r0, 16 * ks, lane, a);
          b_nk(sb + G_DL, 64, 32 * ch + 16 * np, 16 * ks, lane, b);   // Delta^T from Delta [i][j]
          mma(aa[0], a, b[0], b[1]);
          mma(aa[1], a, b[2], b[3]);
        }
#pragma unroll
        for (int sub = 0; sub < 2; ++sub)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int r = erow(e), i = 32 * ch + 16 * np + 8 * sub + 2 * qd + (e & 1);
            if (i > r) aa[sub][e] = 0.f;
          }
      }
      st_mn(sb + G_AQK, 64, r0, 32 * ch + 16 * np, lane, aa[0], aa[1], 1.f);
    }
  }
  __syncthreads();                      // dO, Delta, dS no longer read
  for (int i = tid; i < 1024; i += NTH) {
    const int t = i >> 4, c8 = i & 15;
    cp_async16(sm + G_DO + io(t, 8 * c8, 64), v + ((rb + min(t, L - 1)) * H + h) * D + 8 * c8,
               t < L ? 16u : 0u);
  }
  cp_async_commit();
  // Kb = diag(beta) Kbar = beta k e^Gamma (image [i][c] at G_DS)
  for (int i = tid; i < 1024; i += NTH) {
    const int t = i >> 4, c8 = i & 15;
    const float bt = s_beta[t];
    float x[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int c = 8 * c8 + e;
      x[e] = bt * qk(G_K, t, c) * __expf(G[t * LDG + c]);
    }
    *reinterpret_cast<uint4*>(sm + G_DS + io(t, 8 * c8, 64)) =
        make_uint4(pack_bf16(x[0], x[1]), pack_bf16(x[2], x[3]), pack_bf16(x[4], x[5]),
                   pack_bf16(x[6], x[7]));
  }
  cp_async_wait_all();
  __syncthreads();
  const float* Tm = reinterpret_cast<const float*>(sm + G_S0);           // T [r][i]
  const float* Am = reinterpret_cast<const float*>(sm + G_S0 + 16384);   // A [r][i]
  // T image (bf16 [r][i] at G_DL) and Vb = diag(beta) V (image [i][j] at G_DS + 16384)
  for (int i = tid; i < 1536; i += NTH) {
    float x[8];
    if (i < 512) {
      const int r = i >> 3, c8 = i & 7;
#pragma unroll
      for (int e = 0; e < 8; ++e) x[e] = Tm[r * 64 + 8 * c8 + e];
      *reinterpret_cast<uint4*>(sm + G_DL + io(r, 8 * c8, 64)) =
          make_uint4(pack_bf16(x[0], x[1]), pack_bf16(x[2], x[3]), pack_bf16(x[4], x[5]),
                     pack_bf16(x[6], x[7]));
    } else {
      const int t = (i - 512) >> 4, c8 = (i - 512) & 15;
      const float bt = s_beta[t];
#pragma unroll
      for (int e = 0; e < 8; ++e) x[e] = bt * qk(G_DO, t, 8 * c8 + e);
      *reinterpret_cast<uint4*>(sm + G_DS + 16384 + io(t, 8 * c8, 64)) =
          make_uint4(pack_bf16(x[0], x[1]), pack_bf16(x[2], x[3]), pack_bf16(x[4], x[5]),
                     pack_bf16(x[6], x[7]));
    }
  }
  __syncthreads();

  // ---- phase 2: [dVb | dKb] = T^T [dDelta | dW] for token rows i in block tb
  {
    float dbp[2] = {0.f, 0.f};                 // dbeta parts of rows r0 + g8 (+8)
#pragma unroll
    for (int np = 0; np < 4; ++np) {
      float av[2][4] = {}, ak[2][4] = {};
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        if (ks < tb) continue;                 // T[r][i] = 0 for r < i
        uint32_t a[4], bv[4], bk[4];
        a_km(sb + G_DL, 64, r0, 16 * ks, lane, a);                  // T^T [i][r] from T [r][i]
        b_kn(sb + G_DD, 64, c0 + 16 * np, 16 * ks, lane, bv);      // dDelta [r][j]
        b_kn(sb + G_DW, 64, c0 + 16 * np, 16 * ks, lane, bk);      // dW [r][c]
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
          const float2 vv = bf2_at(sm + G_DO + io(i, c, 64));
          const float x0 = av[sub][2 * hf], x1 = av[sub][2 * hf + 1];
          if (i < L)
            *reinterpret_cast<float2*>(dv + ((rb + i) * H + h) * D + c) =
                make_float2(bi * x0, bi * x1);
          dbp[hf] += x0 * vv.x + x1 * vv.y;
#pragma unroll
          for (int e1 = 0; e1 < 2; ++e1) {
            const int e = 2 * hf + e1;
            const float eg = __expf(G[i * LDG + c + e1]);
            const float kb = qk(G_K, i, c + e1) * eg;          // Kbar
            const float y = ak[sub][e];
            dK[nt][e] = fmaf(bi * y, eg, dK[nt][e]);
            dG[nt][e] = fmaf(bi * y, kb, dG[nt][e]);
            dbp[hf] = fmaf(y, kb, dbp[hf]);
          }
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
  __syncthreads();                      // V and the T image no longer read

  // ---- phase 3: dT = dDelta Vb^T + dW Kb^T (strictly lower part), stored as dT^T
  float* dTt = reinterpret_cast<float*>(sm + G_DO);    // [i][r], stride 68
  if (ch == 0 || tb >= 2) {
#pragma unroll
    for (int np = 0; np < 2; ++np) {
      float at[2][4] = {};
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        uint32_t a[4], b[4];
        a_mk(sb + G_DD, 64, r0, 16 * ks, lane, a);
        b_nk(sb + G_DS + 16384, 64, 32 * ch + 16 * np, 16 * ks, lane, b);   // Vb^T from Vb [i][j]
        mma(at[0], a, b[0], b[1]);
        mma(at[1], a, b[2], b[3]);
      }
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        uint32_t a[4], b[4];
        a_mk(sb + G_DW, 64, r0, 16 * ks, lane, a);
        b_nk(sb + G_DS, 64, 32 * ch + 16 * np, 16 * ks, lane, b);           // Kb^T from Kb [i][c]
        mma(at[0], a, b[0], b[1]);
        mma(at[1], a, b[2], b[3]);
      }
#pragma unroll
      for (int sub = 0; sub < 2; ++sub)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int r = erow(e), i = 32 * ch + 16 * np + 8 * sub + 2 * qd + (e & 1);
          dTt[i * 68 + r] = at[sub][e];
        }
    }
  }
  __syncthreads();                      // dDelta, dW, Kb, Vb no longer read
  float* Tt = reinterpret_cast<float*>(sm + G_DD);     // T^T [i][b], stride 68
  for (int i = tid; i < 4096; i += NTH) {
    const int b = i >> 6, ii = i & 63;
    Tt[ii * 68 + b] = Tm[b * 64 + ii];
  }
  __syncthreads();
  // X[r][b] = sum_i dT[r][i] T[b][i] (needed for r > b; i <= b < r) -> G_DS, stride 68
  float* Xm = reinterpret_cast<float*>(sm + G_DS);
  {
    const int rt = tid >> 4, bt = tid & 15;
    float acc[4][4] = {};
    if (rt >= bt) {
#pragma unroll 4
      for (int i = 0; i < 4 * bt + 4; ++i) {
        const float4 x4 = *reinterpret_cast<const float4*>(dTt + i * 68 + 4 * rt);
        const float4 t4 = *reinterpret_cast<const float4*>(Tt + i * 68 + 4 * bt);
        const float xv[4] = {x4.x, x4.y, x4.z, x4.w}, tv[4] = {t4.x, t4.y, t4.z, t4.w};
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
          for (int b = 0; b < 4; ++b) acc[a][b] = fmaf(xv[a], tv[b], acc[a][b]);
      }
    }
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      float4 o;
      o.x = (4 * rt + a > 4 * bt + 0) ? acc[a][0] : 0.f;
      o.y = (4 * rt + a > 4 * bt + 1) ? acc[a][1] : 0.f;
      o.z = (4 * rt + a > 4 * bt + 2) ? acc[a][2] : 0.f;
      o.w = (4 * rt + a > 4 * bt + 3) ? acc[a][3] : 0.f;
      *reinterpret_cast<float4*>(Xm + (4 * rt + a) * 68 + 4 * bt) = o;
    }
  }
  __syncthreads();
  // dM[a][b] = -sum_{r >= a} T[r][a] X[r][b] (a > b); dA = diag(beta) dM (image);
  // dbeta_a += sum_b dM[a][b] A[a][b]
  {
    const int at = tid >> 4, bt = tid & 15;
    float acc[4][4] = {};
    if (at >= bt) {
#pragma unroll 4
      for (int r = 4 * at; r < 64; ++r) {
        const float4 t4 = *reinterpret_cast<const float4*>(Tm + r * 64 + 4 * at);
        const float4 x4 = *reinterpret_cast<const float4*>(Xm + r * 68 + 4 * bt);
        const float tv[4] = {t4.x, t4.y, t4.z, t4.w}, xv[4] = {x4.x, x4.y, x4.z, x4.w};
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
          for (int b = 0; b < 4; ++b) acc[a][b] = fmaf(tv[a], xv[b], acc[a][b]);
      }
    }
    float dbp[4];
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      const int ra = 4 * at + a;
      const float ba = s_beta[ra];
      float m[4];
      dbp[a] = 0.f;
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        m[b] = (ra > 4 * bt + b) ? -acc[a][b] : 0.f;
        dbp[a] = fmaf(m[b], Am[ra * 64 + 4 * bt + b], dbp[a]);
      }
      *reinterpret_cast<uint2*>(sm + G_DA + io(ra, 4 * bt, 64)) =
          make_uint2(pack_bf16(ba * m[0], ba * m[1]), pack_bf16(ba * m[2], ba * m[3]));
    }
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      float x = dbp[a];
      x += __shfl_xor_sync(0xffffffffu, x, 1);
      x += __shfl_xor_sync(0xffffffffu, x, 2);
      x += __shfl_xor_sync(0xffffffffu, x, 4);
      x += __shfl_xor_sync(0xffffffffu, x, 8);
      if (bt == 0) atomicAdd(&s_dbeta[4 * at + a], x);
    }
  }
  __syncthreads();                      // T, A, X, dT^T no longer read

  // ---- phase 4: the decay-weighted Gram products
  // R^(a)[i][c] = k_ic e^{G_16a,c - G_ic}, i < 16(a+1) (block a's own rows zero where
  // unsafe); R'x^(b)[r - 16b][c] = x_rc e^{G_rc - G_16b+15,c}, r >= 16b (likewise)
  for (int i = tid; i < 160 * 16; i += NTH) {
    const int row = i >> 4, c8 = i & 15;
    int a = 0;
    while (row >= (a + 1) * (a + 2) * 8) ++a;         // rows of R^(0..3): 16, 32, 48, 64
    const int ii = row - a * (a + 1) * 8;
    float x[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int c = 8 * c8 + e;
      const bool zero = ii >= 16 * a && s_uns[a][c];
      const float ex = fminf(G[16 * a * LDG + c] - G[ii * LDG + c], 80.f);
      x[e] = zero ? 0.f : qk(G_K, ii, c) * __expf(ex);
    }
    *reinterpret_cast<uint4*>(sm + G_RR + r_row(a) + io(ii, 8 * c8, 16 * (a + 1))) =
        make_uint4(pack_bf16(x[0], x[1]), pack_bf16(x[2], x[3]), pack_bf16(x[4], x[5]),
                   pack_bf16(x[6], x[7]));
  }
  for (int i = tid; i < 160 * 16; i += NTH) {
    const int row = i >> 4, c8 = i & 15;
    int b = 0, acc_rows = 0;
    while (row >= acc_rows + (64 - 16 * b)) { acc_rows += 64 - 16 * b; ++b; }
    const int rr = row - acc_rows, r = 16 * b + rr, nrows = 64 - 16 * b;
    float xk[8], xq[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int c = 8 * c8 + e;
      const bool zero = rr < 16 && s_uns[b][c];
      const float f = __expf(fminf(G[r * LDG + c] - G[(16 * b + 15) * LDG + c], 80.f));
      xk[e] = zero ? 0.f : qk(G_K, r, c) * f;
      xq[e] = zero ? 0.f : qk(G_Q, r, c) * f;
    }
    *reinterpret_cast<uint4*>(sm + G_RK + r_col(b) + io(rr, 8 * c8, nrows)) =
        make_uint4(pack_bf16(xk[0], xk[1]), pack_bf16(xk[2], xk[3]), pack_bf16(xk[4], xk[5]),
                   pack_bf16(xk[6], xk[7]));
    *reinterpret_cast<uint4*>(sm + G_RQ + r_col(b) + io(rr, 8 * c8, nrows)) =
        make_uint4(pack_bf16(xq[0], xq[1]), pack_bf16(xq[2], xq[3]), pack_bf16(xq[4], xq[5]),
                   pack_bf16(xq[6], xq[7]));
  }
  __syncthreads();
  // row side: [YA | YQ] = [dA | dAqk] R^(tb) for rows r0.. (times e^{G_r - G_16tb})
#pragma unroll
  for (int np = 0; np < 4; ++np) {
    float ya[2][4] = {}, yq[2][4] = {};
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
      if (ks > tb) continue;
      uint32_t aa[4], aq[4], b[4];
      a_mk(sb + G_DA, 64, r0, 16 * ks, lane, aa);
      a_mk(sb + G_AQK, 64, r0, 16 * ks, lane, aq);
      b_kn(sb + G_RR + r_row(tb), 16 * (tb + 1), c0 + 16 * np, 16 * ks, lane, b);
      mma(ya[0], aa, b[0], b[1]);
      mma(ya[1], aa, b[2], b[3]);
      mma(yq[0], aq, b[0], b[1]);
      mma(yq[1], aq, b[2], b[3]);
    }
#pragma unroll
    for (int sub = 0; sub < 2; ++sub) {
      const int nt = 2 * np + sub;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int r = erow(e), c = ecol(nt, e);
        const float f = __expf(fminf(G[r * LDG + c] - G[r0 * LDG + c], 80.f));
        const float yA = ya[sub][e] * f, yQ = yq[sub][e] * f;
        dK[nt][e] += yA;
        dQ[nt][e] += yQ;
        dG[nt][e] += yA * qk(G_K, r, c) + yQ * qk(G_Q, r, c);
      }
    }
  }
  // column side: Z = dA^T R'k^(tb) + dAqk^T R'q^(tb) for rows i = r0.. (times e^{G_16tb+15 - G_i})
#pragma unroll
  for (int np = 0; np < 4; ++np) {
    float z[2][4] = {};
#pragma unroll
    for (int rho = 0; rho < 4; ++rho) {
      if (rho < tb) continue;
      uint32_t aa[4], aq[4], bk[4], bq[4];
      a_km(sb + G_DA, 64, r0, 16 * rho, lane, aa);
      a_km(sb + G_AQK, 64, r0, 16 * rho, lane, aq);
      b_kn(sb + G_RK + r_col(tb), 64 - 16 * tb, c0 + 16 * np, 16 * (rho - tb), lane, bk);
      b_kn(sb + G_RQ + r_col(tb), 64 - 16 * tb, c0 + 16 * np, 16 * (rho - tb), lane, bq);
      mma(z[0], aa, bk[0], bk[1]);
      mma(z[1], aa, bk[2], bk[3]);
      mma(z[0], aq, bq[0], bq[1]);
      mma(z[1], aq, bq[2], bq[3]);
    }
#pragma unroll
    for (int sub = 0; sub < 2; ++sub) {
      const int nt = 2 * np + sub;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int r = erow(e), c = ecol(nt, e);
        const float f = __expf(fminf(G[(r0 + 15) * LDG + c] - G[r * LDG + c], 80.f));
        const float zz = z[sub][e] * f;
        dK[nt][e] += zz;
        dG[nt][e] -= zz * qk(G_K, r, c);
      }
    }
  }
  if (fix) {
    // exact within-block pairs of unsafe (block, channel) pairs, by running products
    // of alpha_j = e^{g_j} (exponents from the block's own g, never from Gamma)
    __syncthreads();                    // R images no longer read
    float* cya = reinterpret_cast<float*>(sm + G_CYA);
    float* cyq = reinterpret_cast<float*>(sm + G_CYQ);
    float* cz = reinterpret_cast<float*>(sm + G_CZ);
    for (int i = tid; i < 3 * 64 * 128; i += NTH) cya[i] = 0.f;   // the three are contiguous
    __syncthreads();
    for (int item = tid; item < 4 * D; item += NTH) {
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
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int r = erow(e), c = ecol(nt, e);
        if (!s_uns[tb][c]) continue;
        const float yA = cya[r * 128 + c], yQ = cyq[r * 128 + c], zz = cz[r * 128 + c];
        const float kv = qk(G_K, r, c), qv = qk(G_Q, r, c);
        dK[nt][e] += yA + zz;
        dQ[nt][e] += yQ;
        dG[nt][e] += yA * kv + yQ * qv - zz * kv;
      }
  }

  // ---- phase 5: outputs
#pragma unroll
  for (int nt = 0; nt < 8; ++nt)
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      const int r = r0 + g8 + 8 * hf, c = c0 + 8 * nt + 2 * qd;
      if (r < L) {
        const long long o = ((rb + r) * H + h) * D + c;
        *reinterpret_cast<float2*>(dq + o) = make_float2(dQ[nt][2 * hf], dQ[nt][2 * hf + 1]);
        *reinterpret_cast<float2*>(dk + o) = make_float2(dK[nt][2 * hf], dK[nt][2 * hf + 1]);
      }
    }
  __syncthreads();                      // R images / corrections no longer read
  float* dGs = reinterpret_cast<float*>(sm + G_S0);    // dGamma [64][LDG]
#pragma unroll
  for (int nt = 0; nt < 8; ++nt)
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      const int r = r0 + g8 + 8 * hf, c = c0 + 8 * nt + 2 * qd;
      *reinterpret_cast<float2*>(dGs + r * LDG + c) = make_float2(dG[nt][2 * hf], dG[nt][2 * hf + 1]);
    }
  __syncthreads();
  if (tid < D) dGs[63 * LDG + tid] += s_dgl[tid];
  __syncthreads();
  // dg = reverse cumulative sum of dGamma: two threads per channel, 32 rows each
  {
    const int c = tid & 127, part = tid >> 7;
    float x[32];
#pragma unroll
    for (int e = 0; e < 32; ++e) x[e] = dGs[(32 * part + e) * LDG + c];
#pragma unroll
    for (int e = 30; e >= 0; --e) x[e] += x[e + 1];
    if (part == 1) s_half[c] = x[0];
    __syncthreads();
    const float add = part ? 0.f : s_half[c];
#pragma unroll
    for (int e = 0; e < 32; ++e) dGs[(32 * part + e) * LDG + c] = x[e] + add;
  }
  __syncthreads();
  if constexpr (!GRPD) {
    for (int i = tid; i < C * 32; i += NTH) {
      const int r = i >> 5, c4 = i & 31;
      if (r < L)
        *reinterpret_cast<float4*>(dg + ((rb + r) * H + h) * D + 4 * c4) =
            *reinterpret_cast<const float4*>(dGs + r * LDG + 4 * c4);
    }
  } else {
    const int ng = D >> gsh, gs = 1 << gsh;
    for (int i = tid; i < C * ng; i += NTH) {
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

constexpr int kChainNB = 16;

bool set_attrs() {
  return once_per_device(kOnceBwdTc, []() {
    return cudaFuncSetAttribute(kda_bwd_chain_kernel<kChainNB>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                Chain<kChainNB>::SMEM) == cudaSuccess &&
           cudaFuncSetAttribute(kda_bwd_grad_kernel<false>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, GRAD_SMEM) == cudaSuccess &&
           cudaFuncSetAttribute(kda_bwd_grad_kernel<true>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, GRAD_SMEM) == cudaSuccess;
  });
}

struct BwdTcScratch {
  long long nslots;
  size_t rec, simg, dlimg, dsimg, ddimg, total;
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
  r.total = r.ddimg + per * kImgD;
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
    using CF = Chain<kChainNB>;
    KDA_TIMED(KDA_KERNEL_BWD_CHAIN, stream,
              (kda_bwd_chain_kernel<kChainNB><<<dim3(2 * CF::NJB, H, B), NTH, CF::SMEM, stream>>>(
                  rec, h0, cu_seqlens, static_cast<const bf16*>(dout), dhT, dh0, base + sc.simg,
                  base + sc.dlimg, base + sc.dsimg, base + sc.ddimg, T, H, sc.nslots)));
    note_launches(1);
    e = cudaGetLastError();
  }
  if (e == cudaSuccess && sc.nslots > 0) {
    auto grad = gsh != 0 ? kda_bwd_grad_kernel<true> : kda_bwd_grad_kernel<false>;
    KDA_TIMED(KDA_KERNEL_BWD_GRAD, stream,
              grad<<<dim3((unsigned)sc.nslots, H), NTH, GRAD_SMEM, stream>>>(
                  static_cast<const bf16*>(q), static_cast<const bf16*>(k),
                  static_cast<const bf16*>(v), g, beta, static_cast<const bf16*>(dout),
                  cu_seqlens, rec, base + sc.simg, base + sc.dlimg, base + sc.dsimg,
                  base + sc.ddimg, dq, dk, dv, dg, dbeta, B, T, H, gsh, sc.nslots));
    note_launches(1);
    e = cudaGetLastError();
  }
  if (pooled) cudaFreeAsync(scratch, stream);
  return e;
}

}  // namespace kda
