// KDA prefill backward on the GPU (recurrent, fp32 CUDA cores).
//
// The chunked form is what trains (miniKimiK3 model card, "Kimi Delta Attention"
// bullet: "trains through a chunked parallel form"); its gradients are those of
// the recurrence it equals.  For L = sum(out * dout) + sum(hT * dhT) this kernel
// differentiates the recurrence step by step in reverse.  Forward step t:
//     a = Diag(exp(g_t)) S_{t-1};  e = v_t - a^T k_t;  S_t = a + beta_t k_t e^T;
//     o_t = S_t^T q_t.
// Reverse step with G = dL/dS_t:
//     G += q_t do_t^T;  dq_t = S_t do_t;  w = G^T k_t;  dbeta_t = w . e;
//     de = beta_t w = dv_t;  dk_t = beta_t G e - a de;  da = G - k_t de^T;
//     dg_t[c] = sum_j da[c][j] a[c][j];  G <- Diag(exp(g_t)) da.
//
// Column independence.  Every column j of S (and of G) evolves on its own: the
// sums that couple entries run over the rows (a^T k, G^T k), never over the
// columns.  So a warp owns NC = 8 columns and all dk rows (lane l: rows
// [l R, l R + R), R = dk / 32) and runs its chain with warp shuffles only -- no
// CTA barrier per token.  Only the per-token row gradients dq, dk, dg and dbeta
// sum over columns; each warp adds its part with one vector atomic per lane
// (the sum order across warps is not fixed, so those four differ between runs
// by fp32 rounding; dv and dh0 are column-local and reproducible).
//
// Memory.  Per chunk of 64 tokens the CTA stages its inputs in shared memory
// (fp32).  The states S_t are needed in reverse order: a forward sweep keeps the
// warp's slice of S at every chunk start (checkpoints, global scratch); the
// reverse sweep re-runs each chunk forward from its checkpoint, storing the
// pre-token states S_{t-1} (global scratch reused per chunk, L2-resident) and
// e_t (shared), then walks the chunk backwards, streaming the states back through
// a 4-deep cp.async ring.  Packed documents are separate chains: neither the
// state nor its gradient crosses a boundary.
#include "kda_common.cuh"
#include "segments.cuh"
#include "sm100.cuh"

namespace kda {
namespace {

using namespace sm100;

constexpr int NC = 8;             // state columns per warp
constexpr int WPC = 4;            // warps per CTA
constexpr int CPC = NC * WPC;     // state columns per CTA
constexpr int NTB = 32 * WPC;
constexpr int RING = 4;           // depth of the reverse sweep's state prefetch
constexpr unsigned FULL = 0xffffffffu;

// Sum over the 32 lanes of each of the 8 per-lane values p[j]; every lane gets
// all 8 totals.  Transpose-reduce (the halves exchanged at lane distance 16, 8,
// 4 leave each lane one column), two butterfly steps, then a gather.
__device__ __forceinline__ void colsum8(const float (&p)[8], float (&tot)[8], int lane) {
  const bool b4 = lane & 16, b3 = lane & 8, b2 = lane & 4;
  float x[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float keep = b4 ? p[i + 4] : p[i];
    const float send = b4 ? p[i] : p[i + 4];
    x[i] = keep + __shfl_xor_sync(FULL, send, 16);
  }
  float y[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const float keep = b3 ? x[i + 2] : x[i];
    const float send = b3 ? x[i] : x[i + 2];
    y[i] = keep + __shfl_xor_sync(FULL, send, 8);
  }
  float z = (b2 ? y[1] : y[0]) + __shfl_xor_sync(FULL, b2 ? y[0] : y[1], 4);
  z += __shfl_xor_sync(FULL, z, 2);
  z += __shfl_xor_sync(FULL, z, 1);
  // lane holds column 4*b4 + 2*b3 + b2
#pragma unroll
  for (int j = 0; j < 8; ++j)
    tot[j] = __shfl_sync(FULL, z, ((j >> 2) & 1) * 16 + ((j >> 1) & 1) * 8 + (j & 1) * 4);
}

template <int R> struct Rows;
template <> struct Rows<4> {
  static __device__ __forceinline__ void ld(const float* p, float (&x)[4]) {
    const float4 t = *reinterpret_cast<const float4*>(p);
    x[0] = t.x; x[1] = t.y; x[2] = t.z; x[3] = t.w;
  }
  static __device__ __forceinline__ void add(float* p, const float (&x)[4]) {
    atomicAdd(reinterpret_cast<float4*>(p), make_float4(x[0], x[1], x[2], x[3]));
  }
};
template <> struct Rows<2> {
  static __device__ __forceinline__ void ld(const float* p, float (&x)[2]) {
    const float2 t = *reinterpret_cast<const float2*>(p);
    x[0] = t.x; x[1] = t.y;
  }
  static __device__ __forceinline__ void add(float* p, const float (&x)[2]) {
    atomicAdd(reinterpret_cast<float2*>(p), make_float2(x[0], x[1]));
  }
};

__device__ __forceinline__ void ld8(const float* p, float (&x)[8]) {
  const float4 a = *reinterpret_cast<const float4*>(p);
  const float4 b = *reinterpret_cast<const float4*>(p + 4);
  x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
  x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}
__device__ __forceinline__ void st8(float* p, const float (&x)[8]) {
  *reinterpret_cast<float4*>(p) = make_float4(x[0], x[1], x[2], x[3]);
  *reinterpret_cast<float4*>(p + 4) = make_float4(x[4], x[5], x[6], x[7]);
}

// 8 consecutive input elements (16-byte aligned) as fp32
__device__ __forceinline__ void gld8(const float* p, float (&x)[8]) { ld8(p, x); }
__device__ __forceinline__ void gld8(const __nv_bfloat16* p, float (&x)[8]) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    x[2 * i] = __uint_as_float(w[i] << 16);
    x[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

// Shared-memory layout (floats): per chunk the staged inputs, then per-warp e_t,
// then the per-warp state ring.
template <int DK>
struct BwdSmem {
  static constexpr int G = 0;                         // [64][DK] log-decay
  static constexpr int K = G + kChunk * DK;           // [64][DK]
  static constexpr int Q = K + kChunk * DK;           // [64][DK]
  static constexpr int V = Q + kChunk * DK;           // [64][CPC] this CTA's columns
  static constexpr int DO = V + kChunk * CPC;         // [64][CPC]
  static constexpr int BETA = DO + kChunk * CPC;      // [64]
  static constexpr int E = BETA + kChunk;             // [WPC][64][NC]
  static constexpr int RINGB = E + WPC * kChunk * NC; // [WPC][RING][DK * NC]
  static constexpr int TOTAL = RINGB + WPC * RING * DK * NC;
  static constexpr size_t BYTES = (size_t)TOTAL * sizeof(float);
};

// Stage tokens [0, L) of a chunk whose first token row is `rowbase` (head h): g, k
// and this CTA's CPC columns of v; with `rev` also q and dout.
template <typename Tin, int DK, int DV>
__device__ __forceinline__ void stage_chunk(float* sm, const Tin* __restrict__ q,
                                            const Tin* __restrict__ k, const Tin* __restrict__ v,
                                            const float* __restrict__ g,
                                            const float* __restrict__ beta,
                                            const Tin* __restrict__ dout, long long rowbase, int L,
                                            int H, int h, int cta_c0, bool rev) {
  using S = BwdSmem<DK>;
  const int tid = threadIdx.x;
  constexpr int P8 = DK / 8;                  // 8-element pieces per row
  for (int i = tid; i < L * P8; i += NTB) {
    const int t = i / P8, c = (i % P8) * 8;
    const long long src = ((rowbase + t) * H + h) * (long long)DK + c;
    float x[8];
    ld8(g + src, x);
    st8(sm + S::G + t * DK + c, x);
    gld8(k + src, x);
    st8(sm + S::K + t * DK + c, x);
    if (rev) {
      gld8(q + src, x);
      st8(sm + S::Q + t * DK + c, x);
    }
  }
  constexpr int PV = CPC / 8;
  for (int i = tid; i < L * PV; i += NTB) {
    const int t = i / PV, c = (i % PV) * 8;
    const long long src = ((rowbase + t) * H + h) * (long long)DV + cta_c0 + c;
    float x[8];
    gld8(v + src, x);
    st8(sm + S::V + t * CPC + c, x);
    if (rev) {
      gld8(dout + src, x);
      st8(sm + S::DO + t * CPC + c, x);
    }
  }
  for (int t = tid; t < L; t += NTB) sm[S::BETA + t] = beta[(rowbase + t) * H + h];
}

// One CTA per (column block of CPC state columns, head, sequence).
template <typename Tin, int DK, int DV>
__global__ void __launch_bounds__(NTB, 1)
kda_chunk_bwd_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k,
                     const Tin* __restrict__ v, const float* __restrict__ g,
                     const float* __restrict__ beta, const float* __restrict__ h0,
                     const int32_t* __restrict__ cu_seqlens, const Tin* __restrict__ dout,
                     const float* __restrict__ dhT, float* __restrict__ dq,
                     float* __restrict__ dk, float* __restrict__ dvo, float* __restrict__ dg,
                     float* __restrict__ dbeta, float* __restrict__ dh0,
                     float* __restrict__ ckpt, float* __restrict__ cst, int T, int H) {
  constexpr int R = DK / 32;            // state rows per lane
  constexpr int NV = R * NC / 4;        // float4 per lane in a warp's state slice
  constexpr int SLICE = DK * NC;        // floats in a warp's state slice
  constexpr int NB = DV / CPC;          // CTAs per (sequence, head)
  constexpr long long SZ = (long long)DK * DV;
  using SM = BwdSmem<DK>;
  extern __shared__ __align__(16) float sm[];

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int bx = blockIdx.x, h = blockIdx.y, s = blockIdx.z;
  const int cta_c0 = bx * CPC, wc = warp * NC;
  const int c0 = cta_c0 + wc;           // this warp's first state column
  const int rl = lane * R;              // this lane's first state row
  long long row0, t_beg, t_end;
  seq_range(cu_seqlens, s, T, row0, t_beg, t_end);
  const int nch = (int)chunk_count(t_end - t_beg);
  const long long sidx = ((long long)s * H + h) * SZ;
  // checkpoint of chunk c: ckpt + ck0 + c * H * SZ (chunks of all sequences numbered
  // consecutively, heads inside a chunk, warp slices inside a head)
  const long long ck0 =
      (seq_chunk_base(cu_seqlens, s, T) * H + h) * SZ + (long long)(bx * WPC + warp) * SLICE;
  // pre-token state of token t of the current chunk: cs + t * WPC * SLICE
  float* const cs = cst + ((((long long)s * H + h) * NB + bx) * kChunk * WPC + warp) * SLICE;
  float* const e_sm = sm + SM::E + warp * kChunk * NC;
  float* const ring = sm + SM::RINGB + warp * RING * SLICE;

  // a warp's state slice: lane element (i, j) in float4 m = 2 i + j / 4, at (m * 32 + lane) * 4
  auto st_slice = [&](float* base, const float (&X)[R][NC]) {
#pragma unroll
    for (int i = 0; i < R; ++i)
#pragma unroll
      for (int jq = 0; jq < 2; ++jq)
        *reinterpret_cast<float4*>(base + ((i * 2 + jq) * 32 + lane) * 4) =
            make_float4(X[i][jq * 4], X[i][jq * 4 + 1], X[i][jq * 4 + 2], X[i][jq * 4 + 3]);
  };
  auto ld_slice = [&](const float* base, float (&X)[R][NC]) {
#pragma unroll
    for (int i = 0; i < R; ++i)
#pragma unroll
      for (int jq = 0; jq < 2; ++jq) {
        const float4 t4 = *reinterpret_cast<const float4*>(base + ((i * 2 + jq) * 32 + lane) * 4);
        X[i][jq * 4] = t4.x; X[i][jq * 4 + 1] = t4.y;
        X[i][jq * 4 + 2] = t4.z; X[i][jq * 4 + 3] = t4.w;
      }
  };
  // one forward step on staged token t: S <- a + beta k e^T, e = v - a^T k
  auto fwd = [&](float (&S)[R][NC], int t, float (&e)[NC]) {
    float gl[R], kr[R];
    Rows<R>::ld(sm + SM::G + t * DK + rl, gl);
    Rows<R>::ld(sm + SM::K + t * DK + rl, kr);
    float p[NC];
#pragma unroll
    for (int j = 0; j < NC; ++j) p[j] = 0.f;
#pragma unroll
    for (int i = 0; i < R; ++i) {
      const float al = __expf(gl[i]);
#pragma unroll
      for (int j = 0; j < NC; ++j) {
        S[i][j] *= al;
        p[j] = fmaf(S[i][j], kr[i], p[j]);
      }
    }
    float tot[NC];
    colsum8(p, tot, lane);
    float vv[NC];
    ld8(sm + SM::V + t * CPC + wc, vv);
    const float b = sm[SM::BETA + t];
#pragma unroll
    for (int j = 0; j < NC; ++j) {
      e[j] = vv[j] - tot[j];
      const float u = b * e[j];
#pragma unroll
      for (int i = 0; i < R; ++i) S[i][j] = fmaf(kr[i], u, S[i][j]);
    }
  };

  // ---- forward sweep: the warp's slice of S at every chunk start
  float S[R][NC], e[NC];
#pragma unroll
  for (int i = 0; i < R; ++i) {
    if (h0) {
      ld8(h0 + sidx + (long long)(rl + i) * DV + c0, S[i]);
    } else {
#pragma unroll
      for (int j = 0; j < NC; ++j) S[i][j] = 0.f;
    }
  }
#pragma unroll 1
  for (int c = 0; c < nch; ++c) {
    st_slice(ckpt + ck0 + (long long)c * H * SZ, S);
    if (c == nch - 1) break;            // the last chunk is re-run by the reverse sweep
    const long long rb = row0 + t_beg + (long long)c * kChunk;
    __syncthreads();                    // the previous chunk's staged inputs are consumed
    stage_chunk<Tin, DK, DV>(sm, q, k, v, g, beta, dout, rb, kChunk, H, h, cta_c0, false);
    __syncthreads();
#pragma unroll 1
    for (int t = 0; t < kChunk; ++t) fwd(S, t, e);
  }

  // ---- reverse sweep
  float G[R][NC];
#pragma unroll
  for (int i = 0; i < R; ++i) {
    if (dhT) {
      ld8(dhT + sidx + (long long)(rl + i) * DV + c0, G[i]);
    } else {
#pragma unroll
      for (int j = 0; j < NC; ++j) G[i][j] = 0.f;
    }
  }
#pragma unroll 1
  for (int c = nch - 1; c >= 0; --c) {
    const long long rb = row0 + t_beg + (long long)c * kChunk;
    const int L = (int)min((long long)kChunk, t_end - t_beg - (long long)c * kChunk);
    __syncthreads();
    stage_chunk<Tin, DK, DV>(sm, q, k, v, g, beta, dout, rb, L, H, h, cta_c0, true);
    __syncthreads();
    ld_slice(ckpt + ck0 + (long long)c * H * SZ, S);
    // re-run the chunk: pre-token states to scratch, e_t to shared, dq_t = S_t do_t
#pragma unroll 1
    for (int t = 0; t < L; ++t) {
      st_slice(cs + (long long)t * WPC * SLICE, S);
      fwd(S, t, e);
      if (lane == 0) st8(e_sm + t * NC, e);
      float dov[NC];
      ld8(sm + SM::DO + t * CPC + wc, dov);
      float dqp[R];
#pragma unroll
      for (int i = 0; i < R; ++i) {
        float acc = 0.f;
#pragma unroll
        for (int j = 0; j < NC; ++j) acc = fmaf(S[i][j], dov[j], acc);
        dqp[i] = acc;
      }
      Rows<R>::add(dq + ((rb + t) * H + h) * DK + rl, dqp);
    }
    __syncwarp();
    // walk the chunk backwards; pre-token states arrive through the ring
#pragma unroll
    for (int d = 0; d < RING; ++d) {
      const int t = L - 1 - d;
      if (t >= 0) {
#pragma unroll
        for (int m = 0; m < NV; ++m)
          cp_async16(ring + (t % RING) * SLICE + (m * 32 + lane) * 4,
                     cs + (long long)t * WPC * SLICE + (m * 32 + lane) * 4, 16);
      }
      cp_async_commit();
    }
#pragma unroll 1
    for (int t = L - 1; t >= 0; --t) {
      cp_async_wait_group<RING - 1>();
      float A[R][NC];
      ld_slice(ring + (t % RING) * SLICE, A);
      float gl[R], kr[R], qr[R], dov[NC], ee[NC];
      Rows<R>::ld(sm + SM::G + t * DK + rl, gl);
      Rows<R>::ld(sm + SM::K + t * DK + rl, kr);
      Rows<R>::ld(sm + SM::Q + t * DK + rl, qr);
      ld8(sm + SM::DO + t * CPC + wc, dov);
      ld8(e_sm + t * NC, ee);
      const float b = sm[SM::BETA + t];
      float al[R], pw[NC];
#pragma unroll
      for (int j = 0; j < NC; ++j) pw[j] = 0.f;
#pragma unroll
      for (int i = 0; i < R; ++i) {
        al[i] = __expf(gl[i]);
#pragma unroll
        for (int j = 0; j < NC; ++j) {
          A[i][j] *= al[i];
          G[i][j] = fmaf(qr[i], dov[j], G[i][j]);
          pw[j] = fmaf(G[i][j], kr[i], pw[j]);
        }
      }
      float w[NC];
      colsum8(pw, w, lane);
      float de[NC], dbp = 0.f;
#pragma unroll
      for (int j = 0; j < NC; ++j) {
        de[j] = b * w[j];
        dbp = fmaf(w[j], ee[j], dbp);
      }
      const long long tok = (rb + t) * H + h;
      if (lane == 0) {
        st8(dvo + tok * DV + c0, de);
        atomicAdd(dbeta + tok, dbp);
      }
      float dkp[R], dgp[R];
#pragma unroll
      for (int i = 0; i < R; ++i) {
        float a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
        for (int j = 0; j < NC; ++j) {
          a1 = fmaf(G[i][j], ee[j], a1);
          a2 = fmaf(A[i][j], de[j], a2);
          const float da = fmaf(-kr[i], de[j], G[i][j]);
          a3 = fmaf(da, A[i][j], a3);
          G[i][j] = al[i] * da;
        }
        dkp[i] = b * a1 - a2;
        dgp[i] = a3;
      }
      Rows<R>::add(dk + tok * DK + rl, dkp);
      Rows<R>::add(dg + tok * DK + rl, dgp);
      const int tn = t - RING;
      if (tn >= 0) {
#pragma unroll
        for (int m = 0; m < NV; ++m)
          cp_async16(ring + (tn % RING) * SLICE + (m * 32 + lane) * 4,
                     cs + (long long)tn * WPC * SLICE + (m * 32 + lane) * 4, 16);
      }
      cp_async_commit();
    }
    __syncwarp();
  }
  cp_async_wait_all();
  if (dh0) {
#pragma unroll
    for (int i = 0; i < R; ++i) st8(dh0 + sidx + (long long)(rl + i) * DV + c0, G[i]);
  }
}

template <typename Tin, int DK, int DV>
cudaError_t launch_t(const void* q, const void* k, const void* v, const float* g,
                     const float* beta, const float* h0, const int32_t* cu, const void* dout,
                     const float* dhT, float* dq, float* dk, float* dv, float* dg, float* dbeta,
                     float* dh0, float* ckpt, float* cst, int B, int T, int H,
                     cudaStream_t stream) {
  constexpr size_t smem = BwdSmem<DK>::BYTES;
  const cudaError_t ea = cudaFuncSetAttribute(kda_chunk_bwd_kernel<Tin, DK, DV>,
                                              cudaFuncAttributeMaxDynamicSharedMemorySize,
                                              (int)smem);
  if (ea != cudaSuccess) return ea;
  KDA_TIMED(KDA_KERNEL_BWD, stream,
            kda_chunk_bwd_kernel<Tin, DK, DV><<<dim3(DV / CPC, H, B), NTB, smem, stream>>>(
                static_cast<const Tin*>(q), static_cast<const Tin*>(k), static_cast<const Tin*>(v),
                g, beta, h0, cu, static_cast<const Tin*>(dout), dhT, dq, dk, dv, dg, dbeta, dh0,
                ckpt, cst, T, H));
  note_launches(1);
  return cudaGetLastError();
}

template <typename Tin>
cudaError_t launch_dtype(const void* q, const void* k, const void* v, const float* g,
                         const float* beta, const float* h0, const int32_t* cu, const void* dout,
                         const float* dhT, float* dq, float* dk, float* dv, float* dg,
                         float* dbeta, float* dh0, float* ckpt, float* cst, int B, int T, int H,
                         int dkk, int dvv, cudaStream_t stream) {
#define KDA_BWD_CASE(A, Bv)                                                                   \
  if (dkk == A && dvv == Bv)                                                                 \
    return launch_t<Tin, A, Bv>(q, k, v, g, beta, h0, cu, dout, dhT, dq, dk, dv, dg, dbeta, \
                                dh0, ckpt, cst, B, T, H, stream);
  KDA_BWD_CASE(128, 128)
  KDA_BWD_CASE(128, 64)
  KDA_BWD_CASE(64, 128)
  KDA_BWD_CASE(64, 64)
#undef KDA_BWD_CASE
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_chunk_bwd(const void* q, const void* k, const void* v, const float* g,
                             const float* beta, const float* h0, const int32_t* cu_seqlens,
                             const void* dout, const float* dhT, float* dq, float* dkk,
                             float* dvv, float* dg, float* dbeta, float* dh0, int B, int T, int H,
                             int dk, int dv, int in_dtype, cudaStream_t stream) {
  int sms = 148;
  cudaMemPool_t pool = nullptr;
  if (!device_ctx(&sms, &pool)) return cudaErrorInvalidDevice;
  if (!pool) return cudaErrorMemoryAllocation;
  // dq, dk, dg and dbeta are sums of per-warp parts
  const size_t rows = cu_seqlens ? (size_t)T : (size_t)B * T;
  cudaError_t e = cudaSuccess;
  if (rows > 0) {
    const size_t n = rows * H * dk * sizeof(float);
    if ((e = cudaMemsetAsync(dq, 0, n, stream)) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(dkk, 0, n, stream)) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(dg, 0, n, stream)) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(dbeta, 0, rows * H * sizeof(float), stream)) != cudaSuccess)
      return e;
  }
  const size_t sz = (size_t)dk * dv;
  // checkpoints: one state per chunk of every sequence, per head; the pre-token
  // states of one chunk per (sequence, head)
  const size_t nck = (size_t)(chunk_slots(B, T, cu_seqlens != nullptr) + B) * H;
  const size_t ncs = (size_t)B * H * kChunk;
  void* scratch = nullptr;
  e = cudaMallocFromPoolAsync(&scratch, (nck + ncs) * sz * sizeof(float), pool, stream);
  if (e != cudaSuccess) return e;
  float* ckpt = static_cast<float*>(scratch);
  float* cst = ckpt + nck * sz;
  if (in_dtype == KDA_BF16)
    e = launch_dtype<__nv_bfloat16>(q, k, v, g, beta, h0, cu_seqlens, dout, dhT, dq, dkk, dvv, dg,
                                    dbeta, dh0, ckpt, cst, B, T, H, dk, dv, stream);
  else
    e = launch_dtype<float>(q, k, v, g, beta, h0, cu_seqlens, dout, dhT, dq, dkk, dvv, dg, dbeta,
                            dh0, ckpt, cst, B, T, H, dk, dv, stream);
  cudaFreeAsync(scratch, stream);
  return e;
}

}  // namespace kda
