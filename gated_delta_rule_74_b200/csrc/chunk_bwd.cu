// KDA prefill backward on the GPU (first path: recurrent, fp32 CUDA cores).
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
// The states S_t are needed in reverse order: a forward sweep keeps S at every
// chunk start (64 tokens) in scratch; the reverse sweep recomputes each chunk's
// 65 states from its checkpoint into scratch and then walks it backwards.
//
// Mapping: one CTA of 512 threads per (sequence, head).  Warp w owns rows
// [w R, (w+1) R) of S (R = dk / 16) and lane l the columns [l CPT, (l+1) CPT)
// (CPT = dv / 32): sums over columns (dq, dk, dg) are a per-lane partial and an
// xor-shuffle over the warp; sums over rows (a^T k, G^T k) go through shared
// memory, double-buffered so that each step costs one CTA barrier.  Packed
// documents are separate chains (the state does not cross a boundary), so their
// gradients are separate too.
#include "kda_common.cuh"
#include "segments.cuh"

namespace kda {
namespace {

constexpr int NTB = 512;
constexpr int NWB = NTB / 32;

template <int CPT> struct VecT;
template <> struct VecT<4> {
  static __device__ __forceinline__ void ld(const float* p, float (&x)[4]) {
    const float4 t = *reinterpret_cast<const float4*>(p);
    x[0] = t.x; x[1] = t.y; x[2] = t.z; x[3] = t.w;
  }
  static __device__ __forceinline__ void st(float* p, const float (&x)[4]) {
    *reinterpret_cast<float4*>(p) = make_float4(x[0], x[1], x[2], x[3]);
  }
};
template <> struct VecT<2> {
  static __device__ __forceinline__ void ld(const float* p, float (&x)[2]) {
    const float2 t = *reinterpret_cast<const float2*>(p);
    x[0] = t.x; x[1] = t.y;
  }
  static __device__ __forceinline__ void st(float* p, const float (&x)[2]) {
    *reinterpret_cast<float2*>(p) = make_float2(x[0], x[1]);
  }
};

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

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
  constexpr int R = DK / NWB;          // rows per warp
  constexpr int CPT = DV / 32;         // columns per lane
  constexpr int SZ = DK * DV;
  __shared__ float s_red[2][2][NWB][DV];   // [buffer][quantity][warp][column]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = blockIdx.x, s = blockIdx.y;
  const int r0 = warp * R, col0 = lane * CPT;
  long long row0, t_beg, t_end;
  seq_range(cu_seqlens, s, T, row0, t_beg, t_end);
  const long long len = t_end - t_beg;
  const int nch = (int)chunk_count(len);
  const long long sidx = ((long long)s * H + h) * SZ;
  // scratch of this chain: checkpoints (one per chunk) and one chunk's states
  float* ck = ckpt + (seq_chunk_base(cu_seqlens, s, T) * H + (long long)h * nch) * SZ;
  float* cs = cst + ((long long)s * H + h) * (long long)(kChunk + 1) * SZ;
  auto tile = [&](float* base, int i) { return base + (long long)(r0 + i) * DV + col0; };
  auto ctile = [&](const float* base, int i) { return base + (long long)(r0 + i) * DV + col0; };

  // one forward step of the tile: S <- a + beta k e^T, e = v - a^T k (column sums
  // through shared memory, buffer `buf`)
  auto fwd_step = [&](float (&S)[R][CPT], long long tok, int buf) {
    float kr[R];
    float part[CPT];
#pragma unroll
    for (int j = 0; j < CPT; ++j) part[j] = 0.f;
#pragma unroll
    for (int i = 0; i < R; ++i) {
      const float al = __expf(g[tok * DK + r0 + i]);
      kr[i] = to_f32(k[tok * DK + r0 + i]);
#pragma unroll
      for (int j = 0; j < CPT; ++j) {
        S[i][j] *= al;
        part[j] = fmaf(S[i][j], kr[i], part[j]);
      }
    }
#pragma unroll
    for (int j = 0; j < CPT; ++j) s_red[buf][0][warp][col0 + j] = part[j];
    __syncthreads();
    const float b = beta[tok];
#pragma unroll
    for (int j = 0; j < CPT; ++j) {
      float r = 0.f;
#pragma unroll
      for (int w = 0; w < NWB; ++w) r += s_red[buf][0][w][col0 + j];
      const float u = b * (to_f32(v[tok * DV + col0 + j]) - r);
#pragma unroll
      for (int i = 0; i < R; ++i) S[i][j] = fmaf(kr[i], u, S[i][j]);
    }
  };

  // ---- forward sweep: checkpoints at every chunk start
  float S[R][CPT];
#pragma unroll
  for (int i = 0; i < R; ++i)
#pragma unroll
    for (int j = 0; j < CPT; ++j) S[i][j] = h0 ? h0[sidx + (long long)(r0 + i) * DV + col0 + j] : 0.f;
  int buf = 0;
#pragma unroll 1
  for (int c = 0; c < nch; ++c) {
#pragma unroll
    for (int i = 0; i < R; ++i) VecT<CPT>::st(tile(ck + (long long)c * SZ, i), S[i]);
    const long long tb0 = t_beg + (long long)c * kChunk;
    const int L = (int)min((long long)kChunk, t_end - tb0);
    if (c == nch - 1) break;                       // the last chunk is recomputed below
#pragma unroll 1
    for (int t = 0; t < L; ++t) {
      fwd_step(S, (row0 + tb0 + t) * H + h, buf);
      buf ^= 1;
    }
  }

  // ---- reverse sweep
  float G[R][CPT];
#pragma unroll
  for (int i = 0; i < R; ++i)
#pragma unroll
    for (int j = 0; j < CPT; ++j) G[i][j] = dhT ? dhT[sidx + (long long)(r0 + i) * DV + col0 + j] : 0.f;
#pragma unroll 1
  for (int c = nch - 1; c >= 0; --c) {
    const long long tb0 = t_beg + (long long)c * kChunk;
    const int L = (int)min((long long)kChunk, t_end - tb0);
    // recompute the chunk's states S_0 .. S_L (own tile only: no barrier needed
    // between the stores and the reads below, both by this thread)
#pragma unroll
    for (int i = 0; i < R; ++i) {
      VecT<CPT>::ld(ctile(ck + (long long)c * SZ, i), S[i]);
      VecT<CPT>::st(tile(cs, i), S[i]);
    }
#pragma unroll 1
    for (int t = 0; t < L; ++t) {
      fwd_step(S, (row0 + tb0 + t) * H + h, buf);
      buf ^= 1;
#pragma unroll
      for (int i = 0; i < R; ++i) VecT<CPT>::st(tile(cs + (long long)(t + 1) * SZ, i), S[i]);
    }
#pragma unroll 1
    for (int t = L - 1; t >= 0; --t) {
      const long long tok = (row0 + tb0 + t) * H + h;
      float dov[CPT];
#pragma unroll
      for (int j = 0; j < CPT; ++j) dov[j] = to_f32(dout[tok * DV + col0 + j]);
      // dq_t = S_t do_t (S_t = state after this token)
      float qr[R], kr[R], al[R], dqp[R];
#pragma unroll
      for (int i = 0; i < R; ++i) {
        float sn[CPT];
        VecT<CPT>::ld(ctile(cs + (long long)(t + 1) * SZ, i), sn);
        float acc = 0.f;
#pragma unroll
        for (int j = 0; j < CPT; ++j) acc = fmaf(sn[j], dov[j], acc);
        dqp[i] = acc;
        qr[i] = to_f32(q[tok * DK + r0 + i]);
        kr[i] = to_f32(k[tok * DK + r0 + i]);
        al[i] = __expf(g[tok * DK + r0 + i]);
      }
      // a = Diag(alpha) S_{t-1};  G += q do^T;  partial column sums of a^T k, G^T k
      float A[R][CPT];
      float pr[CPT], pw[CPT];
#pragma unroll
      for (int j = 0; j < CPT; ++j) { pr[j] = 0.f; pw[j] = 0.f; }
#pragma unroll
      for (int i = 0; i < R; ++i) {
        VecT<CPT>::ld(ctile(cs + (long long)t * SZ, i), A[i]);
#pragma unroll
        for (int j = 0; j < CPT; ++j) {
          A[i][j] *= al[i];
          G[i][j] = fmaf(qr[i], dov[j], G[i][j]);
          pr[j] = fmaf(A[i][j], kr[i], pr[j]);
          pw[j] = fmaf(G[i][j], kr[i], pw[j]);
        }
      }
#pragma unroll
      for (int j = 0; j < CPT; ++j) {
        s_red[buf][0][warp][col0 + j] = pr[j];
        s_red[buf][1][warp][col0 + j] = pw[j];
      }
      __syncthreads();
      const float b = beta[tok];
      float e[CPT], de[CPT], dbp = 0.f;
#pragma unroll
      for (int j = 0; j < CPT; ++j) {
        float r = 0.f, w = 0.f;
#pragma unroll
        for (int ww = 0; ww < NWB; ++ww) {
          r += s_red[buf][0][ww][col0 + j];
          w += s_red[buf][1][ww][col0 + j];
        }
        e[j] = to_f32(v[tok * DV + col0 + j]) - r;
        de[j] = b * w;
        dbp = fmaf(w, e[j], dbp);
      }
      buf ^= 1;
      if (warp == 0) {
        VecT<CPT>::st(dvo + tok * DV + col0, de);
        dbp = warp_sum(dbp);
        if (lane == 0) dbeta[tok] = dbp;
      }
      // dk_t = beta G e - a de;  da = G - k de^T;  dg_t = rowsum(da * a);  G <- Diag(alpha) da
      float dkp[R], dgp[R];
#pragma unroll
      for (int i = 0; i < R; ++i) {
        float a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
        for (int j = 0; j < CPT; ++j) {
          a1 = fmaf(G[i][j], e[j], a1);
          a2 = fmaf(A[i][j], de[j], a2);
          const float da = fmaf(-kr[i], de[j], G[i][j]);
          a3 = fmaf(da, A[i][j], a3);
          G[i][j] = al[i] * da;
        }
        dkp[i] = b * a1 - a2;
        dgp[i] = a3;
      }
#pragma unroll
      for (int i = 0; i < R; ++i) {
        const float xq = warp_sum(dqp[i]);
        const float xk = warp_sum(dkp[i]);
        const float xg = warp_sum(dgp[i]);
        if (lane == i) {
          dq[tok * DK + r0 + i] = xq;
          dk[tok * DK + r0 + i] = xk;
          dg[tok * DK + r0 + i] = xg;
        }
      }
    }
  }
  if (dh0) {
#pragma unroll
    for (int i = 0; i < R; ++i) VecT<CPT>::st(dh0 + sidx + (long long)(r0 + i) * DV + col0, G[i]);
  }
}

template <typename Tin, int DK, int DV>
cudaError_t launch_t(const void* q, const void* k, const void* v, const float* g,
                     const float* beta, const float* h0, const int32_t* cu, const void* dout,
                     const float* dhT, float* dq, float* dk, float* dv, float* dg, float* dbeta,
                     float* dh0, float* ckpt, float* cst, int B, int T, int H,
                     cudaStream_t stream) {
  KDA_TIMED(KDA_KERNEL_BWD, stream,
            kda_chunk_bwd_kernel<Tin, DK, DV><<<dim3(H, B), NTB, 0, stream>>>(
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
  const size_t sz = (size_t)dk * dv;
  // checkpoints: one per chunk of every sequence (plus one per sequence), per head;
  // one chunk of states per (sequence, head)
  const size_t nck = (size_t)(chunk_slots(B, T, cu_seqlens != nullptr) + B) * H;
  const size_t ncs = (size_t)B * H * (kChunk + 1);
  void* scratch = nullptr;
  cudaError_t e = cudaMallocFromPoolAsync(&scratch, (nck + ncs) * sz * sizeof(float), pool,
                                          stream);
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
