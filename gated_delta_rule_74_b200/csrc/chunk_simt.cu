// KDA prefill through the chunked parallel form, fp32 on the CUDA cores.
//
// This is the path for fp32 inputs: a tensor-core contraction in tf32 would
// carry ~1e-3 relative error, so every step here is an fp32 FMA.
//
// Chunked form (miniKimiK3 model card, "Kimi Delta Attention" bullet: the
// recurrence trains through a chunked parallel form).  For a chunk of L <= 64
// tokens with initial state S (dk x dv), per key channel c:
//     G_r     = g_0 + ... + g_r                         (within the chunk)
//     A[r,i]  = sum_c k_rc k_ic exp(G_rc - G_ic),   i <  r
//     Aqk[r,i]= sum_c q_rc k_ic exp(G_rc - G_ic),   i <= r
//     (I + diag(beta) A) D = diag(beta) (V - Kbar S),   Kbar_r = exp(G_r) * k_r
//     O       = Qbar S + Aqk D,                         Qbar_r = exp(G_r) * q_r
//     S_next  = Diag(exp(G_{L-1})) S + Kend^T D,        Kend_i = exp(G_{L-1} - G_i) * k_i
// The triangular system is solved by forward substitution, row by row.  All
// exponents exp(G_r - G_i) (i <= r) and exp(G_{L-1} - G_i) are <= 1 for g <= 0,
// and exp(G_r) <= 1, so nothing can overflow.
//
// Mapping: one CTA per (sequence, head, 32-column tile of dv); the CTA walks the
// sequence's chunks in order and keeps its 32 columns of S in shared memory.
// Packed documents (cu_seqlens) restart the state from their own h0 slot and
// restart chunking at the document start (Mini-K3-1H-mamba2 card, packed-
// document paragraph: state flow resets at every boundary).
#include "kda_common.cuh"

namespace kda {
namespace {

constexpr int C = 64;          // chunk length
constexpr int DVT = 32;        // dv columns per CTA
constexpr int NT = 256;        // threads per CTA

template <int DK>
struct SimtSmem {
  static constexpr int LD = DK + 1;            // padded row stride (bank spread)
  float k[C * LD];
  float q[C * LD];                             // q, later reused for Kend
  double G[C * LD];                            // cumulative log-decay (fp64: exponents are
                                               // differences G_r - G_i, exact to fp32
                                               // rounding however large |G| grows)
  float E[C * LD];                             // exp(G)
  float A[C * (C + 1)];
  float Aqk[C * (C + 1)];
  float S[DK * DVT];
  float X[C * DVT];                            // right-hand side, then D in place
  float v[C * DVT];
  float beta[C];
};

template <typename Tin, int DK>
__global__ void __launch_bounds__(NT, 1)
kda_chunk_simt_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k,
                      const Tin* __restrict__ v, const float* __restrict__ g,
                      const float* __restrict__ beta, const float* h0,
                      const int32_t* __restrict__ cu_seqlens, Tin* __restrict__ out,
                      float* hT, int T, int H, int dv, int gsh) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  SimtSmem<DK>& sm = *reinterpret_cast<SimtSmem<DK>*>(smem_raw);
  constexpr int LD = SimtSmem<DK>::LD;
  const int tid = threadIdx.x;
  const int j0 = blockIdx.x * DVT;      // first dv column of this CTA
  const int h = blockIdx.y;
  const int s = blockIdx.z;             // sequence / document

  long long row0, t_beg, t_end;         // token rows are (row0 + t) in [B*T]
  if (cu_seqlens) {
    int a = cu_seqlens[s], b = cu_seqlens[s + 1];
    a = min(max(a, 0), T);
    b = min(max(b, a), T);
    row0 = 0; t_beg = a; t_end = b;
  } else {
    row0 = (long long)s * T; t_beg = 0; t_end = T;
  }

  // initial state columns [j0, j0 + DVT)
  const long long sbase = ((long long)s * H + h) * DK * dv;
  for (int idx = tid; idx < DK * DVT; idx += NT) {
    const int c = idx / DVT, j = idx % DVT;
    sm.S[idx] = h0 ? h0[sbase + (long long)c * dv + j0 + j] : 0.f;
  }

  for (long long t0 = t_beg; t0 < t_end; t0 += C) {
    const int L = (int)min((long long)C, t_end - t0);
    __syncthreads();   // previous chunk finished with the buffers
    // ---- load the chunk (rows >= L padded with zeros: they contribute nothing)
    for (int idx = tid; idx < C * DK; idx += NT) {
      const int r = idx / DK, c = idx % DK;
      float kv = 0.f, qv = 0.f, gv = 0.f;
      if (r < L) {
        const long long tok = ((row0 + t0 + r) * H + h);
        kv = to_f32(k[tok * DK + c]);
        qv = to_f32(q[tok * DK + c]);
        gv = g[tok * (DK >> gsh) + (c >> gsh)];
      }
      sm.k[r * LD + c] = kv; sm.q[r * LD + c] = qv; sm.G[r * LD + c] = gv;
    }
    for (int idx = tid; idx < C * DVT; idx += NT) {
      const int r = idx / DVT, j = idx % DVT;
      float vv = 0.f;
      if (r < L) vv = to_f32(v[((row0 + t0 + r) * H + h) * dv + j0 + j]);
      sm.v[idx] = vv;
    }
    if (tid < C) sm.beta[tid] = tid < L ? beta[(row0 + t0 + tid) * H + h] : 0.f;
    __syncthreads();
    // ---- cumulative log-decay along the chunk, one thread per channel
    if (tid < DK) {
      double acc = 0.0;
      for (int r = 0; r < C; ++r) {
        acc += sm.G[r * LD + tid];
        sm.G[r * LD + tid] = acc;
        sm.E[r * LD + tid] = expf((float)acc);
      }
    }
    __syncthreads();
    // ---- A (strictly lower) and Aqk (lower incl. diagonal), pairwise exponents
    for (int idx = tid; idx < C * C; idx += NT) {
      const int r = idx / C, i = idx % C;
      float a = 0.f, aq = 0.f;
      if (i <= r) {
        const float* kr = sm.k + r * LD;
        const float* qr = sm.q + r * LD;
        const float* ki = sm.k + i * LD;
        const double* Gr = sm.G + r * LD;
        const double* Gi = sm.G + i * LD;
        for (int c = 0; c < DK; ++c) {
          const float e = expf((float)(Gr[c] - Gi[c]));
          const float kie = ki[c] * e;
          a = fmaf(kr[c], kie, a);
          aq = fmaf(qr[c], kie, aq);
        }
      }
      sm.A[r * (C + 1) + i] = (i < r) ? a : 0.f;
      sm.Aqk[r * (C + 1) + i] = aq;
    }
    // ---- right-hand side X = diag(beta) (V - Kbar S)
    for (int idx = tid; idx < C * DVT; idx += NT) {
      const int r = idx / DVT, j = idx % DVT;
      float acc = 0.f;
      const float* kr = sm.k + r * LD;
      const float* Er = sm.E + r * LD;
      for (int c = 0; c < DK; ++c) acc = fmaf(kr[c] * Er[c], sm.S[c * DVT + j], acc);
      sm.X[idx] = sm.beta[r] * (sm.v[idx] - acc);
    }
    __syncthreads();
    // ---- forward substitution: D_r = X_r - beta_r sum_{i<r} A[r,i] D_i.
    // Warp w solves columns 4w..4w+3; 8 lanes per column split the i-sum.
    {
      const int warp = tid >> 5, lane = tid & 31;
      const int j = warp * 4 + (lane >> 3), part = lane & 7;
      for (int r = 0; r < C; ++r) {
        float acc = 0.f;
        for (int i = part; i < r; i += 8) acc = fmaf(sm.A[r * (C + 1) + i], sm.X[i * DVT + j], acc);
        acc += __shfl_xor_sync(0xffffffffu, acc, 1);
        acc += __shfl_xor_sync(0xffffffffu, acc, 2);
        acc += __shfl_xor_sync(0xffffffffu, acc, 4);
        if (part == 0) sm.X[r * DVT + j] -= sm.beta[r] * acc;
        __syncwarp();
      }
    }
    __syncthreads();
    // ---- output O = Qbar S + Aqk D
    for (int idx = tid; idx < C * DVT; idx += NT) {
      const int r = idx / DVT, j = idx % DVT;
      if (r >= L) continue;
      float acc = 0.f;
      const float* qr = sm.q + r * LD;
      const float* Er = sm.E + r * LD;
      for (int c = 0; c < DK; ++c) acc = fmaf(qr[c] * Er[c], sm.S[c * DVT + j], acc);
      for (int i = 0; i <= r; ++i) acc = fmaf(sm.Aqk[r * (C + 1) + i], sm.X[i * DVT + j], acc);
      out[((row0 + t0 + r) * H + h) * dv + j0 + j] = from_f32<Tin>(acc);
    }
    __syncthreads();
    // ---- Kend_i = exp(G_{L-1} - G_i) * k_i, stored over q (rows >= L have k = 0;
    //      G of padded rows equals G_{L-1} because their g is 0)
    for (int idx = tid; idx < C * DK; idx += NT) {
      const int r = idx / DK, c = idx % DK;
      sm.q[r * LD + c] = sm.k[r * LD + c] * expf((float)(sm.G[(C - 1) * LD + c] - sm.G[r * LD + c]));
    }
    __syncthreads();
    // ---- S_next = Diag(exp(G_{L-1})) S + Kend^T D
    for (int idx = tid; idx < DK * DVT; idx += NT) {
      const int c = idx / DVT, j = idx % DVT;
      float acc = sm.E[(C - 1) * LD + c] * sm.S[idx];
      for (int i = 0; i < C; ++i) acc = fmaf(sm.q[i * LD + c], sm.X[i * DVT + j], acc);
      sm.S[idx] = acc;
    }
  }
  __syncthreads();
  if (hT) {
    for (int idx = tid; idx < DK * DVT; idx += NT) {
      const int c = idx / DVT, j = idx % DVT;
      hT[sbase + (long long)c * dv + j0 + j] = sm.S[idx];
    }
  }
}

template <typename Tin, int DK>
cudaError_t launch_t(const void* q, const void* k, const void* v, const float* g,
                     const float* beta, const float* h0, const int32_t* cu, void* out,
                     float* hT, int B, int T, int H, int dv, int gsh, cudaStream_t stream) {
  const size_t smem = sizeof(SimtSmem<DK>);
  cudaError_t e = cudaFuncSetAttribute(kda_chunk_simt_kernel<Tin, DK>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(dv / DVT, H, B);
  KDA_TIMED(KDA_KERNEL_SIMT, stream,
            kda_chunk_simt_kernel<Tin, DK><<<grid, NT, smem, stream>>>(
                static_cast<const Tin*>(q), static_cast<const Tin*>(k), static_cast<const Tin*>(v), g,
                beta, h0, cu, static_cast<Tin*>(out), hT, T, H, dv, gsh));
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_chunk_simt(const void* q, const void* k, const void* v, const float* g,
                              const float* beta, const float* h0, const int32_t* cu_seqlens,
                              void* out, float* hT, int B, int T, int H, int dk, int dv,
                              int in_dtype, int gsh, cudaStream_t stream) {
  if (in_dtype == KDA_BF16) {
    if (dk == 128)
      return launch_t<__nv_bfloat16, 128>(q, k, v, g, beta, h0, cu_seqlens, out, hT, B, T, H, dv, gsh, stream);
    return launch_t<__nv_bfloat16, 64>(q, k, v, g, beta, h0, cu_seqlens, out, hT, B, T, H, dv, gsh, stream);
  }
  if (dk == 128)
    return launch_t<float, 128>(q, k, v, g, beta, h0, cu_seqlens, out, hT, B, T, H, dv, gsh, stream);
  return launch_t<float, 64>(q, k, v, g, beta, h0, cu_seqlens, out, hT, B, T, H, dv, gsh, stream);
}

}  // namespace kda
