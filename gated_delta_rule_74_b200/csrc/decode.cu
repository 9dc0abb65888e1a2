// KDA recurrent decode step (one token per sequence), memory-bound.
//
// miniKimiK3 model card, "Kimi Delta Attention" bullet: decoding is a recurrence
// on a fixed state per head at constant cost per token.  Per (n, h):
//     A   = Diag(exp(g)) S                         (decay the key-channel rows)
//     S'  = A + beta k (v - A^T k)^T               (= (I - beta k k^T) A + beta k v^T)
//     o   = S'^T q = A^T q + beta (v - A^T k) (k . q)
// The two reductions over dk (A^T k and A^T q) are taken in one pass over the
// state, so S is read once and written once; o follows from the rank-1 update
// without a second pass.
//
// Mapping: one CTA of 256 threads per (n, h).  Warp w owns rows
// [w*DK/8, (w+1)*DK/8) of S; lane l owns DV/32 consecutive columns, loaded and
// stored as one 16-byte (DV=128) or 8-byte (DV=64) vector per row, so each warp
// instruction moves one full 512-byte (or 256-byte) row of S.  The whole state
// tile lives in registers between the read and the write.
#include "kda_common.cuh"

namespace kda {
namespace {

template <int CPT> struct VecF;
template <> struct VecF<4> { using T = float4; };
template <> struct VecF<2> { using T = float2; };

__device__ __forceinline__ void vload(const float* p, float (&x)[4]) {
  float4 t = __ldcs(reinterpret_cast<const float4*>(p));
  x[0] = t.x; x[1] = t.y; x[2] = t.z; x[3] = t.w;
}
__device__ __forceinline__ void vload(const float* p, float (&x)[2]) {
  float2 t = __ldcs(reinterpret_cast<const float2*>(p));
  x[0] = t.x; x[1] = t.y;
}
__device__ __forceinline__ void vstore(float* p, const float (&x)[4]) {
  __stcs(reinterpret_cast<float4*>(p), make_float4(x[0], x[1], x[2], x[3]));
}
__device__ __forceinline__ void vstore(float* p, const float (&x)[2]) {
  __stcs(reinterpret_cast<float2*>(p), make_float2(x[0], x[1]));
}

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

template <typename Tin, int DK, int DV>
__global__ void __launch_bounds__(kThreads, 2)
kda_decode_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k,
                  const Tin* __restrict__ v, const float* __restrict__ g,
                  const float* __restrict__ beta, float* __restrict__ S,
                  Tin* __restrict__ out) {
  constexpr int ROWS = DK / kWarps;   // rows of S per warp
  constexpr int CPT = DV / 32;        // columns per lane
  __shared__ float s_k[DK], s_q[DK], s_a[DK], s_v[DV];
  __shared__ float s_r[kWarps][DV], s_p[kWarps][DV];
  __shared__ float s_kq;

  const long long p = blockIdx.x;     // flat (n, h)
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  float* Sp = S + p * (long long)(DK * DV);
  const int col0 = lane * CPT;

  // Issue the state loads first: they do not depend on the small vectors.
  float x[ROWS][CPT];
#pragma unroll
  for (int i = 0; i < ROWS; ++i) vload(Sp + (warp * ROWS + i) * DV + col0, x[i]);

  for (int c = tid; c < DK; c += kThreads) {
    s_k[c] = to_f32(k[p * DK + c]);
    s_q[c] = to_f32(q[p * DK + c]);
    s_a[c] = expf(g[p * DK + c]);
  }
  for (int j = tid; j < DV; j += kThreads) s_v[j] = to_f32(v[p * DV + j]);
  __syncthreads();

  if (warp == 0) {
    float t = 0.f;
    for (int c = lane; c < DK; c += 32) t = fmaf(s_k[c], s_q[c], t);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
    if (lane == 0) s_kq = t;
  }

  float r[CPT], pq[CPT];
#pragma unroll
  for (int j = 0; j < CPT; ++j) { r[j] = 0.f; pq[j] = 0.f; }
#pragma unroll
  for (int i = 0; i < ROWS; ++i) {
    const int c = warp * ROWS + i;
    const float a = s_a[c], kc = s_k[c], qc = s_q[c];
#pragma unroll
    for (int j = 0; j < CPT; ++j) {
      x[i][j] *= a;
      r[j] = fmaf(x[i][j], kc, r[j]);
      pq[j] = fmaf(x[i][j], qc, pq[j]);
    }
  }
#pragma unroll
  for (int j = 0; j < CPT; ++j) { s_r[warp][col0 + j] = r[j]; s_p[warp][col0 + j] = pq[j]; }
  __syncthreads();

  const float b = beta[p];
  const float kq = s_kq;
  float u[CPT];
#pragma unroll
  for (int j = 0; j < CPT; ++j) {
    // pairwise tree ((0+1)+(2+3))+((4+5)+(6+7)) over the warps' partials
    const int c = col0 + j;
    const float rt = ((s_r[0][c] + s_r[1][c]) + (s_r[2][c] + s_r[3][c])) +
                     ((s_r[4][c] + s_r[5][c]) + (s_r[6][c] + s_r[7][c]));
    const float pt = ((s_p[0][c] + s_p[1][c]) + (s_p[2][c] + s_p[3][c])) +
                     ((s_p[4][c] + s_p[5][c]) + (s_p[6][c] + s_p[7][c]));
    u[j] = b * (s_v[col0 + j] - rt);
    if (warp == 0) out[p * DV + col0 + j] = from_f32<Tin>(fmaf(u[j], kq, pt));
  }
#pragma unroll
  for (int i = 0; i < ROWS; ++i) {
    const float kc = s_k[warp * ROWS + i];
#pragma unroll
    for (int j = 0; j < CPT; ++j) x[i][j] = fmaf(kc, u[j], x[i][j]);
    vstore(Sp + (warp * ROWS + i) * DV + col0, x[i]);
  }
}

// Multi-token decode: L consecutive tokens per (n, h) with the state held in
// registers, so S is read once and written once for all L tokens.  Warp w owns
// columns [w DV/8, (w+1) DV/8) of S over all rows, lane (g, c) = (lane / 4,
// lane % 4) the rows [g DK/8, (g+1) DK/8) and DV/32 of those columns, so the
// two reductions over dk are a per-lane partial followed by an xor-shuffle tree
// over the 8 row groups inside the warp: no barrier per token.  The single
// step above forms its partials over the same rows in the same order and adds
// the 8 partials in the same pairwise tree, so L tokens here give bit-for-bit
// the results of L single steps.  Token vectors are staged in shared memory 16
// tokens at a time (one barrier pair per 16 tokens).
constexpr int kTile = 16;

template <typename Tin, int DK, int DV>
__global__ void __launch_bounds__(kThreads, 2)
kda_decode_tokens_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k,
                         const Tin* __restrict__ v, const float* __restrict__ g,
                         const float* __restrict__ beta, float* __restrict__ S,
                         Tin* __restrict__ out, int L, int H, int gsh) {
  constexpr int R = DK / 8;           // rows per lane (one row group)
  constexpr int CPL = DV / 32;        // columns per lane
  // (a = exp(g), k, q) of row c = grp R + i at [t][i][grp]: the 8 row groups a
  // warp reads together are consecutive 16-byte words (no bank conflicts)
  __shared__ float4 s_akq[kTile][R][8];
  __shared__ float s_v[kTile][DV];
  __shared__ float s_b[kTile], s_kq[kTile];

  const long long p = blockIdx.x;     // flat (n, h)
  const long long n = p / H;
  const int h = (int)(p - n * H);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int grp = lane >> 2;
  const int col0 = warp * (DV / 8) + (lane & 3) * CPL;
  float* Sp = S + p * (long long)(DK * DV);

  float x[R][CPL];
#pragma unroll
  for (int i = 0; i < R; ++i) vload(Sp + (grp * R + i) * DV + col0, x[i]);

#pragma unroll 1
  for (int t0 = 0; t0 < L; t0 += kTile) {
    const int nt = min(kTile, L - t0);
    __syncthreads();                  // the previous tile's vectors are no longer read
    for (int e = tid; e < nt * DK; e += kThreads) {
      const int t = e / DK, c = e - t * DK;
      const long long row = (n * L + t0 + t) * H + h;
      s_akq[t][c % R][c / R] =
          make_float4(expf(g[row * (DK >> gsh) + (c >> gsh)]), to_f32(k[row * DK + c]),
                      to_f32(q[row * DK + c]), 0.f);
    }
    for (int e = tid; e < nt * DV; e += kThreads) {
      const int t = e / DV, j = e - t * DV;
      s_v[t][j] = to_f32(v[((n * L + t0 + t) * H + h) * DV + j]);
    }
    if (tid < nt) s_b[tid] = beta[(n * L + t0 + tid) * H + h];
    __syncthreads();
    // k . q per token, each by one warp, in the single step's order
    for (int t = warp; t < nt; t += kWarps) {
      float a = 0.f;
      for (int c = lane; c < DK; c += 32) a = fmaf(s_akq[t][c % R][c / R].y, s_akq[t][c % R][c / R].z, a);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
      if (lane == 0) s_kq[t] = a;
    }
    __syncthreads();
#pragma unroll 1
    for (int t = 0; t < nt; ++t) {
      float r[CPL], pq[CPL];
#pragma unroll
      for (int j = 0; j < CPL; ++j) { r[j] = 0.f; pq[j] = 0.f; }
#pragma unroll
      for (int i = 0; i < R; ++i) {
        const float4 akq = s_akq[t][i][grp];
#pragma unroll
        for (int j = 0; j < CPL; ++j) {
          x[i][j] *= akq.x;
          r[j] = fmaf(x[i][j], akq.y, r[j]);
          pq[j] = fmaf(x[i][j], akq.z, pq[j]);
        }
      }
      // pairwise tree over the 8 row groups (lanes 4 apart hold neighbouring groups)
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {
#pragma unroll
        for (int j = 0; j < CPL; ++j) {
          r[j] += __shfl_xor_sync(0xffffffffu, r[j], o);
          pq[j] += __shfl_xor_sync(0xffffffffu, pq[j], o);
        }
      }
      const float b = s_b[t], kq = s_kq[t];
      float u[CPL];
#pragma unroll
      for (int j = 0; j < CPL; ++j) {
        u[j] = b * (s_v[t][col0 + j] - r[j]);
        if (grp == 0)
          out[((n * L + t0 + t) * H + h) * DV + col0 + j] = from_f32<Tin>(fmaf(u[j], kq, pq[j]));
      }
#pragma unroll
      for (int i = 0; i < R; ++i) {
        const float kc = s_akq[t][i][grp].y;
#pragma unroll
        for (int j = 0; j < CPL; ++j) x[i][j] = fmaf(kc, u[j], x[i][j]);
      }
    }
  }
#pragma unroll
  for (int i = 0; i < R; ++i) vstore(Sp + (grp * R + i) * DV + col0, x[i]);
}

template <typename Tin, int DK, int DV>
cudaError_t launch_tokens_t(const void* q, const void* k, const void* v, const float* g,
                            const float* beta, float* S, void* out, long long pairs, int L, int H,
                            int gsh, cudaStream_t stream) {
  KDA_TIMED(KDA_KERNEL_DECODE, stream,
            kda_decode_tokens_kernel<Tin, DK, DV><<<(unsigned)pairs, kThreads, 0, stream>>>(
                static_cast<const Tin*>(q), static_cast<const Tin*>(k), static_cast<const Tin*>(v),
                g, beta, S, static_cast<Tin*>(out), L, H, gsh));
  note_launches(1);
  return cudaGetLastError();
}

template <typename Tin>
cudaError_t launch_tokens_dtype(const void* q, const void* k, const void* v, const float* g,
                                const float* beta, float* S, void* out, long long pairs, int L,
                                int H, int dk, int dv, int gsh, cudaStream_t stream) {
  if (dk == 128 && dv == 128)
    return launch_tokens_t<Tin, 128, 128>(q, k, v, g, beta, S, out, pairs, L, H, gsh, stream);
  if (dk == 128 && dv == 64)
    return launch_tokens_t<Tin, 128, 64>(q, k, v, g, beta, S, out, pairs, L, H, gsh, stream);
  if (dk == 64 && dv == 128)
    return launch_tokens_t<Tin, 64, 128>(q, k, v, g, beta, S, out, pairs, L, H, gsh, stream);
  return launch_tokens_t<Tin, 64, 64>(q, k, v, g, beta, S, out, pairs, L, H, gsh, stream);
}

template <typename Tin, int DK, int DV>
cudaError_t launch_t(const void* q, const void* k, const void* v, const float* g,
                     const float* beta, float* S, void* out, long long pairs,
                     cudaStream_t stream) {
  // pairs <= INT32_MAX by construction (N, H are ints and N*H is checked).
  KDA_TIMED(KDA_KERNEL_DECODE, stream,
            kda_decode_kernel<Tin, DK, DV><<<(unsigned)pairs, kThreads, 0, stream>>>(
                static_cast<const Tin*>(q), static_cast<const Tin*>(k), static_cast<const Tin*>(v),
                g, beta, S, static_cast<Tin*>(out)));
  note_launches(1);
  return cudaGetLastError();
}

template <typename Tin>
cudaError_t launch_dtype(const void* q, const void* k, const void* v, const float* g,
                         const float* beta, float* S, void* out, long long pairs, int dk,
                         int dv, cudaStream_t stream) {
  if (dk == 128 && dv == 128) return launch_t<Tin, 128, 128>(q, k, v, g, beta, S, out, pairs, stream);
  if (dk == 128 && dv == 64) return launch_t<Tin, 128, 64>(q, k, v, g, beta, S, out, pairs, stream);
  if (dk == 64 && dv == 128) return launch_t<Tin, 64, 128>(q, k, v, g, beta, S, out, pairs, stream);
  return launch_t<Tin, 64, 64>(q, k, v, g, beta, S, out, pairs, stream);
}

}  // namespace

cudaError_t launch_decode_tokens(const void* q, const void* k, const void* v, const float* g,
                                 const float* beta, float* S, void* out, int N, int L, int H,
                                 int dk, int dv, int in_dtype, int gsh, cudaStream_t stream) {
  const long long pairs = (long long)N * H;
  if (in_dtype == KDA_BF16)
    return launch_tokens_dtype<__nv_bfloat16>(q, k, v, g, beta, S, out, pairs, L, H, dk, dv,
                                              gsh, stream);
  return launch_tokens_dtype<float>(q, k, v, g, beta, S, out, pairs, L, H, dk, dv, gsh, stream);
}

cudaError_t launch_decode(const void* q, const void* k, const void* v, const float* g,
                          const float* beta, float* S, void* out, int N, int H, int dk,
                          int dv, int in_dtype, cudaStream_t stream) {
  const long long pairs = (long long)N * H;
  if (in_dtype == KDA_BF16)
    return launch_dtype<__nv_bfloat16>(q, k, v, g, beta, S, out, pairs, dk, dv, stream);
  return launch_dtype<float>(q, k, v, g, beta, S, out, pairs, dk, dv, stream);
}

}  // namespace kda
