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
// columns.  So a warp owns NC = 4 columns and all dk rows (lane l: rows
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

constexpr int NC = 4;             // state columns per warp
constexpr int WPC = 4;            // warps per CTA
constexpr int CPC = NC * WPC;     // state columns per CTA
constexpr int NTB = 32 * WPC;
constexpr int RING = 4;           // depth of the reverse sweep's state prefetch
constexpr unsigned FULL = 0xffffffffu;

// Sum over the 32 lanes of each of the 4 per-lane values p[j]; every lane gets
// all 4 totals.  Transpose-reduce (the halves exchanged at lane distance 16 and
// 8 leave each lane one column), three butterfly steps, then a gather.
__device__ __forceinline__ void colsum4(const float (&p)[4], float (&tot)[4], int lane) {
  const bool b4 = lane & 16, b3 = lane & 8;
  float x[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const float keep = b4 ? p[i + 2] : p[i];
    const float send = b4 ? p[i] : p[i + 2];
    x[i] = keep + __shfl_xor_sync(FULL, send, 16);
  }
  float z = (b3 ? x[1] : x[0]) + __shfl_xor_sync(FULL, b3 ? x[0] : x[1], 8);
  z += __shfl_xor_sync(FULL, z, 4);
  z += __shfl_xor_sync(FULL, z, 2);
  z += __shfl_xor_sync(FULL, z, 1);
  // lane holds column 2*b4 + b3
#pragma unroll
  for (int j = 0; j < 4; ++j) tot[j] = __shfl_sync(FULL, z, ((j >> 1) & 1) * 16 + (j & 1) * 8);
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

__device__ __forceinline__ void ld4(const float* p, float (&x)[4]) {
  const float4 a = *reinterpret_cast<const float4*>(p);
  x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
}
__device__ __forceinline__ void st4(float* p, const float (&x)[4]) {
  *reinterpret_cast<float4*>(p) = make_float4(x[0], x[1], x[2], x[3]);
}
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

// R (4 or 2) consecutive shared-memory elements as fp32
__device__ __forceinline__ void lds_n(const float* p, float (&x)[4]) { ld4(p, x); }
__device__ __forceinline__ void lds_n(const float* p, float (&x)[2]) {
  const float2 t = *reinterpret_cast<const float2*>(p);
  x[0] = t.x; x[1] = t.y;
}
__device__ __forceinline__ void lds_n(const __nv_bfloat16* p, float (&x)[4]) {
  const uint2 u = *reinterpret_cast<const uint2*>(p);
  x[0] = __uint_as_float(u.x << 16); x[1] = __uint_as_float(u.x & 0xffff0000u);
  x[2] = __uint_as_float(u.y << 16); x[3] = __uint_as_float(u.y & 0xffff0000u);
}
__device__ __forceinline__ void lds_n(const __nv_bfloat16* p, float (&x)[2]) {
  const uint32_t u = *reinterpret_cast<const uint32_t*>(p);
  x[0] = __uint_as_float(u << 16); x[1] = __uint_as_float(u & 0xffff0000u);
}

__device__ int g_chunk_bwd_timeout = 0;      // set if a chunk's inputs never arrived
constexpr uint32_t kWaitLimit = 1u << 22;

// Shared-memory layout (bytes).  NBUF chunk buffers of raw inputs, bulk-copied
// (g in fp32, turned into exp(g) in place once the chunk has landed; k, q, v and
// dout in their storage type; beta written by threads), then the per-warp e_t,
// the per-warp state ring and one mbarrier per buffer.  bf16 inputs use two
// buffers (the next chunk loads while this one is processed), fp32 inputs one.
template <typename Tin, int DK>
struct BwdSmem {
  static constexpr int NBUF = sizeof(Tin) == 2 ? 2 : 1;
  static constexpr int SI = (int)sizeof(Tin);
  static constexpr int G = 0;                                   // fp32 [64][DK >> gsh]
  static constexpr int K = G + kChunk * DK * 4;                 // Tin [64][DK]
  static constexpr int Q = K + kChunk * DK * SI;                // Tin [64][DK]
  static constexpr int V = Q + kChunk * DK * SI;                // Tin [64][CPC]
  static constexpr int DO = V + kChunk * CPC * SI;              // Tin [64][CPC]
  static constexpr int BETA = DO + kChunk * CPC * SI;           // fp32 [64]
  static constexpr int BUF = BETA + kChunk * 4;                 // bytes per buffer
  static constexpr int E = NBUF * BUF;                          // fp32 [WPC][64][NC]
  static constexpr int RINGB = E + WPC * kChunk * NC * 4;       // fp32 [WPC][RING][DK * NC]
  static constexpr int BAR = RINGB + WPC * RING * DK * NC * 4;  // uint64 [NBUF]
  static constexpr size_t BYTES = (size_t)BAR + 8 * NBUF;
  static_assert(BUF % 16 == 0 && CPC * SI % 16 == 0, "bulk copies need 16-byte pieces");
  // g rows of NG = DK >> gsh values go by bulk copy when 16-byte multiples
  static __device__ __forceinline__ bool g_bulk(int gsh) { return ((DK >> gsh) & 3) == 0; }
  static __device__ __forceinline__ uint32_t bytes(int L, bool rev, int gsh) {
    return (uint32_t)L * ((g_bulk(gsh) ? (DK >> gsh) * 4 : 0) + DK * SI + CPC * SI +
                          (rev ? DK * SI + CPC * SI : 0));
  }
};

// Start the bulk copies of tokens [0, L) of a chunk (first token row `rowbase`,
// head h) into buffer `buf`: g, k and this CTA's CPC columns of v, with `rev`
// also q and dout; completion on `bar`, whose transaction count the caller has
// set to BwdSmem::bytes(L, rev, gsh).  Two threads per token.  Returns, for the
// calling thread's token (threads 0 .. L-1): beta, and the token's g row when it
// is too short for a bulk copy (DK >> gsh <= 2 values); else zeros.
struct Staged {
  float beta, g0, g1;
};
template <typename Tin, int DK, int DV>
__device__ __forceinline__ Staged issue_chunk(char* buf, uint64_t* bar, const Tin* __restrict__ q,
                                              const Tin* __restrict__ k,
                                              const Tin* __restrict__ v,
                                              const float* __restrict__ g,
                                              const float* __restrict__ beta,
                                              const Tin* __restrict__ dout, long long rowbase,
                                              int L, int H, int h, int cta_c0, bool rev,
                                              int gsh) {
  using S = BwdSmem<Tin, DK>;
  static_assert(NTB == 2 * kChunk, "two threads per token");
  const int t = threadIdx.x & (kChunk - 1), part = threadIdx.x / kChunk;
  const int ng = DK >> gsh;
  Staged st{0.f, 0.f, 0.f};
  float& b = st.beta;
  if (t < L) {
    const long long row = (rowbase + t) * H + h;
    if (part == 0) {
      if (S::g_bulk(gsh)) {
        bulk_g2s(buf + S::G + t * ng * 4, g + row * ng, ng * 4, bar);
      } else {
        st.g0 = g[row * ng];
        if (ng > 1) st.g1 = g[row * ng + 1];
      }
      bulk_g2s(buf + S::K + t * DK * S::SI, k + row * DK, DK * S::SI, bar);
      if (rev) bulk_g2s(buf + S::Q + t * DK * S::SI, q + row * DK, DK * S::SI, bar);
      b = beta[row];
    } else {
      bulk_g2s(buf + S::V + t * CPC * S::SI, v + row * DV + cta_c0, CPC * S::SI, bar);
      if (rev) bulk_g2s(buf + S::DO + t * CPC * S::SI, dout + row * DV + cta_c0, CPC * S::SI, bar);
    }
  }
  return st;
}

// One CTA per (column block of CPC state columns, head, sequence).  GRP: grouped
// decay (gsh > 0); without it the kernel is compiled for per-channel g.
template <typename Tin, int DK, int DV, bool GRP>
__global__ void __launch_bounds__(NTB, 1)
kda_chunk_bwd_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k,
                     const Tin* __restrict__ v, const float* __restrict__ g,
                     const float* __restrict__ beta, const float* __restrict__ h0,
                     const int32_t* __restrict__ cu_seqlens, const Tin* __restrict__ dout,
                     const float* __restrict__ dhT, float* __restrict__ dq,
                     float* __restrict__ dk, float* __restrict__ dvo, float* __restrict__ dg,
                     float* __restrict__ dbeta, float* __restrict__ dh0,
                     float* __restrict__ ckpt, float* __restrict__ cst, int T, int H,
                     int gsh_arg) {
  const int gsh = GRP ? gsh_arg : 0;
  constexpr int R = DK / 32;            // state rows per lane
  constexpr int NV = R * NC / 4;        // float4 per lane in a warp's state slice
  constexpr int SLICE = DK * NC;        // floats in a warp's state slice
  constexpr int NB = DV / CPC;          // CTAs per (sequence, head)
  constexpr long long SZ = (long long)DK * DV;
  using SM = BwdSmem<Tin, DK>;
  constexpr int NBUF = SM::NBUF;
  extern __shared__ __align__(16) char smc[];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int bx = blockIdx.x, h = blockIdx.y, s = blockIdx.z;
  const int cta_c0 = bx * CPC, wc = warp * NC;
  const int c0 = cta_c0 + wc;           // this warp's first state column
  const int rl = lane * R;              // this lane's first state row
  long long row0, t_beg, t_end;
  seq_range(cu_seqlens, s, T, row0, t_beg, t_end);
  const long long len = t_end - t_beg;
  const int nch = (int)chunk_count(len);
  const long long sidx = ((long long)s * H + h) * SZ;
  // checkpoint of chunk c: ckpt + ck0 + c * H * SZ (chunks of all sequences numbered
  // consecutively, heads inside a chunk, warp slices inside a head)
  const long long ck0 =
      (seq_chunk_base(cu_seqlens, s, T) * H + h) * SZ + (long long)(bx * WPC + warp) * SLICE;
  // pre-token state of token t of the current chunk: cs + t * WPC * SLICE
  float* const cs = cst + ((((long long)s * H + h) * NB + bx) * kChunk * WPC + warp) * SLICE;
  float* const e_sm = reinterpret_cast<float*>(smc + SM::E) + warp * kChunk * NC;
  float* const ring = reinterpret_cast<float*>(smc + SM::RINGB) + warp * RING * SLICE;
  uint64_t* const bars = reinterpret_cast<uint64_t*>(smc + SM::BAR);

  // a warp's state slice: lane row i (NC = 4 columns) is float4 number i, at (i * 32 + lane) * 4
  auto st_slice = [&](float* base, const float (&X)[R][NC]) {
#pragma unroll
    for (int i = 0; i < R; ++i) st4(base + (i * 32 + lane) * 4, X[i]);
  };
  auto ld_slice = [&](const float* base, float (&X)[R][NC]) {
#pragma unroll
    for (int i = 0; i < R; ++i) ld4(base + (i * 32 + lane) * 4, X[i]);
  };

  // Jobs: the forward sweep's chunks 0 .. nch-2, then the reverse sweep's chunks
  // nch-1 .. 0.  Job j's inputs sit in buffer j % NBUF.
  const int nf = nch > 0 ? nch - 1 : 0;
  const int njobs = nf + nch;
  auto job_chunk = [&](int j) { return j < nf ? j : nch - 1 - (j - nf); };
  auto job_len = [&](int j) {
    return (int)min((long long)kChunk, len - (long long)job_chunk(j) * kChunk);
  };
  auto job_row = [&](int j) { return row0 + t_beg + (long long)job_chunk(j) * kChunk; };
  auto issue = [&](int j) {
    const int b = j % NBUF;
    return issue_chunk<Tin, DK, DV>(smc + b * SM::BUF, &bars[b], q, k, v, g, beta, dout,
                                    job_row(j), job_len(j), H, h, cta_c0, j >= nf, gsh);
  };
  const int ng = DK >> gsh;             // decay values per token (groups of 2^gsh channels)
  // the decay of this lane's rows at staged token t
  auto decay_rows = [&](const float* al_s, int t, float (&al)[R]) {
    if (!GRP) {
      lds_n(al_s + t * DK + rl, al);
    } else {
#pragma unroll
      for (int i = 0; i < R; ++i) al[i] = al_s[t * ng + ((rl + i) >> gsh)];
    }
  };

  if (tid == 0) {
#pragma unroll
    for (int b = 0; b < NBUF; ++b) mbar_init(&bars[b], 1);
    fence_mbar_init();
    if (njobs > 0) mbar_arrive_expect_tx(&bars[0], SM::bytes(job_len(0), 0 >= nf, gsh));
  }
  __syncthreads();
  Staged bnext = njobs > 0 ? issue(0) : Staged{0.f, 0.f, 0.f};
  uint32_t parity = 0;                  // bit b: parity of buffer b's next completion
  bool stalled = false;                 // a wait expired (diagnostic flag set)

  float S[R][NC], e[NC], G[R][NC];
#pragma unroll
  for (int i = 0; i < R; ++i) {
    if (h0) {
      ld4(h0 + sidx + (long long)(rl + i) * DV + c0, S[i]);
    } else {
#pragma unroll
      for (int j = 0; j < NC; ++j) S[i][j] = 0.f;
    }
    if (dhT) {
      ld4(dhT + sidx + (long long)(rl + i) * DV + c0, G[i]);
    } else {
#pragma unroll
      for (int j = 0; j < NC; ++j) G[i][j] = 0.f;
    }
  }

#pragma unroll 1
  for (int j = 0; j < njobs; ++j) {
    const int b = j % NBUF;
    char* const buf = smc + b * SM::BUF;
    const int c = job_chunk(j), L = job_len(j);
    const bool rev = j >= nf;
    const long long rb = job_row(j);
    // wait for the chunk, publish beta and exp(g), start the next chunk's copies
    if (!stalled && !mbar_wait(&bars[b], (parity >> b) & 1u, kWaitLimit)) {
      stalled = true;                   // wait no more: finish without blocking
      atomicExch(&g_chunk_bwd_timeout, 1);
    }
    parity ^= 1u << b;
    float* const al_s = reinterpret_cast<float*>(buf + SM::G);
    float* const beta_s = reinterpret_cast<float*>(buf + SM::BETA);
    if (tid < L) {
      beta_s[tid] = bnext.beta;
      if (!SM::g_bulk(gsh)) {
        al_s[tid * ng] = __expf(bnext.g0);
        if (ng > 1) al_s[tid * ng + 1] = __expf(bnext.g1);
      }
    }
    if (SM::g_bulk(gsh)) {
      for (int i = tid; i < L * ng / 4; i += NTB) {
        float4 x = reinterpret_cast<float4*>(al_s)[i];
        x.x = __expf(x.x); x.y = __expf(x.y); x.z = __expf(x.z); x.w = __expf(x.w);
        reinterpret_cast<float4*>(al_s)[i] = x;
      }
    }
    if (NBUF == 2 && tid == 0 && j + 1 < njobs)
      mbar_arrive_expect_tx(&bars[b ^ 1], SM::bytes(job_len(j + 1), j + 1 >= nf, gsh));
    __syncthreads();
    if (NBUF == 2 && j + 1 < njobs) bnext = issue(j + 1);

    const Tin* const k_s = reinterpret_cast<const Tin*>(buf + SM::K);
    const Tin* const q_s = reinterpret_cast<const Tin*>(buf + SM::Q);
    const Tin* const v_s = reinterpret_cast<const Tin*>(buf + SM::V);
    const Tin* const do_s = reinterpret_cast<const Tin*>(buf + SM::DO);
    // one forward step on token t: S <- a + beta k e^T, e = v - a^T k
    auto fwd = [&](int t) {
      float al[R], kr[R];
      decay_rows(al_s, t, al);
      lds_n(k_s + t * DK + rl, kr);
      float p[NC];
#pragma unroll
      for (int jj = 0; jj < NC; ++jj) p[jj] = 0.f;
#pragma unroll
      for (int i = 0; i < R; ++i)
#pragma unroll
        for (int jj = 0; jj < NC; ++jj) {
          S[i][jj] *= al[i];
          p[jj] = fmaf(S[i][jj], kr[i], p[jj]);
        }
      float tot[NC];
      colsum4(p, tot, lane);
      float vv[NC];
      lds_n(v_s + t * CPC + wc, vv);
      const float bt = beta_s[t];
#pragma unroll
      for (int jj = 0; jj < NC; ++jj) {
        e[jj] = vv[jj] - tot[jj];
        const float u = bt * e[jj];
#pragma unroll
        for (int i = 0; i < R; ++i) S[i][jj] = fmaf(kr[i], u, S[i][jj]);
      }
    };

    if (!rev) {
      // forward sweep: checkpoint, then the chunk's 64 tokens
      st_slice(ckpt + ck0 + (long long)c * H * SZ, S);
#pragma unroll 1
      for (int t = 0; t < L; ++t) fwd(t);
    } else {
      // the last chunk starts from the state the forward sweep ended with
      if (c != nch - 1) ld_slice(ckpt + ck0 + (long long)c * H * SZ, S);
      // re-run the chunk: pre-token states to scratch, e_t to shared, dq_t = S_t do_t
#pragma unroll 1
      for (int t = 0; t < L; ++t) {
        st_slice(cs + (long long)t * WPC * SLICE, S);
        fwd(t);
        if (lane == 0) st4(e_sm + t * NC, e);
        float dov[NC];
        lds_n(do_s + t * CPC + wc, dov);
        float dqp[R];
#pragma unroll
        for (int i = 0; i < R; ++i) {
          float acc = 0.f;
#pragma unroll
          for (int jj = 0; jj < NC; ++jj) acc = fmaf(S[i][jj], dov[jj], acc);
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
        float A[R][NC];                 // pre-token state S_{t-1} (a = Diag(alpha) A)
        ld_slice(ring + (t % RING) * SLICE, A);
        float al[R], kr[R], qr[R], dov[NC], ee[NC];
        decay_rows(al_s, t, al);
        lds_n(k_s + t * DK + rl, kr);
        lds_n(q_s + t * DK + rl, qr);
        lds_n(do_s + t * CPC + wc, dov);
        ld4(e_sm + t * NC, ee);
        const float bt = beta_s[t];
        float pw[NC];
#pragma unroll
        for (int jj = 0; jj < NC; ++jj) pw[jj] = 0.f;
#pragma unroll
        for (int i = 0; i < R; ++i)
#pragma unroll
          for (int jj = 0; jj < NC; ++jj) {
            G[i][jj] = fmaf(qr[i], dov[jj], G[i][jj]);
            pw[jj] = fmaf(G[i][jj], kr[i], pw[jj]);
          }
        float w[NC];
        colsum4(pw, w, lane);
        float de[NC], dbp = 0.f;
#pragma unroll
        for (int jj = 0; jj < NC; ++jj) {
          de[jj] = bt * w[jj];
          dbp = fmaf(w[jj], ee[jj], dbp);
        }
        const long long tok = (rb + t) * H + h;
        if (lane == 0) {
          st4(dvo + tok * DV + c0, de);
          atomicAdd(dbeta + tok, dbp);
        }
        // dk = beta G e - a de;  dg = rowsum((G - k de^T) * a);  G <- Diag(alpha)(G - k de^T),
        // with a = alpha_i A_ij: the row factor alpha_i is applied to the row sums
        float dkp[R], dgp[R];
#pragma unroll
        for (int i = 0; i < R; ++i) {
          float a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
          for (int jj = 0; jj < NC; ++jj) {
            a1 = fmaf(G[i][jj], ee[jj], a1);
            a2 = fmaf(A[i][jj], de[jj], a2);
            const float da = fmaf(-kr[i], de[jj], G[i][jj]);
            a3 = fmaf(da, A[i][jj], a3);
            G[i][jj] = al[i] * da;
          }
          dkp[i] = fmaf(bt, a1, -al[i] * a2);
          dgp[i] = al[i] * a3;
        }
        Rows<R>::add(dk + tok * DK + rl, dkp);
        if (!GRP) {
          Rows<R>::add(dg + tok * DK + rl, dgp);
        } else {                        // rows of one group add into one value
          float acc = 0.f;
#pragma unroll
          for (int i = 0; i < R; ++i) {
            acc += dgp[i];
            if (i == R - 1 || ((rl + i + 1) >> gsh) != ((rl + i) >> gsh)) {
              atomicAdd(dg + tok * ng + ((rl + i) >> gsh), acc);
              acc = 0.f;
            }
          }
        }
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
    // this buffer is refilled by bulk copies (async proxy) after the next barrier
    fence_async_smem();
    if (NBUF == 1 && j + 1 < njobs) {
      __syncthreads();
      if (tid == 0) mbar_arrive_expect_tx(&bars[0], SM::bytes(job_len(j + 1), j + 1 >= nf, gsh));
      __syncthreads();
      bnext = issue(j + 1);
    }
  }
  cp_async_wait_all();
  if (dh0) {
#pragma unroll
    for (int i = 0; i < R; ++i) st4(dh0 + sidx + (long long)(rl + i) * DV + c0, G[i]);
  }
}

template <typename Tin, int DK, int DV>
cudaError_t launch_t(const void* q, const void* k, const void* v, const float* g,
                     const float* beta, const float* h0, const int32_t* cu, const void* dout,
                     const float* dhT, float* dq, float* dk, float* dv, float* dg, float* dbeta,
                     float* dh0, float* ckpt, float* cst, int B, int T, int H, int gsh,
                     cudaStream_t stream) {
  constexpr size_t smem = BwdSmem<Tin, DK>::BYTES;
  auto kern = gsh > 0 ? kda_chunk_bwd_kernel<Tin, DK, DV, true>
                     : kda_chunk_bwd_kernel<Tin, DK, DV, false>;
  const cudaError_t ea = cudaFuncSetAttribute(kern,
                                              cudaFuncAttributeMaxDynamicSharedMemorySize,
                                              (int)smem);
  if (ea != cudaSuccess) return ea;
  KDA_TIMED(KDA_KERNEL_BWD, stream,
            kern<<<dim3(DV / CPC, H, B), NTB, smem, stream>>>(
                static_cast<const Tin*>(q), static_cast<const Tin*>(k), static_cast<const Tin*>(v),
                g, beta, h0, cu, static_cast<const Tin*>(dout), dhT, dq, dk, dv, dg, dbeta, dh0,
                ckpt, cst, T, H, gsh));
  note_launches(1);
  return cudaGetLastError();
}

template <typename Tin>
cudaError_t launch_dtype(const void* q, const void* k, const void* v, const float* g,
                         const float* beta, const float* h0, const int32_t* cu, const void* dout,
                         const float* dhT, float* dq, float* dk, float* dv, float* dg,
                         float* dbeta, float* dh0, float* ckpt, float* cst, int B, int T, int H,
                         int dkk, int dvv, int gsh, cudaStream_t stream) {
#define KDA_BWD_CASE(A, Bv)                                                                   \
  if (dkk == A && dvv == Bv)                                                                 \
    return launch_t<Tin, A, Bv>(q, k, v, g, beta, h0, cu, dout, dhT, dq, dk, dv, dg, dbeta, \
                                dh0, ckpt, cst, B, T, H, gsh, stream);
  KDA_BWD_CASE(128, 128)
  KDA_BWD_CASE(128, 64)
  KDA_BWD_CASE(64, 128)
  KDA_BWD_CASE(64, 64)
#undef KDA_BWD_CASE
  return cudaErrorInvalidValue;
}

}  // namespace

// Checkpoints: one state per chunk of every sequence, per head; and the pre-token
// states of one chunk per (sequence, head).
size_t chunk_bwd_scratch_bytes(int B, int T, int H, int dk, int dv, bool varlen) {
  const size_t nck = (size_t)(chunk_slots(B, T, varlen) + B) * H;
  const size_t ncs = (size_t)B * H * kChunk;
  return (nck + ncs) * (size_t)dk * dv * sizeof(float);
}

cudaError_t launch_chunk_bwd(const void* q, const void* k, const void* v, const float* g,
                             const float* beta, const float* h0, const int32_t* cu_seqlens,
                             const void* dout, const float* dhT, float* dq, float* dkk,
                             float* dvv, float* dg, float* dbeta, float* dh0, int B, int T, int H,
                             int dk, int dv, int gsh, int in_dtype, cudaStream_t stream,
                             const Workspace* ws) {
  int sms = 148;
  cudaMemPool_t pool = nullptr;
  if (!device_ctx(&sms, ws ? nullptr : &pool)) return cudaErrorInvalidDevice;
  if (!ws && !pool) return cudaErrorMemoryAllocation;
  const size_t need = chunk_bwd_scratch_bytes(B, T, H, dk, dv, cu_seqlens != nullptr);
  if (ws && (!ws->ptr || ws->bytes < need)) return cudaErrorInvalidValue;
  // dq, dk, dg and dbeta are sums of per-warp parts
  const size_t rows = cu_seqlens ? (size_t)T : (size_t)B * T;
  cudaError_t e = cudaSuccess;
  if (rows > 0) {
    const size_t n = rows * H * dk * sizeof(float);
    if ((e = cudaMemsetAsync(dq, 0, n, stream)) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(dkk, 0, n, stream)) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(dg, 0, n >> gsh, stream)) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(dbeta, 0, rows * H * sizeof(float), stream)) != cudaSuccess)
      return e;
  }
  const size_t sz = (size_t)dk * dv;
  const size_t nck = (size_t)(chunk_slots(B, T, cu_seqlens != nullptr) + B) * H;
  void* scratch = ws ? ws->ptr : nullptr;
  if (!ws) {
    e = cudaMallocFromPoolAsync(&scratch, need, pool, stream);
    if (e != cudaSuccess) return e;
  }
  float* ckpt = static_cast<float*>(scratch);
  float* cst = ckpt + nck * sz;
  if (in_dtype == KDA_BF16)
    e = launch_dtype<__nv_bfloat16>(q, k, v, g, beta, h0, cu_seqlens, dout, dhT, dq, dkk, dvv, dg,
                                    dbeta, dh0, ckpt, cst, B, T, H, dk, dv, gsh, stream);
  else
    e = launch_dtype<float>(q, k, v, g, beta, h0, cu_seqlens, dout, dhT, dq, dkk, dvv, dg, dbeta,
                            dh0, ckpt, cst, B, T, H, dk, dv, gsh, stream);
  if (!ws) cudaFreeAsync(scratch, stream);
  return e;
}

// Reads (and with reset clears) g_chunk_bwd_timeout; host side of kda_device_status.
cudaError_t take_bwd_timeout(int* flag, bool reset) {
  int v = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, g_chunk_bwd_timeout, sizeof(int));
  if (e == cudaSuccess && reset && v != 0) {
    const int zero = 0;
    e = cudaMemcpyToSymbol(g_chunk_bwd_timeout, &zero, sizeof(int));
  }
  *flag = v;
  return e;
}

}  // namespace kda
