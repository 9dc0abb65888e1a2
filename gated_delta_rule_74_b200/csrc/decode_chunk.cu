// Multi-token decode in the chunked form on the tensor cores (kda_decode_chunk).
//
// For each (sequence n, head h) the L <= 16 new tokens form one chunk of the
// chunked form (miniKimiK3 model card, "Kimi Delta Attention" bullet: the chunked
// parallel form equals the recurrence), applied to the stored state S:
//     Gamma = cumsum g;  Qbar = q e^Gamma;  Kbar = k e^Gamma;  Kend_i = k_i e^(Gamma_last - Gamma_i)
//     A_ri   = sum_c k_rc k_ic e^(Gamma_rc - Gamma_ic)   (i < r),   T = (I + diag(beta) A)^-1
//     Aqk_ri = sum_c q_rc k_ic e^(Gamma_rc - Gamma_ic)   (i <= r)
//     W = T diag(beta) Kbar,  U = T diag(beta) V,  Delta = U - W S
//     O = Qbar S + Aqk Delta,  S' = Diag(e^Gamma_last) S + Kend^T Delta.
// One CTA per (n, h), 256 threads.  The chunk-local quantities (16 tokens) are
// formed on the CUDA cores in fp32, with the decay differences split through token
// 8 (factors e^(+-(Gamma - Gamma_8))); a channel whose decay within tokens 0..8 or
// 8..15 exceeds kUnsafeDecay has that half's growing factor zeroed and the half's
// pairs added exactly (decay_pairs.cuh), so strong decay and closed gates stay
// exact.  The three products with
// the state run on the tensor cores with S^T resident in TMEM:
//     [O^T | P]   (128 x 32)  = S^T [Qbar ; W]^T          bf16 operands
//     S^T        (128 x 128) += Delta^T Kend              f16 operands
//     O^T        (128 x 16)  += Delta^T Aqk^T             f16 operands
// S is read from and written back to HBM once for all L tokens.  Tokens L .. 15
// are zero (q = k = v = g = beta = 0) and contribute nothing.
//
// TMEM (256 columns, two CTAs per SM): S^T fp32 [0, 128), [O^T | P] fp32
// [128, 160), S^T as bf16 pairs [160, 224), Delta^T as f16 pairs [224, 232).
#include <cuda_fp16.h>

#include "decay_pairs.cuh"
#include "kda_common.cuh"
#include "sm100.cuh"

namespace kda {

// Set when a bounded wait of the chunked decode gives up (diagnostic).
__device__ int g_decode_chunk_timeout = 0;

namespace {
using namespace sm100;
using bf16 = __nv_bfloat16;

constexpr int D = 128;                 // dk = dv
constexpr int LT = 16;                 // tokens per call (padded)
constexpr int NT = 256;
constexpr int LDF = D + 4;             // fp32 row stride of the token tiles (bank spread)
constexpr uint32_t kWaitLimit = 1u << 22;
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t T_S = 0, T_OP = 128, T_SB = 160, T_D = 224;

// shared memory (bytes, from a 1024-aligned base)
constexpr uint32_t M_B1 = 0;                      // [Qbar ; W] bf16, MN-major SW32, N 32 x K 128 (8 KB)
constexpr uint32_t M_KE = M_B1 + 8192;            // Kend f16, MN-major SW128, N 128 x K 16 (4 KB)
constexpr uint32_t M_AQ = M_KE + 4096;            // Aqk^T f16, MN-major SW32, N 16 x K 16 (512 B)
constexpr uint32_t M_F = M_AQ + 1024;             // fp32 tiles [16][LDF]
// q, k, v, Gamma, U = T beta V, and the Gram factors k e^(G - G_8), k e^(G_8 - G),
// q e^(G - G_8) (the first and last later hold Kbar = k e^G and W)
constexpr uint32_t F_Q = 0, F_K = 1, F_V = 2, F_G = 3, F_U = 4, F_KP = 5, F_KM = 6, F_QP = 7;
constexpr uint32_t M_SMALL = M_F + 8 * LT * LDF * 4;   // A, Aqk, T (16 x 16 fp32 each), beta, gamma_last
constexpr uint32_t DC_SMEM = M_SMALL + 3 * 256 * 4 + 64 + D * 4 + 1024;

// The exact pairs of one half (tokens t0 .. t0 + 7) of channel c, when `unsafe`,
// summed over the warp into the half's corrections (decay_pairs.cuh); the tiles
// hold k, q and g (row stride LDF).  Out of line: it runs only for inputs with
// strong decay and keeps its registers to itself.  Warp-cooperative.
__device__ __noinline__ void decode_unsafe_pairs(const float* fk, const float* fq, const float* fg,
                                                 int t0, int c, bool unsafe, float* cA, float* cQ,
                                                 int lane) {
  float al[8][1], kv[8][1], qv[8][1];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    al[e][0] = __expf(fg[(t0 + e) * LDF + c]);
    kv[e][0] = unsafe ? fk[(t0 + e) * LDF + c] : 0.f;
    qv[e][0] = unsafe ? fq[(t0 + e) * LDF + c] : 0.f;
  }
  add_pair_terms<1, 8>(al, kv, qv, cA, cQ, lane);
}

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}
// D (16 x 8, fp32) += A (16 x 16) B (16 x 8), bf16 operands: lane l holds A rows l/4 and
// l/4 + 8, columns 2 (l%4) + {0, 1} and + 8; B rows 2 (l%4) + {0, 1} and + 8, column l/4;
// D rows l/4 and l/4 + 8, columns 2 (l%4) + {0, 1}.
__device__ __forceinline__ void mma_bf16_16x8x16(float (&d)[4], const uint32_t (&a)[4],
                                                 const uint32_t (&b)[2]) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}
__device__ __forceinline__ uint4 pack8_f16v(const float (&x)[8]) {
  return make_uint4(pack_f16(x[0], x[1]), pack_f16(x[2], x[3]), pack_f16(x[4], x[5]),
                    pack_f16(x[6], x[7]));
}

__global__ void __launch_bounds__(NT, 2)
kda_decode_chunk_kernel(const bf16* __restrict__ q, const bf16* __restrict__ k,
                        const bf16* __restrict__ v, const float* __restrict__ g,
                        const float* __restrict__ beta, float* __restrict__ S,
                        bf16* __restrict__ out, int L, int H) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1024(smem_raw);
  __shared__ uint64_t mbar, sbar;
  __shared__ uint32_t tmem_base_sh;
  // exact within-half pairs of unsafe channels (A, Aqk: [r][i], 16 x 16)
  __shared__ __align__(16) float s_cA[LT * LT], s_cQ[LT * LT];
  float* const F = reinterpret_cast<float*>(sm + M_F);
  float* const Sf = F;                          // S [dk][dv] fp32 staged through the tile region
  float* const fq = F + F_Q * LT * LDF;          // q, later Qbar-ready raw q
  float* const fk = F + F_K * LT * LDF;          // k
  float* const fv = F + F_V * LT * LDF;          // v
  float* const fG = F + F_G * LT * LDF;          // g, then Gamma
  float* const fU = F + F_U * LT * LDF;          // U = T beta V
  float* const fKP = F + F_KP * LT * LDF;        // k e^(G - G_8), then Kbar = k e^G
  float* const fKM = F + F_KM * LT * LDF;        // k e^(G_8 - G)
  float* const fQP = F + F_QP * LT * LDF;        // q e^(G - G_8), then W
  float* const sA = reinterpret_cast<float*>(sm + M_SMALL);   // A [16][16] (row r, column i)
  float* const sAqk = sA + 256;                               // Aqk [16][16]
  float* const sT = sAqk + 256;                               // T beta [16][16]
  float* const sBeta = sT + 256;                              // [16]
  float* const sGl = sBeta + 16;                              // exp(Gamma_last) [128]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const long long pr = blockIdx.x;               // flat (n, h)
  const long long n = pr / H;
  const int h = (int)(pr - n * H);
  float* const Sp = S + pr * (long long)(D * D);

  if (warp == 0) {
    tmem_alloc(&tmem_base_sh, kTmemCols);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(&mbar, 1);
    mbar_init(&sbar, 1);
    fence_mbar_init();
    // S (64 KB contiguous) in one bulk copy into the tile region
    mbar_arrive_expect_tx(&sbar, D * D * 4);
    bulk_g2s(Sf, Sp, D * D * 4, &sbar);
  }
  // ---- the tokens (zeros beyond L) into registers meanwhile
  const int st_t = tid >> 4, st_c8 = tid & 15;   // token, 8-channel piece
  float xq[8], xk[8], xv[8], xg[8], xb = 0.f;
  {
    const int t = st_t, c8 = st_c8;
#pragma unroll
    for (int e = 0; e < 8; ++e) xq[e] = xk[e] = xv[e] = xg[e] = 0.f;
    if (t < L) {
      const long long row = (n * L + t) * H + h;
      const uint4 uq = __ldg(reinterpret_cast<const uint4*>(q + row * D + c8 * 8));
      const uint4 uk = __ldg(reinterpret_cast<const uint4*>(k + row * D + c8 * 8));
      const uint4 uv = __ldg(reinterpret_cast<const uint4*>(v + row * D + c8 * 8));
      const uint32_t wq4[4] = {uq.x, uq.y, uq.z, uq.w}, wk4[4] = {uk.x, uk.y, uk.z, uk.w},
                     wv4[4] = {uv.x, uv.y, uv.z, uv.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        xq[2 * e] = __uint_as_float(wq4[e] << 16); xq[2 * e + 1] = __uint_as_float(wq4[e] & 0xffff0000u);
        xk[2 * e] = __uint_as_float(wk4[e] << 16); xk[2 * e + 1] = __uint_as_float(wk4[e] & 0xffff0000u);
        xv[2 * e] = __uint_as_float(wv4[e] << 16); xv[2 * e + 1] = __uint_as_float(wv4[e] & 0xffff0000u);
      }
      const float4 g0 = __ldg(reinterpret_cast<const float4*>(g + row * D + c8 * 8));
      const float4 g1 = __ldg(reinterpret_cast<const float4*>(g + row * D + c8 * 8 + 4));
      xg[0] = g0.x; xg[1] = g0.y; xg[2] = g0.z; xg[3] = g0.w;
      xg[4] = g1.x; xg[5] = g1.y; xg[6] = g1.z; xg[7] = g1.w;
    }
    if (tid < LT && tid < L) xb = beta[(n * L + tid) * H + h];
    sA[tid] = 0.f;
    sAqk[tid] = 0.f;
    s_cA[tid] = 0.f;
    s_cQ[tid] = 0.f;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tb = tmem_base_sh;
  const int wq = warp >> 2;                       // column half of the TMEM tiles
  const int j = 32 * (warp & 3) + lane;           // TMEM lane = dv index
  const uint32_t tl = tb + ((uint32_t)((warp & 3) * 32) << 16);

  // ---- S -> S^T in TMEM and its bf16 copy: channels [64 wq, 64 wq + 64) of lane j,
  //      read from the staged copy (lanes read consecutive words: no bank conflict)
  bool s_ok = mbar_wait(&sbar, 0, kWaitLimit);
#pragma unroll 1
  for (int q4 = 0; q4 < 4; ++q4) {
    uint32_t f[16], pk[8];
    const int c0 = 64 * wq + 16 * q4;
#pragma unroll
    for (int e = 0; e < 16; ++e) f[e] = __float_as_uint(Sf[(c0 + e) * D + j]);
    tmem_st16(tl + T_S + c0, f);
#pragma unroll
    for (int e = 0; e < 8; ++e)
      pk[e] = pack_bf16(__uint_as_float(f[2 * e]), __uint_as_float(f[2 * e + 1]));
    tmem_st8(tl + T_SB + c0 / 2, pk);
  }
  tmem_wait_st();
  __syncthreads();                                // the staged S is consumed
  {
    const int t = st_t, c8 = st_c8;
    float* dq = fq + t * LDF + c8 * 8;
    float* dk = fk + t * LDF + c8 * 8;
    float* dv = fv + t * LDF + c8 * 8;
    float* dg = fG + t * LDF + c8 * 8;
    *reinterpret_cast<float4*>(dq) = make_float4(xq[0], xq[1], xq[2], xq[3]);
    *reinterpret_cast<float4*>(dq + 4) = make_float4(xq[4], xq[5], xq[6], xq[7]);
    *reinterpret_cast<float4*>(dk) = make_float4(xk[0], xk[1], xk[2], xk[3]);
    *reinterpret_cast<float4*>(dk + 4) = make_float4(xk[4], xk[5], xk[6], xk[7]);
    *reinterpret_cast<float4*>(dv) = make_float4(xv[0], xv[1], xv[2], xv[3]);
    *reinterpret_cast<float4*>(dv + 4) = make_float4(xv[4], xv[5], xv[6], xv[7]);
    *reinterpret_cast<float4*>(dg) = make_float4(xg[0], xg[1], xg[2], xg[3]);
    *reinterpret_cast<float4*>(dg + 4) = make_float4(xg[4], xg[5], xg[6], xg[7]);
    if (tid < LT) sBeta[tid] = xb;
  }
  __syncthreads();

  // ---- per channel c, two threads (tokens [0, 8) and [8, 16)): Gamma = cumsum g;
  //      exp(Gamma_last); the Gram factors k e^(G - G_8), k e^(G_8 - G), q e^(G - G_8)
  //      (each e^ clamped at 80); Kbar = k e^G (into the Gamma tile, once both threads
  //      have read g); the Qbar and Kend operand images
  bool unsafe = false;
  {
    const int c = tid & (D - 1), t0 = 8 * (tid >> 7);
    float G[LT];
    float acc = 0.f;
#pragma unroll
    for (int t = 0; t < LT; ++t) {
      acc += fG[t * LDF + c];
      G[t] = acc;
    }
    const float gl = acc;
    if (t0 == 0) sGl[c] = __expf(gl);
    // this half's growing factor: e^(G - G_8) over tokens 0..7, e^(G_8 - G) over 8..15
    unsafe = (t0 == 0 ? G[0] - G[8] : G[8] - G[15]) > kUnsafeDecay;
    // its pairs exactly (the factors below are zeroed for them); fG still holds g
    if (__any_sync(0xffffffffu, unsafe))
      decode_unsafe_pairs(fk, fq, fG, t0, c, unsafe, s_cA + t0 * LT + t0, s_cQ + t0 * LT + t0, lane);
    __syncthreads();
    float qb[8];                          // Qbar of these 8 tokens: one 16-byte chunk
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int t = t0 + i;
      const float Gt = t0 ? G[8 + i] : G[i];      // register-resident either way
      const float kt = fk[t * LDF + c], qt = fq[t * LDF + c];
      const float dG = Gt - G[8];
      float up = __expf(fminf(dG, 80.f)), dn = __expf(fminf(-dG, 80.f));
      if (unsafe) {                       // the growing factor of this half: zero
        if (t0 == 0) up = 0.f;
        else dn = 0.f;
      }
      const float eg = __expf(Gt);
      fKP[t * LDF + c] = kt * up;
      fKM[t * LDF + c] = kt * dn;
      fQP[t * LDF + c] = qt * up;
      fG[t * LDF + c] = kt * eg;                  // Kbar
      qb[i] = qt * eg;
      *reinterpret_cast<__half*>(sm + M_KE + off_mnmajor_sw128(c, t, LT)) =
          __float2half_rn(kt * __expf(gl - Gt));
    }
    *reinterpret_cast<uint4*>(sm + M_B1 + chunk_mnmajor_sw32(t0 >> 3, c, D)) =
        make_uint4(pack_bf16(qb[0], qb[1]), pack_bf16(qb[2], qb[3]), pack_bf16(qb[4], qb[5]),
                   pack_bf16(qb[6], qb[7]));
  }
  __syncthreads();

  // ---- Gram on warp-level tensor-core tiles (mma.sync m16n8k16, bf16 operands as in the
  //      prefill's Gram, fp32 accumulation): [q e^(G - G_8) ; k e^(G - G_8)] (32 x 128)
  //      against the rows of k e^(G_8 - G) (16 x 128).  Warp w < 4 takes the 16 x 8 tile
  //      (w >> 1, w & 1) and keeps Aqk(r, i <= r) resp. A(r, i < r); the products above
  //      the diagonal are not used.
  if (warp < 4) {
    const int gq = lane >> 2, tq = lane & 3;
    const float* X = (warp >> 1) ? fKP : fQP;
    const int n0 = 8 * (warp & 1);
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int k0 = 0; k0 < D; k0 += 16) {
      const float2 a0 = *reinterpret_cast<const float2*>(X + gq * LDF + k0 + 2 * tq);
      const float2 a1 = *reinterpret_cast<const float2*>(X + (gq + 8) * LDF + k0 + 2 * tq);
      const float2 a2 = *reinterpret_cast<const float2*>(X + gq * LDF + k0 + 2 * tq + 8);
      const float2 a3 = *reinterpret_cast<const float2*>(X + (gq + 8) * LDF + k0 + 2 * tq + 8);
      const float2 b0 = *reinterpret_cast<const float2*>(fKM + (n0 + gq) * LDF + k0 + 2 * tq);
      const float2 b1 = *reinterpret_cast<const float2*>(fKM + (n0 + gq) * LDF + k0 + 2 * tq + 8);
      const uint32_t af[4] = {pack_bf16(a0.x, a0.y), pack_bf16(a1.x, a1.y), pack_bf16(a2.x, a2.y),
                              pack_bf16(a3.x, a3.y)};
      const uint32_t bfr[2] = {pack_bf16(b0.x, b0.y), pack_bf16(b1.x, b1.y)};
      mma_bf16_16x8x16(acc, af, bfr);
    }
    const bool isq = (warp >> 1) == 0;
    float* dst = isq ? sAqk : sA;
    const float* cor = isq ? s_cQ : s_cA;   // exact pairs of unsafe channels (else zero)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int r = gq + 8 * (e >> 1), i = n0 + 2 * tq + (e & 1);
      if (isq ? i <= r : i < r) dst[r * LT + i] = acc[e] + cor[r * LT + i];
    }
  }
  __syncthreads();

  // ---- U = (I + diag(beta) A)^-1 diag(beta) V and W likewise with Kbar, by forward
  //      substitution, one column per thread: U_r = beta_r (V_r - sum_{i<r} A_ri U_i).
  //      Threads 0..127: U (kept in fp32 for Delta); 128..255: W (the bf16 operand
  //      image).  Threads 0..31 first write the Aqk^T operand image.
  if (tid < 32) {
    const int c8 = tid >> 4, i = tid & 15;
    float x[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) x[e] = sAqk[(8 * c8 + e) * LT + i];
    *reinterpret_cast<uint4*>(sm + M_AQ + chunk_mnmajor_sw32(c8, i, LT)) = pack8_f16v(x);
  }
  {
    const bool isw = tid >= D;
    const int c = tid & (D - 1);
    const float* src = isw ? fG : fv;             // Kbar or V
    float y[LT];
#pragma unroll
    for (int r = 0; r < LT; ++r) {
      float acc = src[r * LDF + c];
#pragma unroll
      for (int i4 = 0; i4 < (r + 3) / 4; ++i4) {          // row r of A, four at a time
        const float4 a4 = *reinterpret_cast<const float4*>(sA + r * LT + 4 * i4);
        const float av[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if (4 * i4 + e < r) acc = fmaf(-av[e], y[4 * i4 + e], acc);
      }
      y[r] = sBeta[r] * acc;
    }
    if (isw) {                          // tokens 0..7 and 8..15 of W: one 16-byte chunk each
#pragma unroll
      for (int h8 = 0; h8 < 2; ++h8)
        *reinterpret_cast<uint4*>(sm + M_B1 + chunk_mnmajor_sw32(2 + h8, c, D)) =
            make_uint4(pack_bf16(y[8 * h8], y[8 * h8 + 1]), pack_bf16(y[8 * h8 + 2], y[8 * h8 + 3]),
                       pack_bf16(y[8 * h8 + 4], y[8 * h8 + 5]), pack_bf16(y[8 * h8 + 6], y[8 * h8 + 7]));
    } else {
#pragma unroll
      for (int r = 0; r < LT; ++r) fU[r * LDF + c] = y[r];
    }
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  bool alive = __syncthreads_or(!s_ok) == 0;
  do {
    if (!alive) break;
    // ---- [O^T | P] = S^T [Qbar ; W]^T
    if (tid == 0) {
      const uint32_t id1 = idesc_bf16(128, 2 * LT, false, true);
      const uint32_t b1 = smem_u32(sm + M_B1);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk)
        mma_ts(tb + T_OP, tb + T_SB + kk * 8, desc_mnmajor_sw32(b1, D, kk), id1, kk > 0);
      mma_commit(&mbar);
    }
    __syncwarp();
    // meanwhile S^T <- S^T Diag(exp(Gamma_last))
#pragma unroll 1
    for (int q4 = 0; q4 < 4; ++q4) {
      uint32_t f[16];
      const int c0 = 64 * wq + 16 * q4;
      tmem_ld16(tl + T_S + c0, f);
      tmem_wait_ld();
#pragma unroll
      for (int e = 0; e < 16; ++e) f[e] = __float_as_uint(__uint_as_float(f[e]) * sGl[c0 + e]);
      tmem_st16(tl + T_S + c0, f);
    }
    tmem_wait_st();
    tc_fence_before();
    bool good = mbar_wait(&mbar, 0, kWaitLimit);
    tc_fence_after();
    if (__syncthreads_or(!good)) { alive = false; break; }

    // ---- Delta^T = U^T - P (lane j, 16 tokens) -> f16 pairs in TMEM
    if (wq == 0) {
      uint32_t pp[16];
      tmem_ld16(tl + T_OP + LT, pp);
      tmem_wait_ld();
      uint32_t dw[8];
#pragma unroll
      for (int e = 0; e < 8; ++e)
        dw[e] = pack_f16(fU[(2 * e) * LDF + j] - __uint_as_float(pp[2 * e]),
                         fU[(2 * e + 1) * LDF + j] - __uint_as_float(pp[2 * e + 1]));
      tmem_st8(tl + T_D, dw);
      tmem_wait_st();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // ---- S^T += Delta^T Kend;  O^T += Delta^T Aqk^T   (f16 A and B)
    if (tid == 0) {
      mma_ts(tb + T_S, tb + T_D, desc_mnmajor_sw128(smem_u32(sm + M_KE), LT, 0),
             idesc_f16(128, D, false, true), 1);
      mma_ts(tb + T_OP, tb + T_D, desc_mnmajor_sw32(smem_u32(sm + M_AQ), LT, 0),
             idesc_f16(128, LT, false, true), 1);
      mma_commit(&mbar);
    }
    __syncwarp();
    good = mbar_wait(&mbar, 1, kWaitLimit);
    tc_fence_after();
    if (__syncthreads_or(!good)) { alive = false; break; }

    // ---- outputs (tokens < L) and the new state
    if (wq == 0) {
      uint32_t o[16];
      tmem_ld16(tl + T_OP, o);
      tmem_wait_ld();
#pragma unroll
      for (int t = 0; t < LT; ++t)
        if (t < L) out[((n * L + t) * H + h) * D + j] = __float2bfloat16_rn(__uint_as_float(o[t]));
    }
    // the new state straight to HBM: lane j holds column j of S, so each warp's store
    // of one row of S covers 128 contiguous bytes
#pragma unroll 1
    for (int q4 = 0; q4 < 4; ++q4) {
      uint32_t f[16];
      const int c0 = 64 * wq + 16 * q4;
      tmem_ld16(tl + T_S + c0, f);
      tmem_wait_ld();
#pragma unroll
      for (int e = 0; e < 16; ++e) Sp[(long long)(c0 + e) * D + j] = __uint_as_float(f[e]);
    }
  } while (false);
  if (!alive && tid == 0) {
    atomicExch(&g_decode_chunk_timeout, 1);
    if (s_ok) mbar_wait(&mbar, 1, kWaitLimit);   // let an MMA still in flight finish
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tb, kTmemCols);
  }
}

}  // namespace

bool decode_chunk_supported(int dk, int dv, int in_dtype, int L) {
  return in_dtype == KDA_BF16 && dk == D && dv == D && L >= 1 && L <= LT;
}

cudaError_t launch_decode_chunk(const void* q, const void* k, const void* v, const float* g,
                                const float* beta, float* S, void* out, int N, int L, int H,
                                cudaStream_t stream) {
  if (!once_per_device(kOnceDecodeChunk, []() {
        return cudaFuncSetAttribute(kda_decode_chunk_kernel,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)DC_SMEM) == cudaSuccess;
      }))
    return cudaErrorInvalidDevice;
  const long long pairs = (long long)N * H;
  KDA_TIMED(KDA_KERNEL_DECODE, stream,
            kda_decode_chunk_kernel<<<(unsigned)pairs, NT, DC_SMEM, stream>>>(
                static_cast<const bf16*>(q), static_cast<const bf16*>(k),
                static_cast<const bf16*>(v), g, beta, S, static_cast<bf16*>(out), L, H));
  note_launches(1);
  return cudaGetLastError();
}

// Reads (and with reset clears) g_decode_chunk_timeout; host side of kda_device_status.
cudaError_t take_decode_chunk_timeout(int* flag, bool reset) {
  int v = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, g_decode_chunk_timeout, sizeof(int));
  if (e == cudaSuccess && reset && v != 0) {
    const int zero = 0;
    e = cudaMemcpyToSymbol(g_decode_chunk_timeout, &zero, sizeof(int));
  }
  *flag = v;
  return e;
}

}  // namespace kda
