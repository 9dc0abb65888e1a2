// KDA prefill, chunked (C = 64) form on the sm_100a tensor cores, dk = dv = 128,
// bf16 q/k/v, fp32 g/beta/state.
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
//     S_next   = Diag(exp(G_63)) S + Kend^T Delta,       Kend_i = exp(G_63 - G_i) k_i
// Rows past the end of a sequence are zero (k = q = v = beta = g = 0) and so
// contribute nothing.
//
// Decay factoring.  exp(G_r - G_i) is split through reference points so that no
// factor overflows: rows are grouped in 16-token blocks a; P_a = G at row 16a.
//   diagonal block (i, r in block a):  (k_r e^{G_r - P_a}) . (k_i e^{P_a - G_i})
//     first factor <= 1, second <= e^{decay over <= 15 tokens} (clamped at e^80)
//   i in an earlier block b < a:        (k_r e^{G_r - P_a}) . (k_i e^{P_a - G_i})
//     with e^{P_a - G_i} = e^{P_{b+1} - G_i} e^{P_a - P_{b+1}}, both <= 1.
// So the Gram of row block a is one MMA against R^(a) = [k_i e^{P_a - G_i}]_{i<16(a+1)}.
// The only range limit: within one 16-token block the cumulative log-decay must
// stay above -80 per channel (|g| below about 5 per token on average).
//
// Everything is computed transposed so that every MMA has M = 128 (the channel
// or value index on the TMEM lanes):
//   Gram   D^(a) [128 x 16(a+1)] = [Lk ; Lq] R^(a)^T       rows 0-63: A, 64-127: Aqk
//   W^T    [dk x 64] = Kbar^T (T beta)^T                    A operand in TMEM
//   U^T    [dv x 64] = V^T (T beta)^T
//   O^T    [dv x 64] = S^T Qbar^T + Delta^T Aqk^T           S^T, Delta^T in TMEM
//   P      [dv x 64] = S^T W^T          Delta^T = U^T - P
//   S^T   += Delta^T Kend   (after S^T <- S^T Diag(exp(G_63)))
// The state S^T [dv x dk] stays in TMEM in fp32 for the whole sequence; a bf16
// copy is the MMA operand.  The 64 x 64 triangular inverse runs on the CUDA
// cores in fp32 (16 x 16 diagonal blocks by forward substitution, then the
// off-diagonal blocks block-row by block-row).
//
// Mapping: one CTA (256 threads) per (sequence, head) walks the chunks in order.
// Threads 0-127 ("channel threads", thread c <-> key channel c = TMEM lane c)
// build the decayed operands; threads 128-255 ("value threads", j <-> value
// column j = TMEM lane j) own the state and the outputs.  Thread 0 issues the
// MMAs.  Packed documents restart the state from their own h0 slot and restart
// chunking at the document start (Mini-K3-1H-mamba2 card, packed-document
// paragraph: state flow resets at every boundary).
#include "kda_common.cuh"
#include "sm100.cuh"

namespace kda {

// Set when a bounded wait on the tensor cores gives up (diagnostic).
__device__ int g_chunk_tc_timeout = 0;

namespace {
using namespace sm100;
using bf16 = __nv_bfloat16;

constexpr int C = 64;
constexpr int D = 128;
constexpr int NT = 256;

// shared memory map (bytes from a 1024-aligned base)
// region A [0, 64K): staging during operand build, then the small operands
constexpr uint32_t OFF_SQ = 0, OFF_SK = 16384, OFF_SG = 32768;
constexpr uint32_t OFF_AQK = 0, OFF_TB = 8192, OFF_WT = 16384;
// region B [64K, 136K): Gram operands, then the triangular-solve scratch
constexpr uint32_t OFF_L = 65536;
// R^(a) buffers: N = 16(a+1) tokens x 128 channels, MN-major SW32 (4, 8, 12, 16 KB)
__host__ __device__ constexpr uint32_t off_r(int a) {
  return a == 0 ? 98304u : a == 1 ? 102400u : a == 2 ? 110592u : 122880u;
}
constexpr uint32_t OFF_A32 = 65536, OFF_T32 = 65536 + 17408, OFF_Y = 65536 + 34816;
constexpr int LDA = 65;   // padded fp32 row stride of the solve scratch
// region C [136K, 184K)
constexpr uint32_t OFF_V = 139264, OFF_QB = 155648, OFF_KE = 172032;
constexpr uint32_t SMEM_USED = 188416;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;

// TMEM columns (512 allocated)
constexpr uint32_t TM_S = 0;        // S^T fp32        [128 lanes x 128]
constexpr uint32_t TM_SB = 128;     // S^T bf16 (A)    [128 x 64]
constexpr uint32_t TM_KB = 192;     // Kbar^T bf16 (A) [128 x 32], later Delta^T bf16 (A)
constexpr uint32_t TM_G = 224;      // Gram D^(0..3) at +0, +16, +48, +96 (160 columns)
constexpr uint32_t TM_P = 224;      // P  [128 x 64] (after the Gram is read)
constexpr uint32_t TM_O = 288;      // O^T [128 x 64]
constexpr uint32_t TM_W = 384;      // W^T [128 x 64]
constexpr uint32_t TM_U = 448;      // U^T [128 x 64]
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kWaitLimit = 1u << 22;

__device__ __forceinline__ void st_shared_v4(uint8_t* base, uint32_t off, uint32_t a, uint32_t b,
                                             uint32_t c, uint32_t d) {
  *reinterpret_cast<uint4*>(base + off) = make_uint4(a, b, c, d);
}

__global__ void __launch_bounds__(NT, 1)
kda_chunk_tc_kernel(const bf16* __restrict__ q, const bf16* __restrict__ k,
                    const bf16* __restrict__ v, const float* __restrict__ g,
                    const float* __restrict__ beta, const float* h0,
                    const int32_t* __restrict__ cu_seqlens, bf16* __restrict__ out, float* hT,
                    int T, int H) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~uintptr_t(1023));
  __shared__ uint64_t bar;
  __shared__ uint32_t tmem_base_sh;
  __shared__ float s_beta[C];
  __shared__ float s_gamma[D];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = blockIdx.x, s = blockIdx.y;
  const bool is_val = tid >= 128;
  const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;

  long long row0, t_beg, t_end;
  if (cu_seqlens) {
    int a = cu_seqlens[s], b = cu_seqlens[s + 1];
    a = min(max(a, 0), T);
    b = min(max(b, a), T);
    row0 = 0; t_beg = a; t_end = b;
  } else {
    row0 = (long long)s * T; t_beg = 0; t_end = T;
  }
  const long long sbase = ((long long)s * H + h) * D * D;

  if (warp == 0) {
    tmem_alloc(&tmem_base_sh, kTmemCols);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tb = tmem_base_sh;
  uint32_t phase = 0;

  // ---- initial state: value thread j holds row j of S^T (= column j of S)
  if (is_val) {
    const int j = tid - 128;
#pragma unroll 1
    for (int c0 = 0; c0 < D; c0 += 32) {
      uint32_t f[16], f2[16], pk[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const float x0 = h0 ? h0[sbase + (long long)(c0 + e) * D + j] : 0.f;
        const float x1 = h0 ? h0[sbase + (long long)(c0 + 16 + e) * D + j] : 0.f;
        f[e] = __float_as_uint(x0);
        f2[e] = __float_as_uint(x1);
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        pk[e] = pack_bf16(__uint_as_float(f[2 * e]), __uint_as_float(f[2 * e + 1]));
        pk[8 + e] = pack_bf16(__uint_as_float(f2[2 * e]), __uint_as_float(f2[2 * e + 1]));
      }
      tmem_st16(tb + lane_base + TM_S + c0, f);
      tmem_st16(tb + lane_base + TM_S + c0 + 16, f2);
      tmem_st16(tb + lane_base + TM_SB + c0 / 2, pk);
    }
    tmem_wait_st();
  }
  tc_fence_before();
  __syncthreads();

  auto mma_wait = [&]() -> bool {
    bool good = mbar_wait(&bar, phase, kWaitLimit);
    phase ^= 1u;
    tc_fence_after();
    return __syncthreads_or(!good) == 0;
  };

  bool alive = true;
#pragma unroll 1
  for (long long t0 = t_beg; t0 < t_end && alive; t0 += C) {
    const int L = (int)min((long long)C, t_end - t0);

    // ================= P0: load the chunk (zero rows >= L) ==================
    {
#pragma unroll
      for (int it = 0; it < 4; ++it) {                      // q, k: 1024 chunks each
        const int idx = tid + it * NT;
        const int r = idx >> 4, ch = idx & 15;
        uint4 qa = make_uint4(0, 0, 0, 0), ka = make_uint4(0, 0, 0, 0);
        if (r < L) {
          const long long e = ((row0 + t0 + r) * H + h) * D + ch * 8;
          qa = __ldg(reinterpret_cast<const uint4*>(q + e));
          ka = __ldg(reinterpret_cast<const uint4*>(k + e));
        }
        *reinterpret_cast<uint4*>(sm + OFF_SQ + r * 256 + ch * 16) = qa;
        *reinterpret_cast<uint4*>(sm + OFF_SK + r * 256 + ch * 16) = ka;
      }
#pragma unroll
      for (int it = 0; it < 8; ++it) {                      // g: 2048 chunks
        const int idx = tid + it * NT;
        const int r = idx >> 5, ch = idx & 31;
        float4 ga = make_float4(0.f, 0.f, 0.f, 0.f);
        if (r < L) ga = __ldg(reinterpret_cast<const float4*>(g + ((row0 + t0 + r) * H + h) * D + ch * 4));
        *reinterpret_cast<float4*>(sm + OFF_SG + r * 512 + ch * 16) = ga;
      }
#pragma unroll
      for (int it = 0; it < 4; ++it) {                      // v -> MN-major SW128 (M = j, K = r)
        const int idx = tid + it * NT;
        const int r = idx >> 4, ch = idx & 15;
        uint4 va = make_uint4(0, 0, 0, 0);
        if (r < L) va = __ldg(reinterpret_cast<const uint4*>(v + ((row0 + t0 + r) * H + h) * D + ch * 8));
        *reinterpret_cast<uint4*>(sm + OFF_V + chunk_mnmajor_sw128(ch, r, C)) = va;
      }
      if (tid < C) s_beta[tid] = tid < L ? beta[(row0 + t0 + tid) * H + h] : 0.f;
    }
    __syncthreads();

    // ================= P1: decay scan and operand build (channel threads) ====
    if (!is_val) {
      const int c = tid;
      float* Gc = reinterpret_cast<float*>(sm + OFF_SG) + c;   // column c, row stride 128
      float acc = 0.f;
#pragma unroll 8
      for (int r = 0; r < C; ++r) { acc += Gc[r * D]; Gc[r * D] = acc; }
      const float P0 = Gc[0], P1 = Gc[16 * D], P2 = Gc[32 * D], P3 = Gc[48 * D], G63 = acc;
      const float P[4] = {P0, P1, P2, P3};
      s_gamma[c] = __expf(G63);
      float eP[4], eE1[3];
#pragma unroll
      for (int a = 0; a < 4; ++a) eP[a] = __expf(P[a]);
      eE1[0] = __expf(G63 - P1); eE1[1] = __expf(G63 - P2); eE1[2] = __expf(G63 - P3);
      // f1[a'][b] = e^{P_a' - P_{b+1}} for a' > b  (a' = b + 1 gives 1)
      const float f1_20 = __expf(P2 - P1), f1_30 = __expf(P3 - P1), f1_31 = __expf(P3 - P2);

      const bf16* kc = reinterpret_cast<const bf16*>(sm + OFF_SK) + c;
      const bf16* qc = reinterpret_cast<const bf16*>(sm + OFF_SQ) + c;
      uint32_t kb_words[32];
#pragma unroll
      for (int g8 = 0; g8 < 8; ++g8) {
        const int a = g8 >> 1;
        float lk[8], lq[8], ke[8], rd[8], ro1[8], ro2[8], ro3[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int r = g8 * 8 + e;
          const float Gr = Gc[r * D];
          const float x = Gr - P[a];
          const float ell = __expf(x);
          const float rho = __expf(fminf(-x, 80.f));
          const float sig = a < 3 ? __expf(P[a < 3 ? a + 1 : 3] - Gr) : __expf(G63 - Gr);
          const float kv = __bfloat162float(kc[r * D]);
          const float qv = __bfloat162float(qc[r * D]);
          lk[e] = kv * ell;
          lq[e] = qv * ell;
          ke[e] = a < 3 ? kv * sig * eE1[a < 3 ? a : 0] : kv * sig;
          rd[e] = kv * rho;
          const float ks = kv * sig;
          ro1[e] = ks;                                  // R^(a+1): factor 1
          ro2[e] = ks * (a == 0 ? f1_20 : f1_31);       // R^(a+2)
          ro3[e] = ks * f1_30;                          // R^(a+3) (a == 0 only)
        }
        // L = [Lk ; Lq]: A operand, MN-major SW128, M = 128, K = 128 rows (channels)
        st_shared_v4(sm, OFF_L + chunk_mnmajor_sw128(g8, c, D), pack_bf16(lk[0], lk[1]),
                     pack_bf16(lk[2], lk[3]), pack_bf16(lk[4], lk[5]), pack_bf16(lk[6], lk[7]));
        st_shared_v4(sm, OFF_L + chunk_mnmajor_sw128(8 + g8, c, D), pack_bf16(lq[0], lq[1]),
                     pack_bf16(lq[2], lq[3]), pack_bf16(lq[4], lq[5]), pack_bf16(lq[6], lq[7]));
        // Qbar^T: B operand, MN-major SW128, N = 64 (tokens), K = 128 (channels)
        const float ea = eP[a];
        st_shared_v4(sm, OFF_QB + chunk_mnmajor_sw128(g8, c, D), pack_bf16(lq[0] * ea, lq[1] * ea),
                     pack_bf16(lq[2] * ea, lq[3] * ea), pack_bf16(lq[4] * ea, lq[5] * ea),
                     pack_bf16(lq[6] * ea, lq[7] * ea));
        // Kbar^T: A operand in TMEM (lane c, 2 tokens per column)
#pragma unroll
        for (int e = 0; e < 4; ++e)
          kb_words[g8 * 4 + e] = pack_bf16(lk[2 * e] * ea, lk[2 * e + 1] * ea);
        // Kend^T: B operand, K-major SW128, N = 128 (channels), K = 64 (tokens)
        st_shared_v4(sm, OFF_KE + chunk_kmajor_sw128(c, g8, D), pack_bf16(ke[0], ke[1]),
                     pack_bf16(ke[2], ke[3]), pack_bf16(ke[4], ke[5]), pack_bf16(ke[6], ke[7]));
        // R^(a') for a' >= a: B operands, MN-major SW32, N = 16(a'+1), K = 128
        st_shared_v4(sm, off_r(a) + chunk_mnmajor_sw32(g8, c, D), pack_bf16(rd[0], rd[1]),
                     pack_bf16(rd[2], rd[3]), pack_bf16(rd[4], rd[5]), pack_bf16(rd[6], rd[7]));
        if (a + 1 <= 3)
          st_shared_v4(sm, off_r(a + 1) + chunk_mnmajor_sw32(g8, c, D),
                       pack_bf16(ro1[0], ro1[1]), pack_bf16(ro1[2], ro1[3]),
                       pack_bf16(ro1[4], ro1[5]), pack_bf16(ro1[6], ro1[7]));
        if (a + 2 <= 3)
          st_shared_v4(sm, off_r(a + 2) + chunk_mnmajor_sw32(g8, c, D),
                       pack_bf16(ro2[0], ro2[1]), pack_bf16(ro2[2], ro2[3]),
                       pack_bf16(ro2[4], ro2[5]), pack_bf16(ro2[6], ro2[7]));
        if (a + 3 <= 3)
          st_shared_v4(sm, off_r(3) + chunk_mnmajor_sw32(g8, c, D), pack_bf16(ro3[0], ro3[1]),
                       pack_bf16(ro3[2], ro3[3]), pack_bf16(ro3[4], ro3[5]),
                       pack_bf16(ro3[6], ro3[7]));
      }
      uint32_t w0[16], w1[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) { w0[e] = kb_words[e]; w1[e] = kb_words[16 + e]; }
      tmem_st16(tb + lane_base + TM_KB, w0);
      tmem_st16(tb + lane_base + TM_KB + 16, w1);
      tmem_wait_st();
      fence_async_smem();
    }
    tc_fence_before();
    __syncthreads();

    // ================= P2: Gram MMAs ==========================================
    if (tid == 0) {
      tc_fence_after();
      const uint32_t l_base = smem_u32(sm + OFF_L);
      uint32_t col = TM_G;
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        const uint32_t idesc = idesc_bf16(128, 16 * (a + 1), true, true);
        const uint32_t r_base = smem_u32(sm + off_r(a));
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss(tb + col, desc_mnmajor_sw128(l_base, D, kk), desc_mnmajor_sw32(r_base, D, kk),
                 idesc, kk > 0);
        col += 16 * (a + 1);
      }
      mma_commit(&bar);
    }
    __syncwarp();
    if (!mma_wait()) { alive = false; break; }

    // ================= P3: read A / Aqk, triangular inverse ===================
    float* A32 = reinterpret_cast<float*>(sm + OFF_A32);
    float* T32 = reinterpret_cast<float*>(sm + OFF_T32);
    float* Y32 = reinterpret_cast<float*>(sm + OFF_Y);
    if (!is_val) {
      // warp w reads TMEM lanes 32w..32w+31: w=0,1 -> A rows, w=2,3 -> Aqk rows
      const int r = (warp & 1) * 32 + lane;
      const bool isA = warp < 2;
      const int a_lo = (warp & 1) * 2;            // blocks a_lo, a_lo + 1 in this warp
      const int colA = a_lo == 0 ? 0 : 48;        // D^(a_lo) column offset in the Gram
      const int colB = a_lo == 0 ? 16 : 96;       // D^(a_lo+1)
      const int nA = 16 * (a_lo + 1), nB = 16 * (a_lo + 2);
      const int a_me = r >> 4;
      float vals[64];
#pragma unroll
      for (int i = 0; i < 64; ++i) vals[i] = 0.f;
      // first block of the pair
#pragma unroll
      for (int i0 = 0; i0 < 48; i0 += 16) {
        if (i0 < nA) {
          uint32_t t[16];
          tmem_ld16(tb + lane_base + TM_G + colA + i0, t);
          tmem_wait_ld();
          if (a_me == a_lo) {
#pragma unroll
            for (int e = 0; e < 16; ++e) vals[i0 + e] = __uint_as_float(t[e]);
          }
        }
      }
#pragma unroll
      for (int i0 = 0; i0 < 64; i0 += 16) {
        if (i0 < nB) {
          uint32_t t[16];
          tmem_ld16(tb + lane_base + TM_G + colB + i0, t);
          tmem_wait_ld();
          if (a_me == a_lo + 1) {
#pragma unroll
            for (int e = 0; e < 16; ++e) vals[i0 + e] = __uint_as_float(t[e]);
          }
        }
      }
      if (isA) {
#pragma unroll
        for (int i = 0; i < 64; ++i) A32[r * LDA + i] = (i < r) ? vals[i] : 0.f;
      } else {
        // Aqk: B operand of O^T += Delta^T Aqk^T, K-major SW128, N = 64 (r), K = 64 (i)
#pragma unroll
        for (int c8 = 0; c8 < 8; ++c8) {
          float w[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) w[e] = (c8 * 8 + e <= r) ? vals[c8 * 8 + e] : 0.f;
          st_shared_v4(sm, OFF_AQK + chunk_kmajor_sw128(r, c8, C), pack_bf16(w[0], w[1]),
                       pack_bf16(w[2], w[3]), pack_bf16(w[4], w[5]), pack_bf16(w[6], w[7]));
        }
      }
    }
    tc_fence_before();
    __syncthreads();

    // diagonal 16 x 16 blocks of T = (I + diag(beta) A)^-1 by forward substitution
    if (tid < 64) {
      const int a = tid >> 4, jj = tid & 15, o = 16 * a;
      float x[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) x[i] = (i == jj) ? 1.f : 0.f;
#pragma unroll
      for (int i = 1; i < 16; ++i) {
        float acc = 0.f;
#pragma unroll
        for (int m = 0; m < i; ++m) acc = fmaf(A32[(o + i) * LDA + o + m], x[m], acc);
        if (i > jj) x[i] = -s_beta[o + i] * acc;
      }
#pragma unroll
      for (int i = 0; i < 16; ++i) T32[(o + i) * LDA + o + jj] = x[i];
    }
    __syncthreads();
    // off-diagonal blocks, by distance d from the diagonal
#pragma unroll 1
    for (int d = 1; d < 4; ++d) {
      const int nblk = 4 - d;
      for (int idx = tid; idx < nblk * 256; idx += NT) {
        const int bi = idx >> 8, i = (idx >> 4) & 15, jj = idx & 15;
        const int a = bi + d, b = bi;
        const int row = 16 * a + i;
        float acc = 0.f;
        for (int m = 16 * b; m < 16 * a; ++m) acc = fmaf(A32[row * LDA + m], T32[m * LDA + 16 * b + jj], acc);
        Y32[idx] = s_beta[row] * acc;
      }
      __syncthreads();
      for (int idx = tid; idx < nblk * 256; idx += NT) {
        const int bi = idx >> 8, i = (idx >> 4) & 15, jj = idx & 15;
        const int a = bi + d, b = bi;
        float acc = 0.f;
#pragma unroll
        for (int mm = 0; mm < 16; ++mm)
          acc = fmaf(T32[(16 * a + i) * LDA + 16 * a + mm], Y32[(bi << 8) + (mm << 4) + jj], acc);
        T32[(16 * a + i) * LDA + 16 * b + jj] = -acc;
      }
      __syncthreads();
    }
    // T diag(beta) as bf16: B operand of W^T / U^T, K-major SW128, N = 64 (r'), K = 64 (r)
    for (int idx = tid; idx < C * 8; idx += NT) {
      const int rp = idx >> 3, c8 = idx & 7;
      float w[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const int r = c8 * 8 + e;
        w[e] = (r <= rp) ? T32[rp * LDA + r] * s_beta[r] : 0.f;
      }
      st_shared_v4(sm, OFF_TB + chunk_kmajor_sw128(rp, c8, C), pack_bf16(w[0], w[1]),
                   pack_bf16(w[2], w[3]), pack_bf16(w[4], w[5]), pack_bf16(w[6], w[7]));
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();

    // ================= P4: W^T, U^T, O^T = S^T Qbar^T ==========================
    if (tid == 0) {
      tc_fence_after();
      const uint32_t tb_base = smem_u32(sm + OFF_TB);
      const uint32_t v_base = smem_u32(sm + OFF_V);
      const uint32_t qb_base = smem_u32(sm + OFF_QB);
      const uint32_t id_w = idesc_bf16(128, 64, false, false);
      const uint32_t id_u = idesc_bf16(128, 64, true, false);
      const uint32_t id_o = idesc_bf16(128, 64, false, true);
#pragma unroll
      for (int kk = 0; kk < C / 16; ++kk) {
        const uint64_t bt = desc_kmajor_sw128(tb_base, C, kk);
        mma_ts(tb + TM_W, tb + TM_KB + kk * 8, bt, id_w, kk > 0);
        mma_ss(tb + TM_U, desc_mnmajor_sw128(v_base, C, kk), bt, id_u, kk > 0);
      }
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk)
        mma_ts(tb + TM_O, tb + TM_SB + kk * 8, desc_mnmajor_sw128(qb_base, D, kk), id_o, kk > 0);
      mma_commit(&bar);
    }
    __syncwarp();
    if (!mma_wait()) { alive = false; break; }

    // ================= P5: W^T -> bf16 smem; S^T <- S^T Diag(gamma) ===========
    if (!is_val) {
      const int c = tid;
#pragma unroll
      for (int r0 = 0; r0 < C; r0 += 16) {
        uint32_t t[16];
        tmem_ld16(tb + lane_base + TM_W + r0, t);
        tmem_wait_ld();
#pragma unroll
        for (int h8 = 0; h8 < 2; ++h8) {
          const float* f = reinterpret_cast<const float*>(t) + 8 * h8;
          st_shared_v4(sm, OFF_WT + chunk_mnmajor_sw128((r0 >> 3) + h8, c, D),
                       pack_bf16(f[0], f[1]), pack_bf16(f[2], f[3]), pack_bf16(f[4], f[5]),
                       pack_bf16(f[6], f[7]));
        }
      }
      fence_async_smem();
    } else {
#pragma unroll 1
      for (int c0 = 0; c0 < D; c0 += 16) {
        uint32_t t[16];
        tmem_ld16(tb + lane_base + TM_S + c0, t);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 16; ++e) t[e] = __float_as_uint(__uint_as_float(t[e]) * s_gamma[c0 + e]);
        tmem_st16(tb + lane_base + TM_S + c0, t);
      }
      tmem_wait_st();
    }
    tc_fence_before();
    __syncthreads();

    // ================= P6: P = S^T W^T ==========================================
    if (tid == 0) {
      tc_fence_after();
      const uint32_t wt_base = smem_u32(sm + OFF_WT);
      const uint32_t id_p = idesc_bf16(128, 64, false, true);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk)
        mma_ts(tb + TM_P, tb + TM_SB + kk * 8, desc_mnmajor_sw128(wt_base, D, kk), id_p, kk > 0);
      mma_commit(&bar);
    }
    __syncwarp();
    if (!mma_wait()) { alive = false; break; }

    // ================= P7: Delta^T = U^T - P -> bf16 TMEM (value threads) =====
    if (is_val) {
      uint32_t dw[32];
#pragma unroll
      for (int r0 = 0; r0 < C; r0 += 16) {
        uint32_t tu[16], tp[16];
        tmem_ld16(tb + lane_base + TM_U + r0, tu);
        tmem_ld16(tb + lane_base + TM_P + r0, tp);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 8; ++e)
          dw[r0 / 2 + e] = pack_bf16(__uint_as_float(tu[2 * e]) - __uint_as_float(tp[2 * e]),
                                     __uint_as_float(tu[2 * e + 1]) - __uint_as_float(tp[2 * e + 1]));
      }
      uint32_t w0[16], w1[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) { w0[e] = dw[e]; w1[e] = dw[16 + e]; }
      tmem_st16(tb + lane_base + TM_KB, w0);
      tmem_st16(tb + lane_base + TM_KB + 16, w1);
      tmem_wait_st();
    }
    tc_fence_before();
    __syncthreads();

    // ================= P8: S^T += Delta^T Kend; O^T += Delta^T Aqk^T ============
    if (tid == 0) {
      tc_fence_after();
      const uint32_t ke_base = smem_u32(sm + OFF_KE);
      const uint32_t aq_base = smem_u32(sm + OFF_AQK);
      const uint32_t id_s = idesc_bf16(128, 128, false, false);
      const uint32_t id_o = idesc_bf16(128, 64, false, false);
#pragma unroll
      for (int kk = 0; kk < C / 16; ++kk) {
        mma_ts(tb + TM_S, tb + TM_KB + kk * 8, desc_kmajor_sw128(ke_base, D, kk), id_s, 1);
        mma_ts(tb + TM_O, tb + TM_KB + kk * 8, desc_kmajor_sw128(aq_base, C, kk), id_o, 1);
      }
      mma_commit(&bar);
    }
    __syncwarp();
    if (!mma_wait()) { alive = false; break; }

    // ================= P9: outputs; bf16 copy of the new state =================
    if (is_val) {
      const int j = tid - 128;
#pragma unroll
      for (int r0 = 0; r0 < C; r0 += 16) {
        uint32_t t[16];
        tmem_ld16(tb + lane_base + TM_O + r0, t);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int r = r0 + e;
          if (r < L) out[((row0 + t0 + r) * H + h) * D + j] = __float2bfloat16_rn(__uint_as_float(t[e]));
        }
      }
#pragma unroll 1
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t t0w[16], t1w[16], pk[16];
        tmem_ld16(tb + lane_base + TM_S + c0, t0w);
        tmem_ld16(tb + lane_base + TM_S + c0 + 16, t1w);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          pk[e] = pack_bf16(__uint_as_float(t0w[2 * e]), __uint_as_float(t0w[2 * e + 1]));
          pk[8 + e] = pack_bf16(__uint_as_float(t1w[2 * e]), __uint_as_float(t1w[2 * e + 1]));
        }
        tmem_st16(tb + lane_base + TM_SB + c0 / 2, pk);
      }
      tmem_wait_st();
    }
    tc_fence_before();
    __syncthreads();
  }

  // ---- final state
  if (alive && is_val && hT) {
    const int j = tid - 128;
#pragma unroll 1
    for (int c0 = 0; c0 < D; c0 += 16) {
      uint32_t t[16];
      tmem_ld16(tb + lane_base + TM_S + c0, t);
      tmem_wait_ld();
#pragma unroll
      for (int e = 0; e < 16; ++e) hT[sbase + (long long)(c0 + e) * D + j] = __uint_as_float(t[e]);
    }
  }
  if (!alive && tid == 0) {
    atomicExch(&g_chunk_tc_timeout, 1);
    // let any MMA still in flight finish before the TMEM is released
    mbar_wait(&bar, phase, kWaitLimit);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tb, kTmemCols);
  }
}

}  // namespace

bool chunk_tc_supported(int dk, int dv, int in_dtype) {
  return in_dtype == KDA_BF16 && dk == D && dv == D;
}

cudaError_t launch_chunk_tc(const void* q, const void* k, const void* v, const float* g,
                            const float* beta, const float* h0, const int32_t* cu_seqlens,
                            void* out, float* hT, int B, int T, int H, cudaStream_t stream) {
  cudaError_t e = cudaFuncSetAttribute(kda_chunk_tc_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
  if (e != cudaSuccess) return e;
  dim3 grid(H, B);
  kda_chunk_tc_kernel<<<grid, NT, SMEM_BYTES, stream>>>(
      static_cast<const bf16*>(q), static_cast<const bf16*>(k), static_cast<const bf16*>(v), g,
      beta, h0, cu_seqlens, static_cast<bf16*>(out), hT, T, H);
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace kda
