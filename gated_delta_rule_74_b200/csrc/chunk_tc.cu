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
// Rows past the end of a sequence are zero (k = q = beta = g = 0) and so
// contribute nothing.
//
// Decay factoring.  exp(G_r - G_i) is split through reference points so that no
// factor overflows: rows are grouped in 16-token blocks a; P_a = G at row 16a.
//   i, r in block a:   (k_r e^{G_r - P_a}) (k_i e^{P_a - G_i})
//       first factor <= 1; second <= e^{decay inside the block}
//   i in block b < a:  (k_r e^{G_r - P_a}) (k_i e^{P_a - G_i}),  e^{P_a - G_i} <= 1
// So the Gram of row block a is one MMA against R^(a) = [k_i e^{P_a - G_i}]_{i<16(a+1)}.
// A channel whose decay inside block a exceeds kUnsafeDecay (strong decay, or a
// gate that closes) has its within-block entries of R^(a) zeroed; those pairs are
// added exactly on the CUDA cores (decay_pairs.cuh), and its other factors
// (R^(a') for a' > a, Kend) are formed directly, each <= 1.  Exponents are taken as
// differences of per-half sums, so a closed gate (g -> -1e4) in the first half of
// the chunk costs no precision in the second.
//
// Everything is computed transposed so that every MMA has M = 128 (the channel
// or value index on the TMEM lanes):
//   Gram   [D^(0) .. D^(3)] [128 x 160] = [Lk ; Lq] [R^(0); ..; R^(3)]^T
//          (rows 0-63: A, rows 64-127: Aqk; row block a is read from D^(a))
//   W^T    [dk x 64] = Kbar^T (T beta)^T                    A operand in TMEM
//   U^T    [dv x 64] = V^T (T beta)^T
//   [O^T | P]   [dv x 128] = S^T [Qbar^T | W^T]^T            S^T (bf16 copy) in TMEM
//   Delta^T = U^T - P
//   [S^T | O^T] [dv x 192] += Delta^T [Kend^T ; Aqk]^T      (after S^T <- S^T Diag(exp(G_63)))
// Products that share an operand are merged into one wide MMA: each tcgen05.mma
// costs about the same whatever its N, so fewer, wider instructions are faster.
// The state S^T [dv x dk] stays in TMEM in fp32 for the whole sequence; a bf16
// copy is the MMA operand.  The 64 x 64 triangular inverse runs on the CUDA
// cores in fp32: 16 x 16 diagonal blocks by forward substitution, then
// T_ab = -sum_{m=b}^{a-1} (T_aa B_am) T_mb block-row by block-row.
//
// Mapping: one CTA (256 threads) per (sequence, head) walks the chunks in order.
// The next chunk's inputs are fetched with cp.async while the current chunk
// computes.  Threads 0-127 map to key channels / TMEM lanes for the operands
// with M = dk; threads 128-255 own the state rows S^T[j] and the outputs.
// Thread 0 issues the MMAs.  Packed documents restart the state from their own
// h0 slot and restart chunking at the document start (Mini-K3-1H-mamba2 card,
// packed-document paragraph: state flow resets at every boundary).
#include <mutex>
#include <type_traits>

#include "decay_pairs.cuh"
#include "kda_common.cuh"
#include "segments.cuh"
#include "sm100.cuh"

namespace kda {

// Set when a bounded wait on the tensor cores gives up (diagnostic).
__device__ int g_chunk_tc_timeout = 0;

namespace {
using namespace sm100;
using bf16 = __nv_bfloat16;

constexpr int C = kChunk;
constexpr int D = kHead;
constexpr int NT = 256;

// ---- shared memory map (bytes from a 1024-aligned base)
// region A [0, 64K): cp.async staging of q, k (bf16 row-major) and g (fp32)
constexpr uint32_t OFF_SQ = 0, OFF_SK = 16384, OFF_SG = 32768;
// region B [64K, 136K): Gram operands during the build ...
constexpr uint32_t OFF_L = 65536;                       // [Lk; Lq], 32 KB
__host__ __device__ constexpr uint32_t off_r(int a) {   // R^(a): 4, 8, 12, 16 KB
  return a == 0 ? 98304u : a == 1 ? 102400u : a == 2 ? 110592u : 122880u;
}
// ... then, once the Gram has been read: solve scratch and small operands
constexpr int LDA = 68;                                 // fp32 row stride (16-byte rows)
constexpr uint32_t OFF_B32 = 65536;                     // diag(beta) A, fp32
constexpr uint32_t OFF_T32 = 65536 + 17408;             // T, fp32
constexpr uint32_t OFF_M32 = 65536 + 34816;             // T_aa B_am, 6 x 16 x 16 fp32
constexpr uint32_t OFF_TB = 114688;                      // T diag(beta), bf16 K-major
constexpr uint32_t OFF_OUT = 65536;                     // output tile (after the solve)
// region C [136K, 184K)
// region C [136K, 208K): V; then [Qbar^T | W^T] as one MN-major B operand of
// N = 128 (two 64-wide blocks, 16 KB apart); then [Kend^T ; Aqk] as one K-major B
// operand of 192 rows (Kend^T rows 0-127, Aqk rows 128-191)
constexpr uint32_t OFF_V = 139264, OFF_QB = 155648, OFF_WT = OFF_QB + 16384;
constexpr uint32_t OFF_KE = 188416, OFF_AQK = OFF_KE + 16384;
constexpr uint32_t SMEM_USED = 212992;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;

// ---- TMEM columns (512 allocated)
// [S^T | O^T] and [O^T | P] are each the accumulator of one MMA, so O^T sits
// between S^T and P.
constexpr uint32_t TM_S = 0;        // S^T fp32        [128 lanes x 128]
constexpr uint32_t TM_O = 128;      // O^T             [128 x 64]
constexpr uint32_t TM_P = 192;      // P               [128 x 64]
constexpr uint32_t TM_SB = 256;     // S^T bf16 (A)    [128 x 64]
constexpr uint32_t TM_KB = 320;     // Kbar^T bf16 (A) [128 x 32], later Delta^T f16 (A)
constexpr uint32_t TM_G = 352;      // Gram D^(0..3) at +0, +16, +48, +96 (160 columns)
constexpr uint32_t TM_W = 352;      // W^T [128 x 64]  (after the Gram is read)
constexpr uint32_t TM_U = 416;      // U^T [128 x 64]
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kWaitLimit = 1u << 22;

__device__ __forceinline__ void st_v4(uint8_t* base, uint32_t off, uint32_t a, uint32_t b,
                                      uint32_t c, uint32_t d) {
  *reinterpret_cast<uint4*>(base + off) = make_uint4(a, b, c, d);
}
__device__ __forceinline__ void st_v4f(uint8_t* base, uint32_t off, const float (&x)[8], float s) {
  st_v4(base, off, pack_bf16(x[0] * s, x[1] * s), pack_bf16(x[2] * s, x[3] * s),
        pack_bf16(x[4] * s, x[5] * s), pack_bf16(x[6] * s, x[7] * s));
}
// the same as f16: [Kend^T ; Aqk] and Delta^T are f16 (the state update runs in
// kind::f16 with f16 A and B, for the finer rounding)
__device__ __forceinline__ void st_v4h(uint8_t* base, uint32_t off, const float (&x)[8], float s) {
  st_v4(base, off, pack_f16(x[0] * s, x[1] * s), pack_f16(x[2] * s, x[3] * s),
        pack_f16(x[4] * s, x[5] * s), pack_f16(x[6] * s, x[7] * s));
}

// Issue the cp.async loads of one chunk's q, k, g into the staging region
// (rows >= L zero-filled; their source address is clamped in bounds).
__device__ __forceinline__ void prefetch_qkg(uint8_t* sm, const bf16* q, const bf16* k,
                                             const float* g, long long rowbase, int L, int H,
                                             int h, int tid) {
#pragma unroll
  for (int it = 0; it < 4; ++it) {
    const int idx = tid + it * NT;
    const int r = idx >> 4, ch = idx & 15;
    const long long e = ((rowbase + min(r, L - 1)) * H + h) * D + ch * 8;
    const uint32_t n = r < L ? 16u : 0u;
    cp_async16(sm + OFF_SQ + r * 256 + ch * 16, q + e, n);
    cp_async16(sm + OFF_SK + r * 256 + ch * 16, k + e, n);
  }
#pragma unroll
  for (int it = 0; it < 8; ++it) {
    const int idx = tid + it * NT;
    const int r = idx >> 5, ch = idx & 31;
    const long long e = ((rowbase + min(r, L - 1)) * H + h) * D + ch * 4;
    cp_async16(sm + OFF_SG + r * 512 + ch * 16, g + e, r < L ? 16u : 0u);
  }
}
// v rows go straight into the MN-major SW128 operand layout (M = value j, K = token).
__device__ __forceinline__ void prefetch_v(uint8_t* sm, const bf16* v, long long rowbase, int L,
                                           int H, int h, int tid) {
#pragma unroll
  for (int it = 0; it < 4; ++it) {
    const int idx = tid + it * NT;
    const int r = idx >> 4, ch = idx & 15;
    const long long e = ((rowbase + min(r, L - 1)) * H + h) * D + ch * 8;
    cp_async16(sm + OFF_V + chunk_mnmajor_sw128(ch, r, C), v + e, r < L ? 16u : 0u);
  }
}

// Per 16-row block lb of a thread's half (block a = 2 HF + lb), channel c: the
// reference P_a in the half's local frame (x = gv[r] - ref), e^{P_a}, G_63 - P_a and
// its exponential, P_{a2} - P_a and its exponential for a2 > a, and whether the
// block's decay is too strong for the split.
struct BlockRefs {
  float ref[2], eP[2], tl[2], eE[2], dd[2][4], f[2][4];
  bool uns[2];
};

// Operand build for rows [32*HF, 32*HF + 32) of the chunk, key channel c; gv holds
// the cumulative log-decay of those rows from the start of the half.
template <int HF>
__device__ __forceinline__ void build_half(uint8_t* sm, const float (&gv)[32], const bf16* kc,
                                           const bf16* qc, int c, const BlockRefs& br,
                                           uint32_t tm_kb) {
  uint32_t kbw[16];
#pragma unroll
  for (int lb = 0; lb < 2; ++lb) {
    const int a = 2 * HF + lb;
    const float eP = br.eP[lb];                  // Kbar, Qbar: e^{G_r} = e^{G_r - P_a} e^{P_a}
    const float eE = br.eE[lb];                  // Kend: e^{G63 - G_i} = e^{P_a - G_i} e^{G63 - P_a}
    const bool uns = br.uns[lb];
#pragma unroll
    for (int gg = 0; gg < 2; ++gg) {
      const int g8 = 2 * a + gg;                 // global group of 8 rows
      float lk[8], lq[8], kr[8], kv[8], xs[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const int r = g8 * 8 + e;
        const float x = gv[r - 32 * HF] - br.ref[lb];
        const float ell = __expf(x);
        const float rho = __expf(fminf(-x, 80.f));
        kv[e] = __bfloat162float(kc[r * D]);
        const float qv = __bfloat162float(qc[r * D]);
        xs[e] = x;
        lk[e] = kv[e] * ell;
        lq[e] = qv * ell;
        kr[e] = kv[e] * rho;                     // k_i e^{P_a - G_i}
      }
      // L = [Lk ; Lq]: A operand of the Gram, MN-major SW128 (M = 128, K = channels)
      st_v4f(sm, OFF_L + chunk_mnmajor_sw128(g8, c, D), lk, 1.f);
      st_v4f(sm, OFF_L + chunk_mnmajor_sw128(8 + g8, c, D), lq, 1.f);
      // Qbar^T: B operand of O^T, MN-major SW128 (N = tokens, K = channels)
      st_v4f(sm, OFF_QB + chunk_mnmajor_sw128(g8, c, D), lq, eP);
      if (!uns) {
        // Kend^T: B operand of the state update, K-major SW128 (N = channels, K = tokens)
        st_v4h(sm, OFF_KE + chunk_kmajor_sw128(c, g8, D), kr, eE);
        // R^(a'), a' >= a: B operands of the Gram, MN-major SW32 (N = 16(a'+1), K = channels)
#pragma unroll
        for (int a2 = a; a2 < 4; ++a2)
          st_v4f(sm, off_r(a2) + chunk_mnmajor_sw32(g8, c, D), kr, br.f[lb][a2]);
      } else {
        // unsafe: no within-block entries; later blocks' factors and Kend directly
        st_v4(sm, off_r(a) + chunk_mnmajor_sw32(g8, c, D), 0u, 0u, 0u, 0u);
#pragma unroll
        for (int a2 = a + 1; a2 < 4; ++a2) {
          float r2[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) r2[e] = kv[e] * __expf(fminf(br.dd[lb][a2] - xs[e], 0.f));
          st_v4f(sm, off_r(a2) + chunk_mnmajor_sw32(g8, c, D), r2, 1.f);
        }
        float ke[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) ke[e] = kv[e] * __expf(fminf(br.tl[lb] - xs[e], 0.f));
        st_v4h(sm, OFF_KE + chunk_kmajor_sw128(c, g8, D), ke, 1.f);
      }
      // Kbar^T: A operand in TMEM, lane c, two tokens per 32-bit column
#pragma unroll
      for (int e = 0; e < 4; ++e)
        kbw[(lb * 2 + gg) * 4 + e] = pack_bf16(lk[2 * e] * eP, lk[2 * e + 1] * eP);
    }
  }
  tmem_st16(tm_kb + 16 * HF, kbw);
}

__global__ void __launch_bounds__(NT, 1)
kda_chunk_tc_kernel(const bf16* __restrict__ q, const bf16* __restrict__ k,
                    const bf16* __restrict__ v, const float* __restrict__ g,
                    const float* __restrict__ beta, const float* h0,
                    const int32_t* __restrict__ cu_seqlens, bf16* __restrict__ out, float* hT,
                    int T, int H, SegArgs sa) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~uintptr_t(1023));
  __shared__ uint64_t bar;
  __shared__ uint32_t tmem_base_sh;
  __shared__ float s_beta[C];
  __shared__ float s_gamma[D];
  // per channel, each half's local cumulative log-decay at its rows 0, 16, 31
  __shared__ float s_pref[6][D];
  // exact within-block pairs of unsafe channels: A at [block][r][i], then Aqk
  __shared__ __align__(16) float s_corr[2 * 4 * 256];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = blockIdx.x, s = blockIdx.y;
  const bool upper = tid >= 128;       // second warpgroup
  const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;

  long long row0, t_beg, t_end;
  seq_range(cu_seqlens, s, T, row0, t_beg, t_end);
  // what this CTA computes: a token range, where its state starts, where it ends
  const long long hoff = ((long long)s * H + h) * D * D;
  const float* init = h0 ? h0 + hoff : nullptr;   // nullptr: zero state
  bool init_identity = false;
  float* fin = hT ? hT + hoff : nullptr;          // nullptr: final state not kept
  bool outputs = true, homog = false;
  if (sa.pass != 0) {
    const int Ps = seg_count(t_end - t_beg, sa.G);
    const int z = blockIdx.z;
    const long long seg_tok = (long long)sa.G * C;
    auto slot_off = [&](int p) -> long long {
      const int slot = seg_slot_base(cu_seqlens, s, T, sa.G) + p;
      return slot < sa.slots ? ((long long)slot * H + h) * D * D : -1;
    };
    if (sa.pass == 1) {
      const bool xtype = z >= sa.P;
      const int p = xtype ? z - sa.P : z;
      if (Ps <= 1) {
        if (z != 0) return;                       // whole sequence in this one CTA
      } else if (!xtype) {
        if (p > Ps - 2) return;
        const long long o = slot_off(p);
        if (o < 0) return;
        if (p > 0) { init = nullptr; outputs = false; }
        fin = sa.sbuf + o;
        t_beg += p * seg_tok;
        t_end = min(t_end, t_beg + seg_tok);
      } else {
        if (p < 1 || p > Ps - 2) return;
        const long long o = slot_off(p);
        if (o < 0) return;
        init = nullptr; init_identity = true; outputs = false; homog = true;
        fin = sa.xbuf + o;
        t_beg += p * seg_tok;
        t_end = min(t_end, t_beg + seg_tok);
      }
    } else {
      const int p = z + 1;
      if (Ps <= 1 || p > Ps - 1) return;
      const long long o = slot_off(p - 1);
      if (o < 0) return;
      init = sa.sbuf + o;
      if (p != Ps - 1) fin = nullptr;
      t_beg += p * seg_tok;
      t_end = min(t_end, t_beg + seg_tok);
    }
  }

  if (warp == 0) {
    tmem_alloc(&tmem_base_sh, kTmemCols);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
#pragma unroll
  for (int i = 0; i < 2; ++i)
    reinterpret_cast<float4*>(s_corr)[tid + i * NT] = make_float4(0.f, 0.f, 0.f, 0.f);
  // first chunk's inputs
  float beta_next = 0.f;
  if (t_beg < t_end) {
    const int L0 = (int)min((long long)C, t_end - t_beg);
    prefetch_qkg(sm, q, k, g, row0 + t_beg, L0, H, h, tid);
    prefetch_v(sm, v, row0 + t_beg, L0, H, h, tid);
    cp_async_commit();
    if (tid < C && tid < L0) beta_next = beta[(row0 + t_beg + tid) * H + h];
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tb = tmem_base_sh;
  uint32_t phase = 0;

  // ---- initial state: upper thread j holds row j of S^T (= column j of S)
  if (upper) {
    const int j = tid - 128;
#pragma unroll 1
    for (int c0 = 0; c0 < D; c0 += 32) {
      uint32_t f[16], f2[16], pk[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        float x0 = init ? init[(c0 + e) * D + j] : 0.f;
        float x1 = init ? init[(c0 + 16 + e) * D + j] : 0.f;
        if (init_identity) { x0 = (c0 + e == j) ? 1.f : 0.f; x1 = (c0 + 16 + e == j) ? 1.f : 0.f; }
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
    const bool good = mbar_wait(&bar, phase, kWaitLimit);
    phase ^= 1u;
    tc_fence_after();
    return __syncthreads_or(!good) == 0;
  };

  bool alive = true;
#pragma unroll 1
  for (long long t0 = t_beg; t0 < t_end; t0 += C) {
    const int L = (int)min((long long)C, t_end - t0);
    const bool has_next = t0 + C < t_end;
    const int Ln = has_next ? (int)min((long long)C, t_end - t0 - C) : 0;

    // ================= P0: this chunk's inputs have landed ====================
    cp_async_wait_all();
    if (tid < C) s_beta[tid] = beta_next;
    fence_async_smem();
    __syncthreads();

    // ================= P1: decay scan and operand build (all threads) ========
    bool unsafe_any = false;
    {
      const int c = tid & 127, hf = tid >> 7;
      const float* Gc = reinterpret_cast<const float*>(sm + OFF_SG) + c;   // column c
      float gv[32];
#pragma unroll
      for (int r = 0; r < 32; ++r) gv[r] = Gc[(32 * hf + r) * D];
#pragma unroll
      for (int r = 1; r < 32; ++r) gv[r] += gv[r - 1];
      s_pref[3 * hf][c] = gv[0];
      s_pref[3 * hf + 1][c] = gv[16];
      s_pref[3 * hf + 2][c] = gv[31];
      __syncthreads();
      // P_a and G_63 from per-half sums: s0 = G_0, s1 = G_16, s2 = G_31 (first half),
      // s3, s4, s5 = G_32, G_48, G_63 minus G_31 (second half)
      const float s0 = s_pref[0][c], s1 = s_pref[1][c], s2 = s_pref[2][c];
      const float s3 = s_pref[3][c], s4 = s_pref[4][c], s5 = s_pref[5][c];
      if (hf == 1) s_gamma[c] = __expf(s2 + s5);
      BlockRefs br;
      {
        // dP[a][a2] = P_{a2} - P_a (a2 > a), tg[a] = G_63 - P_a, Pabs[a] = P_a
        const float Pabs[4] = {s0, s1, s2 + s3, s2 + s4};
        const float ref[4] = {s0, s1, s3, s4};            // P_a in the half's frame
        const float tg[4] = {(s2 - s0) + s5, (s2 - s1) + s5, s5 - s3, s5 - s4};
        const float dP[4][4] = {{0.f, s1 - s0, (s2 - s0) + s3, (s2 - s0) + s4},
                                {0.f, 0.f, (s2 - s1) + s3, (s2 - s1) + s4},
                                {0.f, 0.f, 0.f, s4 - s3},
                                {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
        for (int lb = 0; lb < 2; ++lb) {
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            if (hh != hf) continue;
            const int a = 2 * hh + lb;
            br.ref[lb] = ref[a];
            br.eP[lb] = __expf(Pabs[a]);
            br.tl[lb] = tg[a];
            br.eE[lb] = __expf(tg[a]);
#pragma unroll
            for (int a2 = 0; a2 < 4; ++a2) {
              br.dd[lb][a2] = dP[a][a2];
              br.f[lb][a2] = a2 > a ? __expf(dP[a][a2]) : 1.f;
            }
            br.uns[lb] = gv[16 * lb] - gv[16 * lb + 15] > kUnsafeDecay;
          }
        }
      }
      const bf16* kc = reinterpret_cast<const bf16*>(sm + OFF_SK) + c;
      const bf16* qc = reinterpret_cast<const bf16*>(sm + OFF_SQ) + c;
      if (hf == 0) build_half<0>(sm, gv, kc, qc, c, br, tb + lane_base + TM_KB);
      else build_half<1>(sm, gv, kc, qc, c, br, tb + lane_base + TM_KB);
      // exact within-block pairs of the unsafe channels, from the staged rows
#pragma unroll
      for (int lb = 0; lb < 2; ++lb) {
        if (__any_sync(0xffffffffu, br.uns[lb])) {
          const int a = 2 * hf + lb;
          float al[16][1], kv[16][1], qv[16][1];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int r = 16 * a + e;
            const bool u = br.uns[lb];
            al[e][0] = u ? __expf(Gc[r * D]) : 1.f;
            kv[e][0] = u ? __bfloat162float(kc[r * D]) : 0.f;
            qv[e][0] = u ? __bfloat162float(qc[r * D]) : 0.f;
          }
          add_pair_terms<1, 16>(al, kv, qv, s_corr + 256 * a, s_corr + 1024 + 256 * a, lane);
        }
      }
      unsafe_any = br.uns[0] || br.uns[1];
      tmem_wait_st();
      fence_async_smem();
    }
    tc_fence_before();
    const bool fix = __syncthreads_or(unsafe_any) != 0;

    // staging is free: fetch the next chunk's q, k, g (and beta) behind the MMAs
    if (has_next) {
      prefetch_qkg(sm, q, k, g, row0 + t0 + C, Ln, H, h, tid);
      cp_async_commit();
      if (tid < C) beta_next = tid < Ln ? beta[(row0 + t0 + C + tid) * H + h] : 0.f;
    }

    // ================= P2: Gram MMAs ==========================================
    if (tid == 0) {
      // the four R^(a) buffers are consecutive 16-token blocks of one MN-major B
      // operand of N = 160, so the four Gram products are one MMA per K step
      tc_fence_after();
      const uint32_t l_base = smem_u32(sm + OFF_L);
      const uint32_t r_base = smem_u32(sm + off_r(0));
      const uint32_t idesc = idesc_bf16(128, 160, true, true);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk)
        mma_ss(tb + TM_G, desc_mnmajor_sw128(l_base, D, kk), desc_mnmajor_sw32(r_base, D, kk),
               idesc, kk > 0);
      mma_commit(&bar);
    }
    __syncwarp();
    // while the Gram runs: S^T <- S^T Diag(exp(G_63)) (upper threads, own TMEM rows;
    // the MMAs read only the bf16 copy of the state until the update in P8)
    if (upper) {
#pragma unroll 1
      for (int c0 = 0; c0 < D; c0 += 64) {
        uint32_t t[4][16];
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) tmem_ld16(tb + lane_base + TM_S + c0 + 16 * q4, t[q4]);
        tmem_wait_ld();
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
#pragma unroll
          for (int e = 0; e < 16; ++e)
            t[q4][e] = __float_as_uint(__uint_as_float(t[q4][e]) * s_gamma[c0 + 16 * q4 + e]);
          tmem_st16(tb + lane_base + TM_S + c0 + 16 * q4, t[q4]);
        }
      }
      tmem_wait_st();
      tc_fence_before();
    }
    if (!mma_wait()) { alive = false; break; }

    // ================= P3: read A / Aqk ======================================
    float* B32 = reinterpret_cast<float*>(sm + OFF_B32);
    float* T32 = reinterpret_cast<float*>(sm + OFF_T32);
    float* M32 = reinterpret_cast<float*>(sm + OFF_M32);
    {
      // warp w (mod 4) reads TMEM lanes 32w..32w+31: w%4 = 0,1 -> A rows, 2,3 -> Aqk rows.
      // Rows of a warp lie in blocks a0, a0+1; the lower warpgroup handles block a0
      // and the upper warpgroup block a0+1.
      const int w4 = warp & 3;
      const int r = (w4 & 1) * 32 + lane;
      const bool isA = w4 < 2;
      const int a0 = (w4 & 1) * 2;
      const int ab = a0 + (upper ? 1 : 0);            // block handled by this thread
      const int colb = ab == 0 ? 0 : ab == 1 ? 16 : ab == 2 ? 48 : 96;
      const int nb = 16 * (ab + 1);
      const bool mine = (r >> 4) == ab;
      uint32_t tv[4][16];
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        if (16 * q4 < nb) tmem_ld16(tb + lane_base + TM_G + colb + 16 * q4, tv[q4]);
        else {
#pragma unroll
          for (int e = 0; e < 16; ++e) tv[q4][e] = 0u;
        }
      }
      tmem_wait_ld();
      if (fix && mine) {             // the exact within-block pairs of unsafe channels
        float* cr = s_corr + (isA ? 0 : 1024) + 256 * ab + 16 * (r - 16 * ab);
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4)
          if (q4 == ab) {
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              tv[q4][e] = __float_as_uint(__uint_as_float(tv[q4][e]) + cr[e]);
              cr[e] = 0.f;             // cleared for the next chunk
            }
          }
      }
      float vals[64];
#pragma unroll
      for (int i = 0; i < 64; ++i) vals[i] = __uint_as_float(tv[i >> 4][i & 15]);
      if (mine) {
        if (isA) {
          const float br = s_beta[r];
#pragma unroll
          for (int i4 = 0; i4 < 16; ++i4) {
            float4 w;
            w.x = (4 * i4 + 0 < r) ? br * vals[4 * i4 + 0] : 0.f;
            w.y = (4 * i4 + 1 < r) ? br * vals[4 * i4 + 1] : 0.f;
            w.z = (4 * i4 + 2 < r) ? br * vals[4 * i4 + 2] : 0.f;
            w.w = (4 * i4 + 3 < r) ? br * vals[4 * i4 + 3] : 0.f;
            *reinterpret_cast<float4*>(B32 + r * LDA + 4 * i4) = w;
          }
        } else {
          // Aqk: B operand of O^T += Delta^T Aqk^T, K-major SW128, N = 64 (r), K = 64 (i)
#pragma unroll
          for (int c8 = 0; c8 < 8; ++c8) {
            float w[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) w[e] = (c8 * 8 + e <= r) ? vals[c8 * 8 + e] : 0.f;
            st_v4h(sm, OFF_AQK + chunk_kmajor_sw128(r, c8, C), w, 1.f);
          }
        }
      }
    }
    tc_fence_before();
    __syncthreads();

    // ================= triangular inverse T = (I + B)^-1, B = diag(beta) A ====
    if (tid < 64) {                         // diagonal blocks: forward substitution
      const int a = tid >> 4, jj = tid & 15, o = 16 * a;
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
      const int a = p == 0 ? 1 : (p < 3 ? 2 : 3);
      const int m = p - a * (a - 1) / 2;
      const float* Ti = T32 + (16 * a + i) * LDA + 16 * a;
      const float* Bc = B32 + 16 * a * LDA + 16 * m + 4 * jq;
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
      const int q = tid >> 6, i = (tid >> 2) & 15, jq = tid & 3;
      const int col = 16 * q + 4 * jq;
      float4 x = mt(2, 1, i, col);                             // M_21 T_1q
      if (q == 0) {
        const float4 y = mt(1, 0, i, col);                     // M_20 T_00
        x.x += y.x; x.y += y.y; x.z += y.z; x.w += y.w;
      }
      put(32 + i, col, x);
    }
    __syncthreads();
    if (tid < 192) {                                           // T_30, T_31, T_32
      const int q = tid >> 6, i = (tid >> 2) & 15, jq = tid & 3;
      const int col = 16 * q + 4 * jq;
      float4 x = mt(5, 2, i, col);                             // M_32 T_2q
      if (q <= 1) {
        const float4 y = mt(4, 1, i, col);                     // M_31 T_1q
        x.x += y.x; x.y += y.y; x.z += y.z; x.w += y.w;
      }
      if (q == 0) {
        const float4 y = mt(3, 0, i, col);                     // M_30 T_00
        x.x += y.x; x.y += y.y; x.z += y.z; x.w += y.w;
      }
      put(48 + i, col, x);
    }
    __syncthreads();
    // T diag(beta) as bf16: B operand of W^T / U^T, K-major SW128, N = 64 (r'), K = 64 (r)
#pragma unroll
    for (int it = 0; it < 2; ++it) {
      const int idx = tid + it * NT;
      const int rp = idx >> 3, c8 = idx & 7;
      float w[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const int r = c8 * 8 + e;
        w[e] = (r <= rp) ? T32[rp * LDA + r] * s_beta[r] : 0.f;
      }
      st_v4f(sm, OFF_TB + chunk_kmajor_sw128(rp, c8, C), w, 1.f);
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();

    // ================= P4: W^T, U^T =============================================
    if (tid == 0) {
      tc_fence_after();
      const uint32_t tb_base = smem_u32(sm + OFF_TB);
      const uint32_t v_base = smem_u32(sm + OFF_V);
      const uint32_t id_w = idesc_bf16(128, 64, false, false);
      const uint32_t id_u = idesc_bf16(128, 64, true, false);
#pragma unroll
      for (int kk = 0; kk < C / 16; ++kk) {
        const uint64_t bt = desc_kmajor_sw128(tb_base, C, kk);
        mma_ts(tb + TM_W, tb + TM_KB + kk * 8, bt, id_w, kk > 0);
        mma_ss(tb + TM_U, desc_mnmajor_sw128(v_base, C, kk), bt, id_u, kk > 0);
      }
      mma_commit(&bar);
    }
    __syncwarp();
    if (!mma_wait()) { alive = false; break; }
    // V has been consumed: fetch the next chunk's v
    if (has_next) {
      prefetch_v(sm, v, row0 + t0 + C, Ln, H, h, tid);
      cp_async_commit();
    }

    // ================= P5: W^T -> bf16 smem ====================================
    if (!upper) {
      const int c = tid;
      uint32_t t[4][16];
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) tmem_ld16(tb + lane_base + TM_W + 16 * q4, t[q4]);
      tmem_wait_ld();
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
#pragma unroll
        for (int h8 = 0; h8 < 2; ++h8) {
          const float* f = reinterpret_cast<const float*>(t[q4]) + 8 * h8;
          st_v4(sm, OFF_WT + chunk_mnmajor_sw128(2 * q4 + h8, c, D), pack_bf16(f[0], f[1]),
                pack_bf16(f[2], f[3]), pack_bf16(f[4], f[5]), pack_bf16(f[6], f[7]));
        }
      }
      fence_async_smem();
    }
    tc_fence_before();
    __syncthreads();

    // ================= P6: [O^T | P] = S^T [Qbar^T | W^T]^T =====================
    if (tid == 0) {
      tc_fence_after();
      if (outputs) {
        const uint32_t qb_base = smem_u32(sm + OFF_QB);        // W^T follows 16 KB later
        const uint32_t id_op = idesc_bf16(128, 128, false, true);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ts(tb + TM_O, tb + TM_SB + kk * 8, desc_mnmajor_sw128(qb_base, D, kk), id_op, kk > 0);
      } else {
        const uint32_t wt_base = smem_u32(sm + OFF_WT);
        const uint32_t id_p = idesc_bf16(128, 64, false, true);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ts(tb + TM_P, tb + TM_SB + kk * 8, desc_mnmajor_sw128(wt_base, D, kk), id_p, kk > 0);
      }
      mma_commit(&bar);
    }
    __syncwarp();
    if (!mma_wait()) { alive = false; break; }

    // ================= P7: Delta^T = U^T - P -> f16 TMEM (upper threads) ======
    if (upper) {
      uint32_t dw[32];
#pragma unroll
      for (int r0 = 0; r0 < C; r0 += 32) {
        uint32_t tu[2][16], tp[2][16];
#pragma unroll
        for (int q2 = 0; q2 < 2; ++q2) {
          tmem_ld16(tb + lane_base + TM_U + r0 + 16 * q2, tu[q2]);
          tmem_ld16(tb + lane_base + TM_P + r0 + 16 * q2, tp[q2]);
        }
        tmem_wait_ld();
#pragma unroll
        for (int q2 = 0; q2 < 2; ++q2) {
          if (homog) {
#pragma unroll
            for (int e = 0; e < 16; ++e) tu[q2][e] = 0u;
          }
#pragma unroll
          for (int e = 0; e < 8; ++e)
            dw[(r0 + 16 * q2) / 2 + e] =
                pack_f16(__uint_as_float(tu[q2][2 * e]) - __uint_as_float(tp[q2][2 * e]),
                         __uint_as_float(tu[q2][2 * e + 1]) - __uint_as_float(tp[q2][2 * e + 1]));
        }
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

    // ================= P8: [S^T | O^T] += Delta^T [Kend^T ; Aqk]^T =============
    if (tid == 0) {
      tc_fence_after();
      // Kend^T (128 rows) and Aqk (64 rows) form one K-major B operand of 192 rows
      const uint32_t ke_base = smem_u32(sm + OFF_KE);
      const int n = outputs ? D + C : D;
      const uint32_t id_s = idesc_f16(128, n, false, false);    // f16 A (Delta^T) and B
#pragma unroll
      for (int kk = 0; kk < C / 16; ++kk)
        mma_ts(tb + TM_S, tb + TM_KB + kk * 8, desc_kmajor_sw128(ke_base, n, kk), id_s, 1);
      mma_commit(&bar);
    }
    __syncwarp();
    if (!mma_wait()) { alive = false; break; }

    // ================= P9: outputs; bf16 copy of the new state =================
    if (upper) {
      const int j = tid - 128;
      bf16* otile = reinterpret_cast<bf16*>(sm + OFF_OUT);      // [64 tokens][128] row-major
      if (outputs) {
        uint32_t t[4][16];
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) tmem_ld16(tb + lane_base + TM_O + 16 * q4, t[q4]);
        tmem_wait_ld();
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4)
#pragma unroll
          for (int e = 0; e < 16; ++e)
            otile[(16 * q4 + e) * D + j] = __float2bfloat16_rn(__uint_as_float(t[q4][e]));
      }
#pragma unroll 1
      for (int c0 = 0; c0 < D; c0 += 64) {
        uint32_t t[4][16], pk[2][16];
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) tmem_ld16(tb + lane_base + TM_S + c0 + 16 * q4, t[q4]);
        tmem_wait_ld();
#pragma unroll
        for (int q2 = 0; q2 < 2; ++q2) {
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            pk[q2][e] = pack_bf16(__uint_as_float(t[2 * q2][2 * e]), __uint_as_float(t[2 * q2][2 * e + 1]));
            pk[q2][8 + e] =
                pack_bf16(__uint_as_float(t[2 * q2 + 1][2 * e]), __uint_as_float(t[2 * q2 + 1][2 * e + 1]));
          }
          tmem_st16(tb + lane_base + TM_SB + c0 / 2 + 16 * q2, pk[q2]);
        }
      }
      tmem_wait_st();
      named_bar(1, 128);
      // coalesced 16-byte stores of the output tile (16 threads per 256-byte row)
#pragma unroll
      for (int it = 0; it < 8; ++it) {
        const int idx = j + it * 128;
        const int r = idx >> 4, ch = idx & 15;
        if (outputs && r < L) {
          const uint4 val = *reinterpret_cast<const uint4*>(sm + OFF_OUT + r * 256 + ch * 16);
          *reinterpret_cast<uint4*>(out + ((row0 + t0 + r) * H + h) * D + ch * 8) = val;
        }
      }
    }
    tc_fence_before();
    __syncthreads();
  }

  // ---- final state
  if (alive && upper && fin) {
    const int j = tid - 128;
#pragma unroll 1
    for (int c0 = 0; c0 < D; c0 += 16) {
      uint32_t t[16];
      tmem_ld16(tb + lane_base + TM_S + c0, t);
      tmem_wait_ld();
#pragma unroll
      for (int e = 0; e < 16; ++e) fin[(c0 + e) * D + j] = __uint_as_float(t[e]);
    }
  }
  cp_async_wait_all();
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

namespace {

// Dynamic shared memory of the kernel, set once per device.
bool set_attrs() {
  return once_per_device(kOnceTc, []() {
    return cudaFuncSetAttribute(kda_chunk_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                SMEM_BYTES) == cudaSuccess;
  });
}

// Chunks per segment (0: no split).  Cost model in units of one chunk step:
// pass A runs NH*(2P-3) CTAs, pass C NH*(P-1), each G chunks long, in waves of
// one CTA per SM; the combine costs about half a chunk per segment.
int plan_segments(int B, int T, int H, bool varlen, int sms) {
  const long long NH = (long long)B * H;
  const long long nch = ((long long)T + C - 1) / C;
  if (NH * 5 >= (long long)sms * 4 || nch < 8) return 0;
  if (varlen) return nch >= 2 * 16 ? 16 : 0;    // at least two segment slots
  double best = (double)nch;
  int bestG = 0;
  for (int P = 2; P <= 64 && P <= nch; ++P) {
    const long long G = (nch + P - 1) / P;
    const long long Pe = (nch + G - 1) / G;
    if (Pe < 2) continue;
    const long long wA = (NH * (2 * Pe - 3) + sms - 1) / sms;
    const long long wC = (NH * (Pe - 1) + sms - 1) / sms;
    const double cost = (double)G * (double)(wA + wC) + 0.5 * (double)Pe + 2.0;
    if (cost < best) { best = cost; bestG = (int)G; }
  }
  return bestG;
}

}  // namespace

// The single-kernel prefill on caller-provided scratch: no pool, no allocation
// of any kind.  Returns a kda_status_t: KDA_ERR_INVALID_ARG when the
// split this call would use needs more than `capacity` bytes of scratch.
int run_chunk_tc_static(const void* q, const void* k, const void* v, const float* g,
                        const float* beta, const float* h0, const int32_t* cu_seqlens, void* out,
                        float* hT, int B, int T, int H, cudaStream_t stream, float* scratch,
                        size_t capacity) {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      !set_attrs()) {
    (void)cudaGetLastError();
    return KDA_ERR_CUDA;
  }
  const bf16* qb = static_cast<const bf16*>(q);
  const bf16* kb = static_cast<const bf16*>(k);
  const bf16* vb = static_cast<const bf16*>(v);
  bf16* ob = static_cast<bf16*>(out);
  SegArgs sa{0, 1, 0, 0, nullptr, nullptr};
  const int G = plan_segments(B, T, H, cu_seqlens != nullptr, sms);
  const long long nch = ((long long)T + C - 1) / C;
  if (G > 0 && (nch + G - 1) / G >= 2) {
    const int P = (int)((nch + G - 1) / G);
    const long long slots = cu_seqlens ? (long long)P + B : (long long)B * P;
    const size_t bytes = (size_t)2 * slots * H * D * D * sizeof(float);
    if (bytes > capacity || scratch == nullptr) return KDA_ERR_INVALID_ARG;
    sa = SegArgs{G, P, 1, (int)slots, scratch, scratch + (size_t)slots * H * D * D};
  }
  if (sa.pass == 0) {
    KDA_TIMED(KDA_KERNEL_FUSED, stream,
              kda_chunk_tc_kernel<<<dim3(H, B, 1), NT, SMEM_BYTES, stream>>>(qb, kb, vb, g, beta, h0,
                                                                            cu_seqlens, ob, hT, T, H, sa));
    note_launches(1);
  } else {
    KDA_TIMED(KDA_KERNEL_FUSED, stream,
              kda_chunk_tc_kernel<<<dim3(H, B, 2 * sa.P), NT, SMEM_BYTES, stream>>>(
                  qb, kb, vb, g, beta, h0, cu_seqlens, ob, hT, T, H, sa));
    if (launch_seg_combine(cu_seqlens, B, T, H, sa, stream) != cudaSuccess) return KDA_ERR_CUDA;
    sa.pass = 2;
    KDA_TIMED(KDA_KERNEL_FUSED, stream,
              kda_chunk_tc_kernel<<<dim3(H, B, sa.P - 1), NT, SMEM_BYTES, stream>>>(
                  qb, kb, vb, g, beta, h0, cu_seqlens, ob, hT, T, H, sa));
    note_launches(2);
  }
  if (cudaGetLastError() != cudaSuccess) return KDA_ERR_CUDA;
  return KDA_OK;
}

// Reads (and with reset clears) g_chunk_tc_timeout; host side of kda_device_status.
cudaError_t take_tc_timeout(int* flag, bool reset) {
  int v = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, g_chunk_tc_timeout, sizeof(int));
  if (e == cudaSuccess && reset && v != 0) {
    const int zero = 0;
    e = cudaMemcpyToSymbol(g_chunk_tc_timeout, &zero, sizeof(int));
  }
  *flag = v;
  return e;
}

}  // namespace kda
