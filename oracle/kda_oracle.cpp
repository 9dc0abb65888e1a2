// KDA oracle: plain, slow, float64 token-by-token recurrence on the CPU, and its
// reverse-mode backward.
//
// TEST INFRASTRUCTURE ONLY.  Only the tests, the package's smoke check and the
// benchmark's CPU-baseline / reference legs may load this library.  The CUDA
// path never calls it, and it shares no code with the CUDA path.
//
// What it computes (the plain definition, no blocking, no chunking):
//   Kimi Delta Attention per (sequence, head), for t = 0 .. len-1
//     S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T
//     o_t = S_t^T q_t,                alpha_t = exp(g_t)  (one value per key channel)
//   * miniKimiK3 model card, Architecture, "Kimi Delta Attention" bullet: the state
//     update is one gradient-descent step on ||S^T k - v||^2 (an error-correcting
//     write) with per-channel gated decay, a fixed dk x dv state per head and a
//     recurrence for decoding.  The exact update and output above are that
//     bullet's method written as a formula.
//   * Mini-K3-1H-mamba2 model card, packed-document paragraph: state flow is
//     reset at every document boundary; here each cu_seqlens slice starts from
//     its own initial state slot (zero when no initial state is given).
//
// The product (I - beta k k^T) A with A = Diag(alpha) S_{t-1} is formed as
// A - beta k (k^T A): the same matrix, written without materialising the dk x dk
// factor.  A test compares this against the fully materialised product.
//
// Layouts (all row-major, last index fastest):
//   q, k [B, T, H, dk]   v [B, T, H, dv]   g [B, T, H, dk]   beta [B, T, H]
//   out  [B, T, H, dv]   h0, hT [Nseq, H, dk, dv]  (state S is dk x dv, dv fastest)
//   With cu_seqlens (int32, Nseq+1 entries, host memory) the tensors are packed
//   [1, T, H, *] and Nseq = B documents.
//
// Build: g++ -O2 -fopenmp -ffp-contract=off -shared -fPIC (no fast-math).
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>
#ifdef _OPENMP
#include <omp.h>
#endif

namespace {

// One KDA step on state S (dk x dv) for one token of one head; writes o (dv).
void kda_step(double* S, const double* q, const double* k, const double* v,
              const double* g, double beta, double* o, int dk, int dv,
              std::vector<double>& kA) {
  // A = Diag(exp(g)) S_{t-1}: row c of S (key channel c) scaled by alpha_c.
  for (int c = 0; c < dk; ++c) {
    const double a = std::exp(g[c]);
    double* row = S + (size_t)c * dv;
    for (int j = 0; j < dv; ++j) row[j] *= a;
  }
  // k^T A  (a row vector over dv)
  for (int j = 0; j < dv; ++j) kA[j] = 0.0;
  for (int c = 0; c < dk; ++c) {
    const double kc = k[c];
    const double* row = S + (size_t)c * dv;
    for (int j = 0; j < dv; ++j) kA[j] += kc * row[j];
  }
  // S_t = A - beta k (k^T A) + beta k v^T
  for (int c = 0; c < dk; ++c) {
    const double bk = beta * k[c];
    double* row = S + (size_t)c * dv;
    for (int j = 0; j < dv; ++j) row[j] += bk * (v[j] - kA[j]);
  }
  // o_t = S_t^T q_t
  for (int j = 0; j < dv; ++j) o[j] = 0.0;
  for (int c = 0; c < dk; ++c) {
    const double qc = q[c];
    const double* row = S + (size_t)c * dv;
    for (int j = 0; j < dv; ++j) o[j] += qc * row[j];
  }
}

}  // namespace

extern "C" {

// Prefill by recurrence.  h0 may be NULL (zero initial state); hT may be NULL.
// head_lo/head_hi restrict the computation to heads [head_lo, head_hi) (outputs
// of other heads are left untouched) so that large workloads can be sampled.
// Returns 0, or -1 on bad arguments.
int kda_oracle_prefill(const double* q, const double* k, const double* v,
                       const double* g, const double* beta, const double* h0,
                       const int32_t* cu_seqlens, double* out, double* hT,
                       int B, int T, int H, int dk, int dv,
                       int head_lo, int head_hi, int nthreads) {
  if (B <= 0 || T < 0 || H <= 0 || dk <= 0 || dv <= 0) return -1;
  if (head_lo < 0 || head_hi > H || head_lo >= head_hi) return -1;
  const int nseq = B;
  if (cu_seqlens) {
    if (cu_seqlens[0] != 0 || cu_seqlens[nseq] != T) return -1;
    for (int s = 0; s < nseq; ++s)
      if (cu_seqlens[s + 1] < cu_seqlens[s]) return -1;
  }
  const int nh = head_hi - head_lo;
  const long long pairs = (long long)nseq * nh;
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
  for (long long p = 0; p < pairs; ++p) {
    const int s = (int)(p / nh);
    const int h = head_lo + (int)(p % nh);
    // token range and row base of this sequence in the [B?, T, H, *] tensors
    long long t0, t1, row0;
    if (cu_seqlens) { t0 = cu_seqlens[s]; t1 = cu_seqlens[s + 1]; row0 = 0; }
    else { t0 = 0; t1 = T; row0 = (long long)s * T; }
    std::vector<double> S((size_t)dk * dv, 0.0), kA(dv);
    const size_t sidx = ((size_t)s * H + h) * (size_t)dk * dv;
    if (h0) std::memcpy(S.data(), h0 + sidx, sizeof(double) * dk * dv);
    for (long long t = t0; t < t1; ++t) {
      const size_t tok = (size_t)(row0 + t) * H + h;  // (b, t, h) flat index
      kda_step(S.data(), q + tok * dk, k + tok * dk, v + tok * dv, g + tok * dk,
               beta[tok], out + tok * dv, dk, dv, kA);
    }
    if (hT) std::memcpy(hT + sidx, S.data(), sizeof(double) * dk * dv);
  }
  return 0;
}

// One decode step for N independent sequences x H heads, S updated in place.
//   q, k [N, H, dk]  v [N, H, dv]  g [N, H, dk]  beta [N, H]
//   S [N, H, dk, dv]  out [N, H, dv]
// pair_lo/pair_hi restrict the work to flat (n, h) pairs [pair_lo, pair_hi).
int kda_oracle_decode(const double* q, const double* k, const double* v,
                      const double* g, const double* beta, double* S, double* out,
                      int N, int H, int dk, int dv, long long pair_lo,
                      long long pair_hi, int nthreads) {
  if (N <= 0 || H <= 0 || dk <= 0 || dv <= 0) return -1;
  const long long total = (long long)N * H;
  if (pair_lo < 0 || pair_hi > total || pair_lo > pair_hi) return -1;
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel
#endif
  {
    std::vector<double> kA(dv);
#ifdef _OPENMP
#pragma omp for schedule(static)
#endif
    for (long long p = pair_lo; p < pair_hi; ++p) {
      kda_step(S + (size_t)p * dk * dv, q + (size_t)p * dk, k + (size_t)p * dk,
               v + (size_t)p * dv, g + (size_t)p * dk, beta[p], out + (size_t)p * dv,
               dk, dv, kA);
    }
  }
  return 0;
}

// Backward of the prefill by reverse-mode differentiation of the recurrence
// (the "trains through" half of the "Kimi Delta Attention" bullet).  For the
// loss L = sum(out * dout) + sum(hT * dhT) it returns dL/dq, dL/dk, dL/dv,
// dL/dg, dL/dbeta and dL/dh0.  Step t of the forward, a = Diag(exp(g_t)) S_{t-1},
// e = v_t - a^T k_t, S_t = a + beta_t k_t e^T, o_t = S_t^T q_t, is differentiated
// in reverse order with G = dL/dS_t:
//   G += q_t do_t^T;  dq_t = S_t do_t;  w = G^T k_t;  dbeta_t = w . e;  de = beta_t w
//   dv_t = de;  dk_t = beta_t G e - a de;  da = G - k_t de^T
//   dg_t[c] = sum_j da[c][j] a[c][j];  dL/dS_{t-1} = Diag(exp(g_t)) da
// Every state S_{t0..t1} of a sequence is kept (plain, memory (len+1) dk dv).
// dhT and dh0 may be NULL (no final-state loss / initial-state gradient not
// wanted); h0 NULL means a zero initial state.  Returns 0, or -1 on bad arguments.
int kda_oracle_backward(const double* q, const double* k, const double* v,
                        const double* g, const double* beta, const double* h0,
                        const int32_t* cu_seqlens, const double* dout, const double* dhT,
                        double* dq, double* dk_out, double* dv_out, double* dg,
                        double* dbeta, double* dh0, int B, int T, int H, int dk, int dv,
                        int head_lo, int head_hi, int nthreads) {
  if (B <= 0 || T < 0 || H <= 0 || dk <= 0 || dv <= 0) return -1;
  if (head_lo < 0 || head_hi > H || head_lo >= head_hi) return -1;
  const int nseq = B;
  if (cu_seqlens) {
    if (cu_seqlens[0] != 0 || cu_seqlens[nseq] != T) return -1;
    for (int s = 0; s < nseq; ++s)
      if (cu_seqlens[s + 1] < cu_seqlens[s]) return -1;
  }
  const int nh = head_hi - head_lo;
  const long long pairs = (long long)nseq * nh;
  const size_t SZ = (size_t)dk * dv;
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
  for (long long p = 0; p < pairs; ++p) {
    const int s = (int)(p / nh);
    const int h = head_lo + (int)(p % nh);
    long long t0, t1, row0;
    if (cu_seqlens) { t0 = cu_seqlens[s]; t1 = cu_seqlens[s + 1]; row0 = 0; }
    else { t0 = 0; t1 = T; row0 = (long long)s * T; }
    const long long len = t1 - t0;
    const size_t sidx = ((size_t)s * H + h) * SZ;
    // forward, keeping every state: states[i] = S after i tokens
    std::vector<double> states((size_t)(len + 1) * SZ, 0.0), kA(dv), o(dv);
    if (h0) std::memcpy(states.data(), h0 + sidx, sizeof(double) * SZ);
    for (long long i = 0; i < len; ++i) {
      const size_t tok = (size_t)(row0 + t0 + i) * H + h;
      double* S = states.data() + (size_t)(i + 1) * SZ;
      std::memcpy(S, states.data() + (size_t)i * SZ, sizeof(double) * SZ);
      kda_step(S, q + tok * dk, k + tok * dk, v + tok * dv, g + tok * dk, beta[tok], o.data(),
               dk, dv, kA);
    }
    // reverse sweep
    std::vector<double> G(SZ, 0.0), a(SZ), e(dv), w(dv), de(dv);
    if (dhT) std::memcpy(G.data(), dhT + sidx, sizeof(double) * SZ);
    for (long long i = len - 1; i >= 0; --i) {
      const size_t tok = (size_t)(row0 + t0 + i) * H + h;
      const double* qt = q + tok * dk;
      const double* kt = k + tok * dk;
      const double* vt = v + tok * dv;
      const double* gt = g + tok * dk;
      const double* dot = dout + tok * dv;
      const double bt = beta[tok];
      const double* Sprev = states.data() + (size_t)i * SZ;
      const double* Snew = states.data() + (size_t)(i + 1) * SZ;
      // a = Diag(exp(g)) S_{t-1};  e = v - a^T k
      for (int c = 0; c < dk; ++c) {
        const double al = std::exp(gt[c]);
        for (int j = 0; j < dv; ++j) a[(size_t)c * dv + j] = al * Sprev[(size_t)c * dv + j];
      }
      for (int j = 0; j < dv; ++j) {
        double r = 0.0;
        for (int c = 0; c < dk; ++c) r += a[(size_t)c * dv + j] * kt[c];
        e[j] = vt[j] - r;
      }
      // the output's contribution to dL/dS_t, and dq
      for (int c = 0; c < dk; ++c) {
        double acc = 0.0;
        for (int j = 0; j < dv; ++j) {
          G[(size_t)c * dv + j] += qt[c] * dot[j];
          acc += Snew[(size_t)c * dv + j] * dot[j];
        }
        dq[tok * dk + c] = acc;
      }
      // w = G^T k, dbeta, de, dv
      double db = 0.0;
      for (int j = 0; j < dv; ++j) {
        double acc = 0.0;
        for (int c = 0; c < dk; ++c) acc += G[(size_t)c * dv + j] * kt[c];
        w[j] = acc;
        db += acc * e[j];
        de[j] = bt * acc;
        dv_out[tok * dv + j] = de[j];
      }
      dbeta[tok] = db;
      // dk, then da = G - k de^T in place of G, dg, and G <- Diag(exp(g)) da
      for (int c = 0; c < dk; ++c) {
        double acc1 = 0.0, acc2 = 0.0;
        for (int j = 0; j < dv; ++j) {
          acc1 += G[(size_t)c * dv + j] * e[j];
          acc2 += a[(size_t)c * dv + j] * de[j];
        }
        dk_out[tok * dk + c] = bt * acc1 - acc2;
      }
      for (int c = 0; c < dk; ++c) {
        const double al = std::exp(gt[c]);
        double acc = 0.0;
        for (int j = 0; j < dv; ++j) {
          const double da = G[(size_t)c * dv + j] - kt[c] * de[j];
          acc += da * a[(size_t)c * dv + j];
          G[(size_t)c * dv + j] = al * da;
        }
        dg[tok * dk + c] = acc;
      }
    }
    if (dh0) std::memcpy(dh0 + sidx, G.data(), sizeof(double) * SZ);
  }
  return 0;
}

int kda_oracle_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

}  // extern "C"
