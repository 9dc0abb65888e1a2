// KDA oracle: plain, slow, float64 token-by-token recurrence on the CPU.
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

int kda_oracle_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

}  // extern "C"
