// C ABI of libkda: host-side argument validation and kernel dispatch.
// The entry points and their contracts are declared and documented in kda.h.
#include <stdint.h>

#include <atomic>
#include <initializer_list>

#include "kda_common.cuh"

namespace kda {
static std::atomic<unsigned long long> g_launches{0};
void note_launches(unsigned long long n) { g_launches.fetch_add(n, std::memory_order_relaxed); }
}  // namespace kda

namespace {

constexpr int kVersionMajor = 0;
constexpr int kVersionMinor = 1;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool head_ok(int d) { return d == 64 || d == 128; }

int status_from(cudaError_t e) {
  if (e == cudaSuccess) return KDA_OK;
  (void)cudaGetLastError();   // clear a sticky launch-config error for the caller
  return KDA_ERR_CUDA;
}

// All required pointers non-null and every given pointer 16-byte aligned.
bool pointers_ok(std::initializer_list<const void*> required,
                 std::initializer_list<const void*> optional) {
  for (const void* p : required)
    if (p == nullptr || !aligned16(p)) return false;
  for (const void* p : optional)
    if (p != nullptr && !aligned16(p)) return false;
  return true;
}


// log2 of a decay group size: 0..log2(dk) for a power of two dividing dk, else -1
int group_shift(int g_group, int dk) {
  if (g_group < 1 || g_group > dk || (g_group & (g_group - 1)) != 0) return -1;
  int sh = 0;
  while ((1 << sh) < g_group) ++sh;
  return sh;
}

bool aligned256(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 255u) == 0; }

// SM count of the current device (no allocation, no pool).
bool current_sms(int* sms) { return kda::device_ctx(sms, nullptr); }

// A caller workspace that is 256-byte aligned and holds `need` bytes (a NULL or
// empty workspace is fine when nothing is needed).
bool workspace_ok(const kda::Workspace* ws, size_t need) {
  if (need == 0) return ws->ptr == nullptr || aligned256(ws->ptr);
  return ws->ptr != nullptr && aligned256(ws->ptr) && ws->bytes >= need;
}

int chunk_fwd_impl(const void* q, const void* k, const void* v, const float* g,
                   const float* beta, const float* h0, const int32_t* cu_seqlens, void* out,
                   float* hT, int B, int T, int H, int dk, int dv, int gsh, int in_dtype,
                   void* stream, const kda::Workspace* ws = nullptr) {
  if (B < 1 || T < 0 || H < 1) return KDA_ERR_INVALID_ARG;
  if (in_dtype != KDA_BF16 && in_dtype != KDA_F32) return KDA_ERR_INVALID_ARG;
  const long long rows = cu_seqlens ? (long long)T : (long long)B * T;
  if (rows > 0) {
    if (!pointers_ok({q, k, v, g, beta, out}, {h0, hT, cu_seqlens})) return KDA_ERR_INVALID_ARG;
  } else {
    // no tokens: the token tensors may be empty (null); only the states are used
    if (!pointers_ok({}, {q, k, v, g, beta, out, h0, hT, cu_seqlens})) return KDA_ERR_INVALID_ARG;
  }
  if (!head_ok(dk) || !head_ok(dv)) return KDA_ERR_UNSUPPORTED;
  if (gsh < 0) return KDA_ERR_INVALID_ARG;
  // element counts must fit the kernels' 64-bit indexing and the grid limits
  if (rows * H * (long long)(dk > dv ? dk : dv) > (1LL << 40)) return KDA_ERR_INVALID_ARG;
  if ((long long)B > 65535LL || H > 65535) return KDA_ERR_UNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (kda::chunk_split_supported(dk, dv, in_dtype)) {
    if (ws) {
      int sms = 0;
      if (!current_sms(&sms)) return KDA_ERR_CUDA;
      if (!workspace_ok(ws, kda::chunk_split_scratch_bytes(B, T, H, cu_seqlens != nullptr, sms)))
        return KDA_ERR_INVALID_ARG;
    }
    return status_from(kda::launch_chunk_split(q, k, v, g, beta, h0, cu_seqlens, out, hT, B, T,
                                               H, dk, dv, gsh, st, nullptr, ws));
  }
  if (ws && !workspace_ok(ws, 0)) return KDA_ERR_INVALID_ARG;
  return status_from(kda::launch_chunk_simt(q, k, v, g, beta, h0, cu_seqlens, out, hT, B, T,
                                            H, dk, dv, in_dtype, gsh, st));
}

int decode_tokens_impl(const void* q, const void* k, const void* v, const float* g,
                       const float* beta, float* S, void* out, int N, int L, int H, int dk,
                       int dv, int gsh, int in_dtype, void* stream) {
  if (N < 1 || L < 1 || H < 1) return KDA_ERR_INVALID_ARG;
  if (in_dtype != KDA_BF16 && in_dtype != KDA_F32) return KDA_ERR_INVALID_ARG;
  if (!pointers_ok({q, k, v, g, beta, S, out}, {})) return KDA_ERR_INVALID_ARG;
  if (!head_ok(dk) || !head_ok(dv)) return KDA_ERR_UNSUPPORTED;
  if (gsh < 0) return KDA_ERR_INVALID_ARG;
  if ((long long)N * H > 0x7fffffffLL) return KDA_ERR_INVALID_ARG;
  if ((long long)N * L * H * (dk > dv ? dk : dv) > (1LL << 40)) return KDA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return status_from(
      kda::launch_decode_tokens(q, k, v, g, beta, S, out, N, L, H, dk, dv, in_dtype, gsh, st));
}

}  // namespace

extern "C" {

int kda_chunk_fwd(const void* q, const void* k, const void* v, const float* g,
                  const float* beta, const float* h0, const int32_t* cu_seqlens, void* out,
                  float* hT, int B, int T, int H, int dk, int dv, int in_dtype,
                  void* stream) {
  return chunk_fwd_impl(q, k, v, g, beta, h0, cu_seqlens, out, hT, B, T, H, dk, dv, 0, in_dtype,
                        stream);
}

int kda_chunk_fwd_grouped(const void* q, const void* k, const void* v, const float* g,
                          const float* beta, const float* h0, const int32_t* cu_seqlens,
                          void* out, float* hT, int B, int T, int H, int dk, int dv, int g_group,
                          int in_dtype, void* stream) {
  return chunk_fwd_impl(q, k, v, g, beta, h0, cu_seqlens, out, hT, B, T, H, dk, dv,
                        group_shift(g_group, dk), in_dtype, stream);
}

int kda_decode_step(const void* q, const void* k, const void* v, const float* g,
                    const float* beta, float* S, void* out, int N, int H, int dk, int dv,
                    int in_dtype, void* stream) {
  if (N < 1 || H < 1) return KDA_ERR_INVALID_ARG;
  if (in_dtype != KDA_BF16 && in_dtype != KDA_F32) return KDA_ERR_INVALID_ARG;
  if (!pointers_ok({q, k, v, g, beta, S, out}, {})) return KDA_ERR_INVALID_ARG;
  if (!head_ok(dk) || !head_ok(dv)) return KDA_ERR_UNSUPPORTED;
  if ((long long)N * H > 0x7fffffffLL) return KDA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return status_from(kda::launch_decode(q, k, v, g, beta, S, out, N, H, dk, dv, in_dtype, st));
}

int kda_decode_tokens(const void* q, const void* k, const void* v, const float* g,
                      const float* beta, float* S, void* out, int N, int L, int H, int dk, int dv,
                      int in_dtype, void* stream) {
  return decode_tokens_impl(q, k, v, g, beta, S, out, N, L, H, dk, dv, 0, in_dtype, stream);
}

int kda_decode_chunk(const void* q, const void* k, const void* v, const float* g,
                     const float* beta, float* S, void* out, int N, int L, int H, int dk, int dv,
                     int in_dtype, void* stream) {
  if (N < 1 || L < 1 || H < 1) return KDA_ERR_INVALID_ARG;
  if (in_dtype != KDA_BF16 && in_dtype != KDA_F32) return KDA_ERR_INVALID_ARG;
  if (!pointers_ok({q, k, v, g, beta, S, out}, {})) return KDA_ERR_INVALID_ARG;
  if (!head_ok(dk) || !head_ok(dv)) return KDA_ERR_UNSUPPORTED;
  if (!kda::decode_chunk_supported(dk, dv, in_dtype, L)) return KDA_ERR_UNSUPPORTED;
  if ((long long)N * H > 0x7fffffffLL) return KDA_ERR_INVALID_ARG;
  if ((long long)N * L * H * (dk > dv ? dk : dv) > (1LL << 40)) return KDA_ERR_INVALID_ARG;
  return status_from(kda::launch_decode_chunk(q, k, v, g, beta, S, out, N, L, H,
                                              static_cast<cudaStream_t>(stream)));
}

int kda_decode_tokens_grouped(const void* q, const void* k, const void* v, const float* g,
                              const float* beta, float* S, void* out, int N, int L, int H, int dk,
                              int dv, int g_group, int in_dtype, void* stream) {
  return decode_tokens_impl(q, k, v, g, beta, S, out, N, L, H, dk, dv, group_shift(g_group, dk),
                            in_dtype, stream);
}

int kda_chunk_fwd_fused(const void* q_raw, const void* k_raw, const void* v, const float* conv_q,
                        const float* conv_k, int conv_w, const float* g, const float* beta,
                        const void* gate, const float* h0, const int32_t* cu_seqlens, void* out,
                        float* hT, int B, int T, int H, int dk, int dv, int in_dtype,
                        void* stream) {
  if (B < 1 || T < 0 || H < 1) return KDA_ERR_INVALID_ARG;
  if (in_dtype != KDA_BF16 && in_dtype != KDA_F32) return KDA_ERR_INVALID_ARG;
  if ((conv_q == nullptr) != (conv_k == nullptr)) return KDA_ERR_INVALID_ARG;
  if (conv_q && (conv_w < 1 || conv_w > 4)) return KDA_ERR_INVALID_ARG;
  const long long rows = cu_seqlens ? (long long)T : (long long)B * T;
  if (rows > 0) {
    if (!pointers_ok({q_raw, k_raw, v, g, beta, out}, {conv_q, conv_k, gate, h0, hT, cu_seqlens}))
      return KDA_ERR_INVALID_ARG;
  } else {
    if (!pointers_ok({}, {q_raw, k_raw, v, g, beta, out, conv_q, conv_k, gate, h0, hT,
                          cu_seqlens}))
      return KDA_ERR_INVALID_ARG;
  }
  if (!head_ok(dk) || !head_ok(dv)) return KDA_ERR_UNSUPPORTED;
  if (!kda::chunk_split_supported(dk, dv, in_dtype)) return KDA_ERR_UNSUPPORTED;
  if (rows * H * (long long)(dk > dv ? dk : dv) > (1LL << 40)) return KDA_ERR_INVALID_ARG;
  if ((long long)B > 65535LL || H > 65535) return KDA_ERR_UNSUPPORTED;
  const kda::InputFusion fz{conv_q, conv_k, conv_q ? conv_w : 0, gate};
  return status_from(kda::launch_chunk_split(q_raw, k_raw, v, g, beta, h0, cu_seqlens, out, hT, B,
                                             T, H, dk, dv, 0, static_cast<cudaStream_t>(stream),
                                             &fz));
}

namespace {
// Scratch of a kda_chunk_bwd call: the chunked form's (bf16, 128-wide heads) or the
// recurrent sweep's.
size_t bwd_scratch(int B, int T, int H, int dk, int dv, bool varlen, int in_dtype) {
  if (kda::chunk_bwd_tc_supported(dk, dv, in_dtype))
    return kda::chunk_bwd_tc_scratch_bytes(B, T, H, varlen);
  return kda::chunk_bwd_scratch_bytes(B, T, H, dk, dv, varlen);
}

int chunk_bwd_impl(const void* q, const void* k, const void* v, const float* g,
                   const float* beta, const float* h0, const int32_t* cu_seqlens,
                   const void* dout, const float* dhT, float* dq, float* dk, float* dv, float* dg,
                   float* dbeta, float* dh0, int B, int T, int H, int dk_dim, int dv_dim, int gsh,
                   int in_dtype, void* stream, const kda::Workspace* ws = nullptr,
                   bool recurrent = false) {
  if (gsh < 0) return KDA_ERR_INVALID_ARG;
  if (B < 1 || T < 0 || H < 1) return KDA_ERR_INVALID_ARG;
  if (in_dtype != KDA_BF16 && in_dtype != KDA_F32) return KDA_ERR_INVALID_ARG;
  const long long rows = cu_seqlens ? (long long)T : (long long)B * T;
  if (rows > 0) {
    if (!pointers_ok({q, k, v, g, beta, dout, dq, dk, dv, dg, dbeta}, {h0, dhT, dh0, cu_seqlens}))
      return KDA_ERR_INVALID_ARG;
  } else {
    if (!pointers_ok({}, {q, k, v, g, beta, dout, dq, dk, dv, dg, dbeta, h0, dhT, dh0,
                          cu_seqlens}))
      return KDA_ERR_INVALID_ARG;
  }
  if (!head_ok(dk_dim) || !head_ok(dv_dim)) return KDA_ERR_UNSUPPORTED;
  if (rows * H * (long long)(dk_dim > dv_dim ? dk_dim : dv_dim) > (1LL << 40))
    return KDA_ERR_INVALID_ARG;
  if ((long long)B > 65535LL || H > 0x7fffffff) return KDA_ERR_UNSUPPORTED;
  const bool chunked = !recurrent && kda::chunk_bwd_tc_supported(dk_dim, dv_dim, in_dtype);
  if (ws && !workspace_ok(ws, bwd_scratch(B, T, H, dk_dim, dv_dim, cu_seqlens != nullptr,
                                          in_dtype)))
    return KDA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (chunked)
    return status_from(kda::launch_chunk_bwd_tc(q, k, v, g, beta, h0, cu_seqlens, dout, dhT, dq,
                                                dk, dv, dg, dbeta, dh0, B, T, H, gsh, st, ws));
  return status_from(kda::launch_chunk_bwd(q, k, v, g, beta, h0, cu_seqlens, dout, dhT, dq, dk,
                                           dv, dg, dbeta, dh0, B, T, H, dk_dim, dv_dim, gsh,
                                           in_dtype, st, ws));
}
}  // namespace

int kda_chunk_bwd(const void* q, const void* k, const void* v, const float* g,
                  const float* beta, const float* h0, const int32_t* cu_seqlens,
                  const void* dout, const float* dhT, float* dq, float* dk, float* dv, float* dg,
                  float* dbeta, float* dh0, int B, int T, int H, int dk_dim, int dv_dim,
                  int in_dtype, void* stream) {
  return chunk_bwd_impl(q, k, v, g, beta, h0, cu_seqlens, dout, dhT, dq, dk, dv, dg, dbeta, dh0,
                        B, T, H, dk_dim, dv_dim, 0, in_dtype, stream);
}

int kda_chunk_bwd_grouped(const void* q, const void* k, const void* v, const float* g,
                          const float* beta, const float* h0, const int32_t* cu_seqlens,
                          const void* dout, const float* dhT, float* dq, float* dk, float* dv,
                          float* dg, float* dbeta, float* dh0, int B, int T, int H, int dk_dim,
                          int dv_dim, int g_group, int in_dtype, void* stream) {
  return chunk_bwd_impl(q, k, v, g, beta, h0, cu_seqlens, dout, dhT, dq, dk, dv, dg, dbeta, dh0,
                        B, T, H, dk_dim, dv_dim, group_shift(g_group, dk_dim), in_dtype, stream);
}

int kda_chunk_bwd_recurrent(const void* q, const void* k, const void* v, const float* g,
                            const float* beta, const float* h0, const int32_t* cu_seqlens,
                            const void* dout, const float* dhT, float* dq, float* dk, float* dv,
                            float* dg, float* dbeta, float* dh0, int B, int T, int H, int dk_dim,
                            int dv_dim, int g_group, int in_dtype, void* stream) {
  return chunk_bwd_impl(q, k, v, g, beta, h0, cu_seqlens, dout, dhT, dq, dk, dv, dg, dbeta, dh0,
                        B, T, H, dk_dim, dv_dim, group_shift(g_group, dk_dim), in_dtype, stream,
                        nullptr, true);
}

int kda_workspace_size(int op, int B, int T, int H, int dk, int dv, int packed, int in_dtype,
                       int sms, size_t* bytes) {
  if (!bytes || B < 1 || T < 0 || H < 1 || sms < 0) return KDA_ERR_INVALID_ARG;
  if (op != KDA_OP_CHUNK_FWD && op != KDA_OP_CHUNK_BWD) return KDA_ERR_INVALID_ARG;
  if (in_dtype != KDA_BF16 && in_dtype != KDA_F32) return KDA_ERR_INVALID_ARG;
  if (!head_ok(dk) || !head_ok(dv)) return KDA_ERR_UNSUPPORTED;
  if (op == KDA_OP_CHUNK_BWD) {
    *bytes = bwd_scratch(B, T, H, dk, dv, packed != 0, in_dtype);
    return KDA_OK;
  }
  if (!kda::chunk_split_supported(dk, dv, in_dtype)) {
    *bytes = 0;                                     // the fp32 path keeps everything on chip
    return KDA_OK;
  }
  if (sms == 0 && !current_sms(&sms)) return KDA_ERR_CUDA;
  *bytes = kda::chunk_split_scratch_bytes(B, T, H, packed != 0, sms);
  return KDA_OK;
}

int kda_chunk_fwd_ws(const void* q, const void* k, const void* v, const float* g,
                     const float* beta, const float* h0, const int32_t* cu_seqlens, void* out,
                     float* hT, int B, int T, int H, int dk, int dv, int g_group, int in_dtype,
                     void* workspace, size_t workspace_bytes, void* stream) {
  const kda::Workspace ws{workspace, workspace_bytes};
  return chunk_fwd_impl(q, k, v, g, beta, h0, cu_seqlens, out, hT, B, T, H, dk, dv,
                        group_shift(g_group, dk), in_dtype, stream, &ws);
}

int kda_chunk_bwd_ws(const void* q, const void* k, const void* v, const float* g,
                     const float* beta, const float* h0, const int32_t* cu_seqlens,
                     const void* dout, const float* dhT, float* dq, float* dk, float* dv,
                     float* dg, float* dbeta, float* dh0, int B, int T, int H, int dk_dim,
                     int dv_dim, int g_group, int in_dtype, void* workspace,
                     size_t workspace_bytes, void* stream) {
  const kda::Workspace ws{workspace, workspace_bytes};
  return chunk_bwd_impl(q, k, v, g, beta, h0, cu_seqlens, dout, dhT, dq, dk, dv, dg, dbeta, dh0,
                        B, T, H, dk_dim, dv_dim, group_shift(g_group, dk_dim), in_dtype, stream,
                        &ws);
}

int kda_pool_usage(int reset, unsigned long long* used_high_bytes) {
  if (!used_high_bytes) return KDA_ERR_INVALID_ARG;
  return kda::pool_used_high(reset != 0, used_high_bytes);
}

int kda_device_status(int reset) {
  if (cudaDeviceSynchronize() != cudaSuccess) return status_from(cudaErrorUnknown);
  int any = 0;
  for (auto take : {kda::take_split_timeout, kda::take_tc_timeout, kda::take_bwd_timeout,
                    kda::take_bwd_tc_timeout, kda::take_combine_timeout,
                    kda::take_selftest_timeout, kda::take_decode_chunk_timeout}) {
    int f = 0;
    if (take(&f, reset != 0) != cudaSuccess) return status_from(cudaErrorUnknown);
    any |= f;
  }
  return any ? KDA_ERR_TIMEOUT : KDA_OK;
}

int kda_selftest_bounded_wait(unsigned polls, void* stream) {
  if (polls < 1 || polls > (1u << 20)) return KDA_ERR_INVALID_ARG;
  return status_from(kda::launch_selftest_wait(polls, static_cast<cudaStream_t>(stream)));
}

const char* kda_status_string(int status) {
  switch (status) {
    case KDA_OK: return "KDA_OK";
    case KDA_ERR_INVALID_ARG: return "KDA_ERR_INVALID_ARG";
    case KDA_ERR_UNSUPPORTED: return "KDA_ERR_UNSUPPORTED";
    case KDA_ERR_CUDA: return "KDA_ERR_CUDA";
    case KDA_ERR_TIMEOUT: return "KDA_ERR_TIMEOUT";
    default: return "KDA_ERR_UNKNOWN";
  }
}

int kda_version(void) { return (kVersionMajor << 16) | kVersionMinor; }

unsigned long long kda_launch_count(void) {
  return kda::g_launches.load(std::memory_order_relaxed);
}

int kda_prefill_plan(int B, int T, int H, int packed, int sms, int* segment_chunks,
                     int* half_chunks) {
  if (B < 1 || T < 0 || H < 1 || sms < 1 || !segment_chunks || !half_chunks)
    return KDA_ERR_INVALID_ARG;
  kda::chunk_split_plan(B, T, H, packed != 0, sms, segment_chunks, half_chunks);
  return KDA_OK;
}

}  // extern "C"
