// kda_chunk_fwd_noalloc: the prefill for callers that cannot allocate device
// memory (see kda.h).  Its segment scratch is a fixed array in this library's
// device image instead of memory from an allocator.
#include <stdint.h>

#include <initializer_list>

#include "kda_common.cuh"

namespace {

// Scratch shared by every call on a device: per segment and head, a local end
// state and a transition matrix (2 x 64 KB of fp32).  Every slot a call reads
// is written earlier in the same call, so nothing needs clearing between calls.
static __device__ __align__(256) float g_noalloc_scratch[KDA_NOALLOC_SCRATCH_BYTES / sizeof(float)];

// Device address of the array on the current device.  In host code the array's
// name only stands in for it, so the address is looked up on every call (the lookup
// allocates nothing); a cached address would go stale if the context were rebuilt.
float* scratch_address() {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) {
    (void)cudaGetLastError();
    return nullptr;
  }
  return static_cast<float*>(p);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" int kda_chunk_fwd_noalloc(const void* q, const void* k, const void* v,
                                     const float* g, const float* beta, const float* h0,
                                     const int32_t* cu_seqlens, void* out, float* hT, int B,
                                     int T, int H, int dk, int dv, int in_dtype, void* stream) {
  if (B < 1 || T < 0 || H < 1) return KDA_ERR_INVALID_ARG;
  if (in_dtype != KDA_BF16 && in_dtype != KDA_F32) return KDA_ERR_INVALID_ARG;
  const long long rows = cu_seqlens ? (long long)T : (long long)B * T;
  for (const void* p : std::initializer_list<const void*>{h0, hT, cu_seqlens})
    if (p && !aligned16(p)) return KDA_ERR_INVALID_ARG;
  for (const void* p : std::initializer_list<const void*>{q, k, v, g, beta, out}) {
    if (p && !aligned16(p)) return KDA_ERR_INVALID_ARG;
    if (!p && rows > 0) return KDA_ERR_INVALID_ARG;
  }
  if ((dk != 64 && dk != 128) || (dv != 64 && dv != 128)) return KDA_ERR_UNSUPPORTED;
  if (rows * H * (long long)(dk > dv ? dk : dv) > (1LL << 40)) return KDA_ERR_INVALID_ARG;
  if ((long long)B > 65535LL || H > 65535) return KDA_ERR_UNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (!kda::chunk_tc_supported(dk, dv, in_dtype)) {
    // this path keeps everything on chip and needs no scratch
    const cudaError_t e = kda::launch_chunk_simt(q, k, v, g, beta, h0, cu_seqlens, out, hT, B, T,
                                                 H, dk, dv, in_dtype, 0, st);
    if (e != cudaSuccess) { (void)cudaGetLastError(); return KDA_ERR_CUDA; }
    return KDA_OK;
  }
  float* scratch = scratch_address();
  if (!scratch) return KDA_ERR_CUDA;
  return kda::run_chunk_tc_static(q, k, v, g, beta, h0, cu_seqlens, out, hT, B, T, H, st, scratch,
                                  KDA_NOALLOC_SCRATCH_BYTES);
}
