// Internal helpers shared by the KDA CUDA kernels (not part of the C ABI).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "kda.h"

namespace kda {

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// Runs setup() (kernel attributes and the like) once per call site and device, with
// that device current; thread-safe.  A setup that fails is retried on the next call.
enum OnceSite {
  kOnceSplit = 0, kOnceTc, kOnceDecodeChunk, kOnceCombine, kOnceCombineImg, kOnceBwdTc, kOnceSites
};
bool once_per_device(int site, bool (*setup)());

// Most bytes the library pool of the current device has had in use at once; with
// reset, the count restarts (kda_pool_usage).
int pool_used_high(bool reset, unsigned long long* used_high);
// SM count (and, when pool != nullptr, the library's memory pool) of the current device.
bool device_ctx(int* sms, cudaMemPool_t* pool);

// Count of kernel launches made by the library (see kda_launch_count()).
void note_launches(unsigned long long n);

// Per-kernel timing (kda_timing_*): bracket one launch of kernel kind `kind`
// on `stream`; timing_begin returns a handle (-1 when timing is off).
int timing_begin(int kind, cudaStream_t stream);
void timing_end(int handle, cudaStream_t stream);
#define KDA_TIMED(kind, stream, ...)                  \
  do {                                                \
    const int kda_th_ = timing_begin(kind, stream);   \
    __VA_ARGS__;                                      \
    timing_end(kda_th_, stream);                      \
  } while (0)

// Launch `kern` with programmatic stream serialization: it may start while the
// kernel before it on `stream` is still running, and must call grid_dep_wait()
// before touching anything that kernel writes (see sm100.cuh).
template <typename... KArgs, typename... Args>
cudaError_t launch_after(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                         cudaStream_t stream, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// Launchers implemented in the kernel translation units.  Each returns a
// cudaError_t from the launch (cudaSuccess when the launch was accepted).
cudaError_t launch_decode(const void* q, const void* k, const void* v, const float* g,
                          const float* beta, float* S, void* out, int N, int H, int dk,
                          int dv, int in_dtype, cudaStream_t stream);

// gsh: log2 of the decay group (g holds one value per 2^gsh key channels).
cudaError_t launch_decode_tokens(const void* q, const void* k, const void* v, const float* g,
                                 const float* beta, float* S, void* out, int N, int L, int H,
                                 int dk, int dv, int in_dtype, int gsh, cudaStream_t stream);

cudaError_t launch_chunk_simt(const void* q, const void* k, const void* v, const float* g,
                              const float* beta, const float* h0, const int32_t* cu_seqlens,
                              void* out, float* hT, int B, int T, int H, int dk, int dv,
                              int in_dtype, int gsh, cudaStream_t stream);

// Tensor-core chunked prefill (bf16, dk = dv = 128) in one kernel per sequence
// (kda_chunk_fwd_noalloc; see run_chunk_tc_static below).
bool chunk_tc_supported(int dk, int dv, int in_dtype);

// Fused input prep and output gate (kda_chunk_fwd_fused; split path only):
// q, k <- L2-normalised causal per-channel convolutions of the raw q, k (q also
// scaled by dk^-1/2), out <- out * sigmoid(gate).
struct InputFusion {
  const float* conv_q;   // [H, dk, W] fp32, or nullptr: q, k used as given
  const float* conv_k;   // [H, dk, W] fp32
  int W;                 // convolution width, 1 .. 4
  const void* gate;      // [rows, H, dv] in the input dtype, or nullptr: no gate
};

// Scratch the caller provides for one call (kda_chunk_fwd_ws / kda_chunk_bwd_ws);
// a launcher given one takes nothing from the library pool.
struct Workspace {
  void* ptr;
  size_t bytes;
};

// Tensor-core prefill split into a parallel per-chunk kernel and a state pass
// (bf16, dk, dv in {64, 128}: 64-wide heads run zero-padded to 128); its
// scratch comes from the library's memory pool.
bool chunk_split_supported(int dk, int dv, int in_dtype);
// The split prefill's plan (host only): chunks per segment, chunks of a half point.
void chunk_split_plan(int B, int T, int H, bool varlen, int sms, int* G, int* half);
// Scratch bytes of one split prefill call on a device with `sms` SMs.
size_t chunk_split_scratch_bytes(int B, int T, int H, bool varlen, int sms);
cudaError_t launch_chunk_split(const void* q, const void* k, const void* v, const float* g,
                               const float* beta, const float* h0, const int32_t* cu_seqlens,
                               void* out, float* hT, int B, int T, int H, int dk, int dv,
                               int gsh, cudaStream_t stream, const InputFusion* fz = nullptr,
                               const Workspace* ws = nullptr);

// Prefill backward (recurrent, fp32): gradients of sum(out*dout) + sum(hT*dhT).
// Scratch bytes of one backward call.
size_t chunk_bwd_scratch_bytes(int B, int T, int H, int dk, int dv, bool varlen);
cudaError_t launch_chunk_bwd(const void* q, const void* k, const void* v, const float* g,
                             const float* beta, const float* h0, const int32_t* cu_seqlens,
                             const void* dout, const float* dhT, float* dq, float* dk, float* dv,
                             float* dg, float* dbeta, float* dh0, int B, int T, int H, int dkd,
                             int dvd, int gsh, int in_dtype, cudaStream_t stream,
                             const Workspace* ws = nullptr);

// Chunked backward on the tensor cores (bf16, dk = dv = 128): the prep kernel's
// backward form, the state chains and the per-chunk gradient kernel.  Scratch:
// chunk_bwd_tc_scratch_bytes() (records, states, Delta and their gradients).
bool chunk_bwd_tc_supported(int dk, int dv, int in_dtype);
size_t chunk_bwd_tc_scratch_bytes(int B, int T, int H, bool varlen);
cudaError_t launch_chunk_bwd_tc(const void* q, const void* k, const void* v, const float* g,
                                const float* beta, const float* h0, const int32_t* cu_seqlens,
                                const void* dout, const float* dhT, float* dq, float* dk,
                                float* dv, float* dg, float* dbeta, float* dh0, int B, int T,
                                int H, int gsh, cudaStream_t stream,
                                const Workspace* ws = nullptr);

// Bounded-wait flags (one per kernel file): read, and with reset clear, the flag a
// kernel raises when one of its bounded waits gives up.
cudaError_t take_split_timeout(int* flag, bool reset);
cudaError_t take_tc_timeout(int* flag, bool reset);
cudaError_t take_bwd_timeout(int* flag, bool reset);
cudaError_t take_bwd_tc_timeout(int* flag, bool reset);
cudaError_t take_combine_timeout(int* flag, bool reset);
cudaError_t take_selftest_timeout(int* flag, bool reset);
cudaError_t take_decode_chunk_timeout(int* flag, bool reset);

// Multi-token decode in the chunked form on the tensor cores (bf16, dk = dv = 128,
// 1 <= L <= 16 tokens per (sequence, head)).
bool decode_chunk_supported(int dk, int dv, int in_dtype, int L);
cudaError_t launch_decode_chunk(const void* q, const void* k, const void* v, const float* g,
                                const float* beta, float* S, void* out, int N, int L, int H,
                                cudaStream_t stream);
// One thread waits, at most `polls` polls, on an mbarrier phase nothing completes.
cudaError_t launch_selftest_wait(uint32_t polls, cudaStream_t stream);

// The tensor-core prefill on caller-provided scratch (allocates nothing).
int run_chunk_tc_static(const void* q, const void* k, const void* v, const float* g,
                        const float* beta, const float* h0, const int32_t* cu_seqlens, void* out,
                        float* hT, int B, int T, int H, cudaStream_t stream, float* scratch,
                        size_t capacity);

}  // namespace kda
