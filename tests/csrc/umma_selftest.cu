// Self-test of the tcgen05 operand layouts and descriptors in sm100.cuh.
//
// One CTA of 128 threads computes D[128 x N] = A[128 x K] * B[N x K]^T with one
// chain of tcgen05.mma (kind::f16, bf16 in, fp32 accumulate), placing A and B in
// the layout selected at run time, and writes D back to global memory.  The
// test compares D with a plain matmul of the same bf16 values.
//
//   a_layout: 0 = K-major SW128 smem, 1 = MN-major SW128 smem, 2 = TMEM
//   b_layout: 0 = K-major SW128 smem, 1 = MN-major SW128 smem, 2 = MN-major SW32 smem
//
// Shapes accepted: N in {16, 32, ..., 128}, K in {16, 32, ..., 128}; MN-major
// SW128 needs its MN extent to be a multiple of 64 (M = 128 always is; N must
// be 64 or 128 for b_layout 1).  Every smem access stays inside the 64 KB of
// operand space; every wait is bounded and reports failure through *status.
#include <cuda_bf16.h>
#include <stdint.h>

#include "sm100.cuh"

using namespace kda::sm100;

namespace {
constexpr int M = 128;
constexpr uint32_t kTmemCols = 256;   // D: columns [0, 128); A (TMEM): columns [128, 192)
}

extern "C" __global__ void __launch_bounds__(128, 1)
umma_selftest_kernel(const __nv_bfloat16* __restrict__ A, const __nv_bfloat16* __restrict__ B,
                     float* __restrict__ D, int N, int K, int a_layout, int b_layout,
                     int* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = base;            // 32 KB
  uint8_t* sB = base + 32768;    // 32 KB
  __shared__ uint64_t bar;
  __shared__ uint32_t tmem_base;
  const int tid = threadIdx.x, warp = tid >> 5;

  if (warp == 0) {
    tmem_alloc(&tmem_base, kTmemCols);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tb = tmem_base;

  // ---- A
  if (a_layout == 2) {
    // thread m owns TMEM lane m; bf16 pairs packed low = even k
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    for (int c0 = 0; c0 < K / 2; c0 += 16) {
      uint32_t r[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int k = 2 * (c0 + j);
        r[j] = pack_bf16(__bfloat162float(A[tid * K + k]), __bfloat162float(A[tid * K + k + 1]));
      }
      tmem_st16(tb + lane_base + 128 + c0, r);
    }
    tmem_wait_st();
  } else {
    for (int idx = tid; idx < M * K; idx += 128) {
      const int m = idx / K, k = idx % K;
      const uint32_t off = a_layout == 0 ? off_kmajor_sw128(m, k, M) : off_mnmajor_sw128(m, k, K);
      *reinterpret_cast<__nv_bfloat16*>(sA + off) = A[idx];
    }
  }
  // ---- B (logical N x K)
  for (int idx = tid; idx < N * K; idx += 128) {
    const int n = idx / K, k = idx % K;
    uint32_t off;
    if (b_layout == 0) off = off_kmajor_sw128(n, k, N);
    else if (b_layout == 1) off = off_mnmajor_sw128(n, k, K);
    else off = off_mnmajor_sw32(n, k, K);
    *reinterpret_cast<__nv_bfloat16*>(sB + off) = B[idx];
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();

  if (tid == 0) {
    tc_fence_after();
    const uint32_t idesc = idesc_bf16(M, N, a_layout == 1, b_layout != 0);
    const uint32_t a_base = smem_u32(sA), b_base = smem_u32(sB);
    for (int kk = 0; kk < K / 16; ++kk) {
      uint64_t bd;
      if (b_layout == 0) bd = desc_kmajor_sw128(b_base, N, kk);
      else if (b_layout == 1) bd = desc_mnmajor_sw128(b_base, K, kk);
      else bd = desc_mnmajor_sw32(b_base, K, kk);
      if (a_layout == 2) {
        mma_ts(tb, tb + 128 + kk * 8, bd, idesc, kk > 0);
      } else {
        const uint64_t ad = a_layout == 0 ? desc_kmajor_sw128(a_base, M, kk)
                                          : desc_mnmajor_sw128(a_base, K, kk);
        mma_ss(tb, ad, bd, idesc, kk > 0);
      }
    }
    mma_commit(&bar);
  }
  __syncwarp();
  const bool ok = mbar_wait(&bar, 0, 1u << 20);
  if (!ok && tid == 0) atomicExch(status, 1);
  tc_fence_after();
  if (ok) {
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    for (int n0 = 0; n0 < N; n0 += 16) {
      uint32_t r[16];
      tmem_ld16(tb + lane_base + n0, r);
      tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < 16; ++j) D[tid * N + n0 + j] = __uint_as_float(r[j]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tb, kTmemCols);
  }
}

extern "C" int umma_selftest(const void* A, const void* B, float* D, int N, int K, int a_layout,
                             int b_layout, int* status, void* stream) {
  if (N < 16 || N > 128 || N % 16 || K < 16 || K > 128 || K % 16) return -1;
  if (b_layout == 1 && N % 64) return -1;
  const int smem = 131072 + 1024;   // slack: operands use the first 64 KB
  cudaFuncSetAttribute(umma_selftest_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  umma_selftest_kernel<<<1, 128, smem, (cudaStream_t)stream>>>(
      (const __nv_bfloat16*)A, (const __nv_bfloat16*)B, D, N, K, a_layout, b_layout, status);
  return (int)cudaGetLastError();
}
