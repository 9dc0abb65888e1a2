// sm_100a primitives: mbarriers, tensor memory (TMEM), tcgen05 MMA descriptors,
// and the shared-memory operand layouts the KDA kernels use.
//
// Layout vocabulary (bf16 operands, all tiles 1024-byte aligned):
//   K-major SW128   rows = M or N index, 64 K-elements (128 B) per row and K-block,
//                   16-byte chunks XOR-swizzled with (row % 8); K-blocks of 64
//                   elements follow each other (stride rows * 128 B).
//   MN-major SW128  rows = K index, 64 MN-elements (128 B) per row and MN-block,
//                   chunk swizzle (row % 8); MN-blocks of 64 follow each other
//                   (stride K * 128 B).
//   MN-major SW32   rows = K index, 16 MN-elements (32 B) per row and MN-block,
//                   chunk swizzle ((row / 4) % 2); MN-blocks of 16 follow each
//                   other (stride K * 32 B).
// Descriptor fields follow the tcgen05 shared-memory matrix descriptor: start
// address, leading-dimension byte offset (LBO), stride-dimension byte offset
// (SBO), descriptor version 1, swizzle mode in bits 61-63.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace kda {
namespace sm100 {

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait: returns false if the phase did not complete within `limit`
// polls (each try_wait itself blocks for a hardware-defined interval).
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint32_t limit) {
  for (uint32_t i = 0; i < limit; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  return false;
}

// Arrive on `bar` (one arrival) and add `bytes` to the transaction count its
// current phase waits for.
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

// ------------------------------------------------------------------ fences
__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
// orders this thread's generic global-memory accesses before later async-proxy
// (bulk copy) accesses to the same addresses
__device__ __forceinline__ void fence_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// 3-D tiled TMA load of one box into shared memory, completing on `bar` (which
// counts the box's bytes).  `tmap` is the address of a CUtensorMap kernel
// parameter (__grid_constant__).  Plain load: no cluster multicast.
__device__ __forceinline__ void tma_load_3d(void* smem_dst, const void* tmap, int c0, int c1,
                                            int c2, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
      : "memory");
}

// ------------------------------------------------- async global -> smem copies
// 16-byte cp.async (L2 only); src_bytes = 0 zero-fills the destination and reads
// nothing (the caller still passes an in-bounds address).
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gsrc, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(smem_dst)),
               "l"(gsrc), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_all;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait_group() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
// Bulk copy (no tensor map, no multicast) of `bytes` contiguous bytes from
// global memory into this CTA's shared memory; completion is signalled on
// `bar` as transaction bytes.  Both addresses 16-byte aligned, bytes % 16 == 0.
__device__ __forceinline__ void bulk_g2s(void* smem_dst, const void* gsrc, uint32_t bytes,
                                         uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(smem_dst)),
      "l"(gsrc), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
// Bulk copy of `bytes` contiguous bytes from this CTA's shared memory to
// global memory (bulk async-group completion).  Both addresses 16-byte aligned,
// bytes % 16 == 0.  The writing threads must have made their shared-memory
// stores visible to the async proxy (fence_async_smem + barrier) first.
__device__ __forceinline__ void bulk_s2g(void* gdst, const void* smem_src, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(gdst),
               "r"(smem_u32(smem_src)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// Wait until at most N committed bulk groups still read their shared-memory source.
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
// Wait until at most N committed bulk groups are incomplete (writes performed).
template <int N>
__device__ __forceinline__ void bulk_wait() {
  asm volatile("cp.async.bulk.wait_group %0;" ::"n"(N) : "memory");
}
// Named barrier over `nthreads` threads (multiple of 32); id 0 is __syncthreads.
__device__ __forceinline__ void named_bar(uint32_t id, uint32_t nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}
// Arrive at named barrier `id` (of `nthreads` participants) without waiting.
__device__ __forceinline__ void named_arrive(uint32_t id, uint32_t nthreads) {
  asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// ------------------------------------------- programmatic dependent launch
// Kernels of one call that follow each other on a stream may be launched with
// programmatic stream serialization: the next grid can start before this one
// ends.  grid_dep_wait() blocks the calling thread until the preceding grid has
// completed and its memory writes are visible (it returns at once when there is no
// such grid); grid_dep_launch() lets the next grid start once every CTA of this
// grid has executed it or exited.
__device__ __forceinline__ void grid_dep_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void grid_dep_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// -------------------------------------------------------------------- TMEM
// Warp-collective.  Writes the allocated TMEM base address to *dst (smem).
__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
// TMEM address: lane in bits 31..16, column in bits 15..0.
__device__ __forceinline__ uint32_t tmem_addr(uint32_t base, uint32_t lane, uint32_t col) {
  return base + (lane << 16) + col;
}

// 32 lanes x 32-bit, N consecutive columns per thread (thread i <-> lane base+i).
#define KDA_TMEM_LD_X16(taddr, r)                                                            \
  asm volatile(                                                                              \
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13," \
      "%14,%15}, [%16];"                                                                     \
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),   \
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),          \
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15])                                                \
      : "r"(taddr))

#define KDA_TMEM_ST_X16(taddr, r)                                                             \
  asm volatile(                                                                               \
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13," \
      "%14,%15,%16};" ::"r"(taddr),                                                            \
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),  \
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),      \
      "r"(r[15]))

__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]));
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  KDA_TMEM_LD_X16(taddr, r);
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  KDA_TMEM_ST_X16(taddr, r);
}
__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// ------------------------------------------------------------ descriptors
enum SwizzleMode : uint32_t { kSwNone = 0, kSw128 = 2, kSw64 = 4, kSw32 = 6 };

__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo,
                                              uint32_t swz) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;                        // descriptor version (sm_100)
  d |= (uint64_t)(swz & 7u) << 61;
  return d;
}

// Instruction descriptor, kind::f16 with bf16 A/B and fp32 accumulation.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool a_mn_major,
                                                  bool b_mn_major) {
  return (1u << 4)                               // D format: f32
         | (1u << 7)                             // A format: bf16
         | (1u << 10)                            // B format: bf16
         | ((a_mn_major ? 1u : 0u) << 15) | ((b_mn_major ? 1u : 0u) << 16) |
         ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// Instruction descriptor, kind::f16 with f16 A and B (both; the format fields are
// 0) and fp32 accumulation.
__host__ __device__ constexpr uint32_t idesc_f16(int M, int N, bool a_mn_major,
                                                 bool b_mn_major) {
  return (1u << 4)                               // D format: f32
         | ((a_mn_major ? 1u : 0u) << 15) | ((b_mn_major ? 1u : 0u) << 16) |
         ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// D[tmem] (+)= A[smem desc] * B[smem desc]^T, one instruction (K = 16).
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}" ::"r"(
          d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(0u), "r"(0u), "r"(0u), "r"(0u)
      : "memory");
}
// D[tmem] (+)= A[tmem] * B[smem desc]^T, one instruction (K = 16).
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, {%5, %6, %7, %8}, p;\n\t}" ::"r"(
          d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(0u), "r"(0u), "r"(0u), "r"(0u)
      : "memory");
}
// Arrive on `bar` when all MMAs issued so far by this thread have completed.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// ------------------------------------------------- operand layout offsets
// Byte offsets inside a tile for one bf16 element; `rows` is the tile's row
// count (K-major: M/N extent; MN-major: K extent).
__host__ __device__ __forceinline__ uint32_t off_kmajor_sw128(uint32_t row, uint32_t k,
                                                              uint32_t rows) {
  return (k >> 6) * rows * 128u + row * 128u + ((((k & 63u) >> 3) ^ (row & 7u)) << 4) +
         ((k & 7u) << 1);
}
__host__ __device__ __forceinline__ uint32_t off_mnmajor_sw128(uint32_t mn, uint32_t k,
                                                               uint32_t krows) {
  return (mn >> 6) * krows * 128u + k * 128u + ((((mn & 63u) >> 3) ^ (k & 7u)) << 4) +
         ((mn & 7u) << 1);
}
__host__ __device__ __forceinline__ uint32_t off_mnmajor_sw32(uint32_t mn, uint32_t k,
                                                              uint32_t krows) {
  return (mn >> 4) * krows * 32u + k * 32u + ((((mn & 15u) >> 3) ^ ((k >> 2) & 1u)) << 4) +
         ((mn & 7u) << 1);
}
// 16-byte chunk (8 consecutive bf16 along the contiguous axis) variants; `c8`
// is the chunk index along the contiguous axis (element index / 8).
__host__ __device__ __forceinline__ uint32_t chunk_kmajor_sw128(uint32_t row, uint32_t c8,
                                                                uint32_t rows) {
  return (c8 >> 3) * rows * 128u + row * 128u + (((c8 & 7u) ^ (row & 7u)) << 4);
}
__host__ __device__ __forceinline__ uint32_t chunk_mnmajor_sw128(uint32_t c8, uint32_t k,
                                                                 uint32_t krows) {
  return (c8 >> 3) * krows * 128u + k * 128u + (((c8 & 7u) ^ (k & 7u)) << 4);
}
__host__ __device__ __forceinline__ uint32_t chunk_mnmajor_sw32(uint32_t c8, uint32_t k,
                                                                uint32_t krows) {
  return (c8 >> 1) * krows * 32u + k * 32u + (((c8 & 1u) ^ ((k >> 2) & 1u)) << 4);
}

// Descriptors of the tile at smem address `base` for MMA step kk (16 K-elements).
__device__ __forceinline__ uint64_t desc_kmajor_sw128(uint32_t base, uint32_t rows, uint32_t kk) {
  return smem_desc(base + (kk >> 2) * rows * 128u + (kk & 3u) * 32u, 16u, 1024u, kSw128);
}
__device__ __forceinline__ uint64_t desc_mnmajor_sw128(uint32_t base, uint32_t krows,
                                                       uint32_t kk) {
  return smem_desc(base + kk * 2048u, krows * 128u, 1024u, kSw128);
}
__device__ __forceinline__ uint64_t desc_mnmajor_sw32(uint32_t base, uint32_t krows, uint32_t kk) {
  return smem_desc(base + kk * 512u, krows * 32u, 256u, kSw32);
}

// Two fp32 values as an f16 pair (round to nearest; values beyond the f16 range
// saturate to the largest finite f16 instead of becoming infinite).
__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.satfinite.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

}  // namespace sm100
}  // namespace kda
