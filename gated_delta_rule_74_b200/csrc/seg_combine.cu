// Segment combine of the split prefill scan:
//   S_start,1 = S_end,0;  S_start,p+1 = X_p S_start,p + Sloc_p  (p = 1 .. Ps-2),
// S_start,p+1 overwriting Sloc_p's slot (see segments.cuh for the split).
#include "kda_common.cuh"
#include "segments.cuh"
#include "sm100.cuh"

namespace kda {

// Set when a bounded wait of the segment combine gives up (diagnostic).
__device__ int g_seg_combine_timeout = 0;

namespace {
using namespace sm100;
constexpr int D = kHead;

// One CTA per (sequence, head) runs the
// chain on the tensor cores with fp32-level accuracy: each fp32 operand is split
// into bf16 hi + lo parts and X S = Xh Sh + Xh Sl + Xl Sh (the dropped Xl Sl is
// ~2^-16 relative), accumulated in fp32 in TMEM.  Global traffic is coalesced
// (warp w, lane l handles rows w + 4i, columns 4l..4l+3); thread c reads row c
// of the product from TMEM lane c.
constexpr int kCombineThreads = 128;
constexpr uint32_t CB_AH = 0, CB_AL = 32768, CB_BH = 65536, CB_BL = 98304;
constexpr uint32_t CB_LOC = 131072;                          // fp32 rows [D][LOC_LD]
constexpr int LOC_LD = 132;                                   // padded: float4 rows conflict-free
constexpr size_t kCombineSmem = 131072 + D * LOC_LD * 4 + 1024;

__device__ __forceinline__ void split2(float a, float b, uint32_t& hi, uint32_t& lo) {
  hi = pack_bf16(a, b);
  lo = pack_bf16(a - __uint_as_float(hi << 16), b - __uint_as_float(hi & 0xffff0000u));
}

__global__ void __launch_bounds__(kCombineThreads, 1)
kda_seg_combine_kernel(const int32_t* __restrict__ cu_seqlens, int T, int H, SegArgs sa) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~uintptr_t(1023));
  __shared__ uint64_t bar;
  __shared__ uint32_t tmem_base_sh;
  const int h = blockIdx.x, s = blockIdx.y;
  long long r0, a, b;
  seq_range(cu_seqlens, s, T, r0, a, b);
  const int Ps = seg_count(b - a, sa.G);
  if (Ps <= 2) return;
  const int base = seg_slot_base(cu_seqlens, s, T, sa.G);
  if (base + Ps - 1 > sa.slots) return;                    // offsets beyond the planned scratch
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, c = tid;
  const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
  float* loc = reinterpret_cast<float*>(sm + CB_LOC);
  auto slot = [&](int p) { return ((long long)(base + p) * H + h) * D * D; };

  // coalesced row copy global -> padded smem rows (cp.async)
  auto load_loc = [&](const float* src) {
#pragma unroll 8
    for (int i = 0; i < D / 4; ++i) {
      const int r = warp + 4 * i;
      cp_async16(loc + r * LOC_LD + 4 * lane, src + (long long)r * D + 4 * lane, 16u);
    }
    cp_async_commit();
  };
  // X rows into registers, coalesced: xr[i] = X[warp + 4i][4 lane .. 4 lane + 3]
  float4 xr[D / 4];
  auto load_x = [&](const float* src) {
#pragma unroll
    for (int i = 0; i < D / 4; ++i)
      xr[i] = *reinterpret_cast<const float4*>(src + (long long)(warp + 4 * i) * D + 4 * lane);
  };
  // A (K-major): element (row r, k) -> 8-byte piece of chunk (r, k / 8)
  auto store_a = [&]() {
#pragma unroll
    for (int i = 0; i < D / 4; ++i) {
      const int r = warp + 4 * i, k = 4 * lane;
      uint32_t h0, l0, h1, l1;
      split2(xr[i].x, xr[i].y, h0, l0);
      split2(xr[i].z, xr[i].w, h1, l1);
      const uint32_t o = chunk_kmajor_sw128(r, k >> 3, D) + (k & 7) * 2;
      *reinterpret_cast<uint2*>(sm + CB_AH + o) = make_uint2(h0, h1);
      *reinterpret_cast<uint2*>(sm + CB_AL + o) = make_uint2(l0, l1);
    }
  };
  // B (MN-major) K-row c from loc row c
  auto store_b = [&]() {
    const float* lr = loc + c * LOC_LD;
#pragma unroll
    for (int c8 = 0; c8 < D / 8; ++c8) {
      const float4 u = *reinterpret_cast<const float4*>(lr + c8 * 8);
      const float4 w = *reinterpret_cast<const float4*>(lr + c8 * 8 + 4);
      uint32_t hw[4], lw[4];
      split2(u.x, u.y, hw[0], lw[0]); split2(u.z, u.w, hw[1], lw[1]);
      split2(w.x, w.y, hw[2], lw[2]); split2(w.z, w.w, hw[3], lw[3]);
      const uint32_t o = chunk_mnmajor_sw128(c8, c, D);
      *reinterpret_cast<uint4*>(sm + CB_BH + o) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
      *reinterpret_cast<uint4*>(sm + CB_BL + o) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
    }
  };

  if (warp == 0) {
    tmem_alloc(&tmem_base_sh, 128);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  load_loc(sa.sbuf + slot(0));                             // S_start,1
  load_x(sa.xbuf + slot(1));
  cp_async_wait_all();
  __syncthreads();
  store_b();
  store_a();
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tb = tmem_base_sh;
  uint32_t phase = 0;
  bool ok = true;
  const uint32_t idesc = idesc_bf16(128, 128, false, true);
  for (int p = 1; p <= Ps - 2 && ok; ++p) {
    if (tid == 0) {
      tc_fence_after();
      const uint32_t ah = smem_u32(sm + CB_AH), al = smem_u32(sm + CB_AL);
      const uint32_t bh = smem_u32(sm + CB_BH), bl = smem_u32(sm + CB_BL);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        mma_ss(tb, desc_kmajor_sw128(ah, D, kk), desc_mnmajor_sw128(bh, D, kk), idesc, kk > 0);
        mma_ss(tb, desc_kmajor_sw128(ah, D, kk), desc_mnmajor_sw128(bl, D, kk), idesc, 1);
        mma_ss(tb, desc_kmajor_sw128(al, D, kk), desc_mnmajor_sw128(bh, D, kk), idesc, 1);
      }
      mma_commit(&bar);
    }
    __syncwarp();
    // while the tensor cores work: Sloc_p -> loc (the B operand is already in
    // smem), X_{p+1} -> registers
    float* Sp = sa.sbuf + slot(p);
    load_loc(Sp);
    const bool more = p + 1 <= Ps - 2;
    if (more) load_x(sa.xbuf + slot(p + 1));
    const bool good = mbar_wait(&bar, phase, 1u << 22);
    phase ^= 1u;
    tc_fence_after();
    cp_async_wait_all();
    if (__syncthreads_or(!good)) { ok = false; break; }
    // S_start,p+1 = X_p S_start,p + Sloc_p: row c from TMEM lane c
    {
      float* lr = loc + c * LOC_LD;
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 16) {
        uint32_t t[16];
        tmem_ld16(tb + lane_base + c0, t);
        tmem_wait_ld();
#pragma unroll
        for (int e4 = 0; e4 < 4; ++e4) {
          float4 l4 = *reinterpret_cast<float4*>(lr + c0 + 4 * e4);
          l4.x += __uint_as_float(t[4 * e4]);
          l4.y += __uint_as_float(t[4 * e4 + 1]);
          l4.z += __uint_as_float(t[4 * e4 + 2]);
          l4.w += __uint_as_float(t[4 * e4 + 3]);
          *reinterpret_cast<float4*>(lr + c0 + 4 * e4) = l4;
        }
      }
    }
    tc_fence_before();
    __syncthreads();
    // coalesced store of S_start,p+1 into Sloc_p's slot; next operands
#pragma unroll 8
    for (int i = 0; i < D / 4; ++i) {
      const int r = warp + 4 * i;
      *reinterpret_cast<float4*>(Sp + (long long)r * D + 4 * lane) =
          *reinterpret_cast<const float4*>(loc + r * LOC_LD + 4 * lane);
    }
    if (more) {
      store_b();
      store_a();
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
  }
  if (!ok && tid == 0) {
    atomicExch(&g_seg_combine_timeout, 1);
    mbar_wait(&bar, phase, 1u << 22);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tb, 128);
  }
}

}  // namespace

cudaError_t launch_seg_combine(const int32_t* cu_seqlens, int B, int T, int H, const SegArgs& sa,
                               cudaStream_t stream) {
  if (!once_per_device(kOnceCombine, []() {
        return cudaFuncSetAttribute(kda_seg_combine_kernel,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)kCombineSmem) == cudaSuccess;
      }))
    return cudaErrorInvalidDevice;
  KDA_TIMED(KDA_KERNEL_COMBINE, stream,
            kda_seg_combine_kernel<<<dim3(H, B), kCombineThreads, kCombineSmem, stream>>>(cu_seqlens, T, H,
                                                                                          sa));
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace kda

namespace kda {

// Reads (and with reset clears) g_seg_combine_timeout; host side of kda_device_status.
cudaError_t take_combine_timeout(int* flag, bool reset) {
  int v = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, g_seg_combine_timeout, sizeof(int));
  if (e == cudaSuccess && reset && v != 0) {
    const int zero = 0;
    e = cudaMemcpyToSymbol(g_seg_combine_timeout, &zero, sizeof(int));
  }
  *flag = v;
  return e;
}

}  // namespace kda
