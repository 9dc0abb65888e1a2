// Sequence bookkeeping shared by the tensor-core prefill kernels: token ranges
// of (possibly packed) sequences, chunk numbering, and the segment split used
// when there are too few (sequence, head) pairs to fill the GPU.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace kda {

constexpr int kChunk = 64;     // C: tokens per chunk
constexpr int kHead = 128;     // dk = dv handled by the tensor-core kernels

// Sequence splitting.  Each sequence is cut into segments of G chunks and the
// scan runs in three steps:
//   pass A  segment 0 runs from h0 and writes its outputs; segments p >= 1 run
//           from a zero state (no outputs) and keep their local end state
//           Sloc_p; further chains run segments 1 <= p <= Ps-2 from the
//           identity with the write term dropped (U = 0), which yields the
//           segment's transition X_p (S_end = X_p S_start + Sloc_p);
//   combine S_start,1 = S_end,0 and S_start,p+1 = X_p S_start,p + Sloc_p (fp32):
//           a separate launch in the single-kernel prefill; in the split prefill
//           each pass C chain forms its own S_start,p from pass A's results;
//   pass C  segments p >= 1 run again from S_start,p and write their outputs;
//           the last one writes hT.
// With a half point Gh (split prefill), the pass A chains of segments 1 .. Ps-2
// also keep their state after the first Gh chunks (Sloc_half,p and X_half,p), and
// pass C runs each of those segments as two chains: [0, Gh) from S_start,p and
// [Gh, G) from S_mid,p = X_half,p S_start,p + Sloc_half,p, which that chain forms
// on the tensor cores before its first chunk.  This halves pass C's serial length.
// This is the chunked recurrence's own affine structure over chunks, grouped.
struct SegArgs {
  int G;          // chunks per segment; 0 = one chain walks the whole sequence
  int P;          // segment slots per sequence in the grid (z extent of pass C)
  int pass;       // 0 = single pass, 1 = pass A, 2 = pass C
  int slots;      // number of (segment) slots the scratch holds per head
  float* sbuf;    // [slots][H][D][D] fp32: Sloc_p (the single-kernel prefill's combine
                  // then overwrites it with S_start,p+1)
  float* xbuf;    // [slots][H][D][D] fp32: X_p
  int half;       // Gh: chunks of the first pass C chain of a split segment (0 = no split)
  float* sbuf_h;  // [slots][H][D][D] fp32: Sloc_half,p
  float* xbuf_h;  // [slots][H][D][D] fp32: X_half,p
};

// Token range of sequence s: rows [row0 + t_beg, row0 + t_end) of the token axis.
__device__ __forceinline__ void seq_range(const int32_t* cu, int s, int T, long long& row0,
                                          long long& t_beg, long long& t_end) {
  if (cu) {
    int a = cu[s], b = cu[s + 1];
    a = min(max(a, 0), T);
    b = min(max(b, a), T);
    row0 = 0; t_beg = a; t_end = b;
  } else {
    row0 = (long long)s * T; t_beg = 0; t_end = T;
  }
}
__device__ __forceinline__ long long chunk_count(long long len) {
  return (len + kChunk - 1) / kChunk;
}
__device__ __forceinline__ int seg_count(long long len, int G) {
  return (int)((chunk_count(len) + G - 1) / G);
}
// first scratch slot of sequence s: segments of all earlier sequences
__device__ __forceinline__ int seg_slot_base(const int32_t* cu, int s, int T, int G) {
  if (!cu) return s * seg_count(T, G);
  int base = 0;
  for (int d = 0; d < s; ++d) {
    long long r0, a, b;
    seq_range(cu, d, T, r0, a, b);
    base += seg_count(b - a, G);
  }
  return base;
}
// index of the first chunk of sequence s when all sequences' chunks are numbered
// consecutively (chunks restart at every sequence start)
__device__ __forceinline__ long long seq_chunk_base(const int32_t* cu, int s, int T) {
  if (!cu) return (long long)s * chunk_count(T);
  long long base = 0;
  for (int d = 0; d < s; ++d) {
    long long r0, a, b;
    seq_range(cu, d, T, r0, a, b);
    base += chunk_count(b - a);
  }
  return base;
}

// Upper bound of the number of chunks over all sequences (packed documents add
// at most one partial chunk each).
__host__ __forceinline__ long long chunk_slots(int B, int T, bool varlen) {
  const long long per = ((long long)T + kChunk - 1) / kChunk;
  return varlen ? per + B : per * B;
}

// Per-device runtime state: SM count and a private stream-ordered memory pool
// that keeps its memory between calls.  Returns false without a usable device.
bool device_ctx(int* sms, cudaMemPool_t* pool);

// Segment combine of the single-kernel prefill (one launch):
// S_start,p+1 = X_p S_start,p + Sloc_p in place, with X_p and the states as fp32
// [128][128].  (The split prefill chains the segments inside its pass C instead.)
cudaError_t launch_seg_combine(const int32_t* cu_seqlens, int B, int T, int H, const SegArgs& sa,
                               cudaStream_t stream);

}  // namespace kda
