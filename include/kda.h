/*
 * kda.h -- C ABI of the B200 (sm_100a) Kimi Delta Attention library, libkda.so.
 *
 * Kimi Delta Attention (KDA) is a gated delta-rule linear attention with a fixed
 * fp32 dk x dv state S per head.  Per token t (miniKimiK3 model card, Architecture,
 * "Kimi Delta Attention" bullet: one gradient-descent step on ||S^T k - v||^2, an
 * error-correcting write, per-channel gated decay, a chunked parallel form for
 * training/prefill and a recurrence for decoding):
 *
 *     S_t = (I - beta_t k_t k_t^T) Diag(exp(g_t)) S_{t-1} + beta_t k_t v_t^T
 *     o_t = S_t^T q_t
 *
 * g_t (one log-decay per key channel, <= 0 in normal use) decays the rows of S.
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are DEVICE pointers owned by the caller; the library
 *     never frees them.  Every pointer must be 16-byte aligned.
 *   - Layouts are dense row-major, last index fastest:
 *       q, k [.., dk]   v, out [.., dv]   g [.., dk] (fp32)   beta [..] (fp32)
 *       states [.., dk, dv] fp32 (row c = key channel, dv contiguous).
 *   - in_dtype (kda_dtype_t) is the storage type of q, k, v and out.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default stream)
 *     and is asynchronous: a KDA_OK return means the work was launched, not done.
 *   - Supported head sizes: dk, dv in {64, 128}.  Others: KDA_ERR_UNSUPPORTED.
 *   - Arguments are validated on the host before anything is launched; on an
 *     error nothing is enqueued and no output is touched.  The library does not
 *     normalise q/k, scale q, or clamp g/beta: those are the caller's inputs.
 *   - Thread safety: calls are independent; concurrent calls on different
 *     streams are safe as long as their output buffers do not overlap.
 */
#ifndef KDA_H_
#define KDA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define KDA_API __attribute__((visibility("default")))
#else
#define KDA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  KDA_OK = 0,
  KDA_ERR_INVALID_ARG = -1,   /* null required pointer, bad size, misalignment */
  KDA_ERR_UNSUPPORTED = -2,   /* valid request the library does not implement  */
  KDA_ERR_CUDA = -3,          /* a CUDA runtime call or kernel launch failed    */
  KDA_ERR_TIMEOUT = -4        /* a bounded device-side wait expired (see kda_device_status) */
} kda_status_t;

typedef enum {
  KDA_BF16 = 0,               /* bfloat16 q, k, v, out */
  KDA_F32 = 1                 /* float32  q, k, v, out */
} kda_dtype_t;

/*
 * kda_chunk_fwd -- KDA prefill through the chunked (C = 64) parallel form.
 *
 * Passage: miniKimiK3 model card, "Kimi Delta Attention" bullet ("trains through a
 * chunked parallel form"); packed-document isolation as in the Mini-K3-1H-mamba2
 * card's packed-document paragraph (state flow reset at every document boundary).
 * The result equals the token-by-token recurrence above up to rounding.
 *
 * Fixed-length mode (cu_seqlens == NULL): B sequences of T tokens each.
 *     q, k, g [B, T, H, dk]   v, out [B, T, H, dv]   beta [B, T, H]
 *     h0, hT  [B, H, dk, dv]
 * Packed mode (cu_seqlens != NULL): B documents packed into one row of T tokens.
 *     q, k, g [1, T, H, dk]   v, out [1, T, H, dv]   beta [1, T, H]
 *     h0, hT  [B, H, dk, dv]  (one state slot per document)
 *     cu_seqlens: DEVICE int32 [B + 1], cu_seqlens[0] = 0, non-decreasing,
 *     cu_seqlens[B] = T.  Documents may be empty.  Document d is tokens
 *     [cu_seqlens[d], cu_seqlens[d+1]) and starts from h0[d] (or zero); no state
 *     crosses a boundary and chunks restart at every document start.  A
 *     document run in one piece gives bit-identical results packed or alone;
 *     when few (document, head) pairs leave SMs idle, long documents are split
 *     into segments whose states are chained afterwards, and then packed and
 *     separate results may differ in rounding order only.  The contents of
 *     cu_seqlens are device memory and are NOT checked on the host; malformed
 *     offsets give undefined results for the affected documents, but every
 *     access stays inside [0, T) (offsets are clamped on the device).
 *
 * h0: initial state, or NULL for zeros.   hT: final state out, or NULL to skip.
 * out must not alias any input.  hT may alias h0 (in-place state update).
 * B >= 1, T >= 0, H >= 1.  T == 0 writes hT = h0 (or zeros) and nothing else.
 *
 * Scratch (KDA_BF16): the call takes its working memory from a library-owned,
 * stream-ordered memory pool of the current device, which keeps its memory for
 * later calls; it is released on the stream when the call's kernels end:
 *   - the chunk records, 74,240 B per (head, chunk), with ceil(T/64) * B chunks
 *     (ceil(T/64) + B in packed mode);
 *   - when few (sequence, head) pairs leave SMs idle and sequences are split into
 *     segments: 2 * 64 KB per segment and head, 4 * 64 KB when the split also
 *     keeps half-way states.
 * If the scratch cannot be allocated nothing is launched and the call returns
 * KDA_ERR_CUDA; kda_chunk_fwd_noalloc runs without allocating.
 * The call's kernels follow each other on `stream` with programmatic stream
 * serialization (a kernel may start while its predecessor in the call drains and
 * waits for it on the device); its first kernel starts after the work queued
 * before it, and work queued after the call sees all of its results, as for a
 * plain launch.  The call can be captured into a CUDA graph.
 *
 * Precision: g, beta and the state are fp32.  With KDA_BF16 inputs the chunk
 * contractions run on the tensor cores with fp32 accumulation, on bf16 operands
 * except the state update's second product (Delta, Kend, Aqk), which runs on
 * f16 operands (finer rounding; values beyond +-65504 saturate there); with
 * KDA_F32 inputs every step runs in fp32 on the CUDA cores.
 *
 * Returns KDA_OK, KDA_ERR_INVALID_ARG, KDA_ERR_UNSUPPORTED or KDA_ERR_CUDA.
 */
KDA_API int kda_chunk_fwd(const void* q, const void* k, const void* v,
                  const float* g, const float* beta, const float* h0,
                  const int32_t* cu_seqlens, void* out, float* hT,
                  int B, int T, int H, int dk, int dv,
                  int in_dtype, void* stream);

/*
 * kda_decode_step -- one recurrent KDA step for N independent sequences.
 *
 * Passage: miniKimiK3 model card, "Kimi Delta Attention" bullet ("decodes as a
 * recurrence with a fixed state per head, so cost per token is constant");
 * the Kimi-K3-Tiny-L13 card's serving paragraph (decode concurrency is bound by
 * the KDA state pool).  Applies the update above once per (n, h), in place:
 *     q, k, g [N, H, dk]   v, out [N, H, dv]   beta [N, H]   S [N, H, dk, dv]
 * S is read once and written once.  out must not alias S or any input.
 * N >= 1, H >= 1.
 *
 * Returns KDA_OK, KDA_ERR_INVALID_ARG, KDA_ERR_UNSUPPORTED or KDA_ERR_CUDA.
 */
KDA_API int kda_decode_step(const void* q, const void* k, const void* v,
                    const float* g, const float* beta, float* S, void* out,
                    int N, int H, int dk, int dv, int in_dtype, void* stream);

/*
 * kda_decode_tokens -- L consecutive recurrent steps for N independent
 * sequences in one launch (multi-token decode, e.g. checking L drafted tokens).
 *
 * Passage: as for kda_decode_step (miniKimiK3 model card, "Kimi Delta
 * Attention" bullet; Kimi-K3-Tiny-L13 card, serving paragraph: decode is bound
 * by the KDA state pool).  The pages give no multi-token interface; this one
 * applies, per (n, h), exactly the update of kda_decode_step to tokens
 * 0 .. L-1 in order, with the same arithmetic, so its results are bit-for-bit
 * those of L successive kda_decode_step calls -- but S is read and written
 * once for all L tokens instead of once per token.
 *     q, k, g [N, L, H, dk]   v, out [N, L, H, dv]   beta [N, L, H]
 *     S [N, H, dk, dv] fp32, in place (the state after token L-1)
 * out must not alias S or any input.  N, L, H >= 1.
 *
 * Returns KDA_OK, KDA_ERR_INVALID_ARG, KDA_ERR_UNSUPPORTED or KDA_ERR_CUDA.
 */
KDA_API int kda_decode_tokens(const void* q, const void* k, const void* v,
                              const float* g, const float* beta, float* S, void* out,
                              int N, int L, int H, int dk, int dv, int in_dtype,
                              void* stream);

/*
 * kda_decode_chunk -- L <= 16 new tokens per (sequence, head) as one chunk of the
 * chunked form, on the tensor cores (speculative verification of drafted tokens,
 * multi-token decode).
 *
 * Passage: as for kda_decode_tokens (miniKimiK3 model card, "Kimi Delta Attention"
 * bullet: the recurrence for decoding and the chunked parallel form, which equal
 * each other).  Same arguments, layouts and in-place state update as
 * kda_decode_tokens:
 *     q, k, g [N, L, H, dk]   v, out [N, L, H, dv]   beta [N, L, H]   S [N, H, dk, dv]
 * The state is read from and written back to HBM once; the chunk-local quantities
 * (16 x 16 Gram, its triangular inverse, W, U) are formed in fp32 on the CUDA
 * cores and the three products with the state run on the tensor cores (S in bf16
 * for the first, f16 operands for the state update), so the results equal L single
 * steps up to that rounding -- not bit for bit, unlike kda_decode_tokens.
 * Supported: KDA_BF16, dk = dv = 128, 1 <= L <= 16 (else KDA_ERR_UNSUPPORTED).
 * out must not alias S or any input.  N, L, H >= 1.
 *
 * Returns KDA_OK, KDA_ERR_INVALID_ARG, KDA_ERR_UNSUPPORTED or KDA_ERR_CUDA.
 */
KDA_API int kda_decode_chunk(const void* q, const void* k, const void* v,
                             const float* g, const float* beta, float* S, void* out,
                             int N, int L, int H, int dk, int dv, int in_dtype,
                             void* stream);

/*
 * kda_chunk_fwd_noalloc -- kda_chunk_fwd for callers that cannot allocate.
 *
 * The pages have no counterpart: this is a deployment variant.  Some callers
 * cannot call cudaMalloc or any allocator: code that runs inside a CUDA graph
 * being captured or replayed under a fixed memory budget, embedders that hand
 * the library only pre-sized buffers, or processes whose allocator is owned by
 * another runtime.  kda_chunk_fwd may take segment scratch from a library pool
 * (see its Scratch note); this entry point instead uses a fixed array of
 * KDA_NOALLOC_SCRATCH_BYTES that lives in the library's device image, so it
 * never allocates, frees or calls an allocating routine.
 *
 * Arguments, layouts, results and error codes are those of kda_chunk_fwd, plus:
 *   - KDA_ERR_INVALID_ARG (nothing launched) when the segment split this call
 *     would use needs more than KDA_NOALLOC_SCRATCH_BYTES of scratch:
 *     2 * 64 KB * H * (number of segment slots); a B=1, T=8192, H=12, d=128
 *     bf16 call needs 19.5 MiB.
 *   - Every GPU that loads the library holds the array (KDA_NOALLOC_SCRATCH_BYTES)
 *     until the process exits.
 *   - The first call on a device looks up the array's device address (one
 *     cudaGetSymbolAddress, with that device current) and keeps it for the life
 *     of the process; make that first call before any stream capture.  Do not
 *     call this entry point again on a device after cudaDeviceReset: the kept
 *     address would be stale.
 *   - All calls on a device share the one array: calls that overlap on the GPU
 *     (different streams without ordering) race on it.  Serialize them.
 */
#define KDA_NOALLOC_SCRATCH_BYTES (32u << 20)
KDA_API int kda_chunk_fwd_noalloc(const void* q, const void* k, const void* v,
                                  const float* g, const float* beta, const float* h0,
                                  const int32_t* cu_seqlens, void* out, float* hT,
                                  int B, int T, int H, int dk, int dv,
                                  int in_dtype, void* stream);

/*
 * Grouped decay ("decay-g64" ablation of the Mini-K3-1H v2 family cards: the
 * decay granularity is one of the varied architecture choices).  The pages
 * name the variant but not its definition; the reading taken here: one log-
 * decay value per group of g_group consecutive key channels, shared by the
 * channels of the group -- channel c decays by exp(g[..., c / g_group]).  g is
 * then [B, T, H, dk / g_group] (prefill) or [N, L, H, dk / g_group] (decode);
 * everything else is as in kda_chunk_fwd / kda_decode_tokens, and g_group = 1
 * is exactly those calls.  g_group must be a power of two, 1 <= g_group <= dk
 * (else KDA_ERR_INVALID_ARG).
 */
KDA_API int kda_chunk_fwd_grouped(const void* q, const void* k, const void* v,
                                  const float* g, const float* beta, const float* h0,
                                  const int32_t* cu_seqlens, void* out, float* hT,
                                  int B, int T, int H, int dk, int dv, int g_group,
                                  int in_dtype, void* stream);
KDA_API int kda_decode_tokens_grouped(const void* q, const void* k, const void* v,
                                      const float* g, const float* beta, float* S, void* out,
                                      int N, int L, int H, int dk, int dv, int g_group,
                                      int in_dtype, void* stream);

/*
 * kda_chunk_fwd_fused -- kda_chunk_fwd with its input prep and output gate fused.
 *
 * Passages: Mini-K3-1H v2 family cards (model architecture: KDA with short
 * convolutions, output gates, decay granularity and convolution length among
 * the varied choices); miniKimiK3 model card (no positional encoding: order
 * enters only through KDA's decay and the short convolutions); Mini-K3-1H-mamba2
 * card, packed-document paragraph (convolution history and recurrent state are
 * reset at every document boundary).  The pages name these pieces but do not
 * define them; the reading taken here (the plainest one):
 *   q_t = dk^-1/2 * n(cq * q_raw)_t,   k_t = n(ck * k_raw)_t,   v_t as given,
 *   (c * x)_t[i] = sum_{j<W} c[h][i][j] x_{t-W+1+j}[i]   (causal, per channel,
 *                  x before the document's first token = 0, no activation),
 *   n(x) = x / max(||x||_2, 1e-12)                       (per token and head),
 *   out_t = o_t * sigmoid(z_t)                           (elementwise, z = gate),
 * with o_t the KDA output of kda_chunk_fwd on (q, k, v, g, beta, h0).
 *     q_raw, k_raw [B, T, H, dk]   v, gate, out [B, T, H, dv]   (in_dtype)
 *     conv_q, conv_k [H, dk, conv_w] fp32 (tap conv_w - 1 multiplies the current
 *     token); conv_w in 1 .. 4.  conv_q = conv_k = NULL: q_raw, k_raw are used as
 *     q, k unchanged (no convolution, normalisation or scaling).  gate NULL: no
 *     gate.  Everything else as in kda_chunk_fwd.
 * The convolution and the normalisation run inside the per-chunk prep kernel
 * (each chunk reads conv_w - 1 rows before it), the gate in the output store:
 * the normalised q, k and the ungated output never reach memory.  Precision:
 * the convolution output is rounded to bf16 before normalisation.
 * Supported: in_dtype KDA_BF16 (KDA_F32: KDA_ERR_UNSUPPORTED).
 *
 * Returns KDA_OK, KDA_ERR_INVALID_ARG (also for only one of conv_q, conv_k, or
 * conv_w out of range), KDA_ERR_UNSUPPORTED or KDA_ERR_CUDA.
 */
KDA_API int kda_chunk_fwd_fused(const void* q_raw, const void* k_raw, const void* v,
                                const float* conv_q, const float* conv_k, int conv_w,
                                const float* g, const float* beta, const void* gate,
                                const float* h0, const int32_t* cu_seqlens, void* out,
                                float* hT, int B, int T, int H, int dk, int dv,
                                int in_dtype, void* stream);

/*
 * kda_chunk_bwd -- gradients of the KDA prefill (training backward).
 *
 * Passage: miniKimiK3 model card, "Kimi Delta Attention" bullet: KDA "trains
 * through a chunked parallel form"; the chunked form equals the recurrence at
 * the top of this file, so its gradients are those of the recurrence.  For the
 * scalar L = sum(out * dout) + sum(hT * dhT) of a kda_chunk_fwd call with the
 * same inputs, this writes
 *     dq, dk [B, T, H, dk]   dv [B, T, H, dv]   dg [B, T, H, dk]   dbeta [B, T, H]
 *     dh0 [B, H, dk, dv]
 * as fp32 (dL/dq, ..., dL/dh0), whatever in_dtype is.  Inputs, layouts,
 * packed mode (cu_seqlens) and in_dtype are those of kda_chunk_fwd; dout has
 * out's shape and dtype; dhT has hT's shape (fp32).  h0 NULL means zeros and
 * then dh0 may be NULL; dhT NULL means zeros.  No gradient flows across a
 * document boundary.  Every token gradient buffer is fully written (empty
 * documents write nothing; their dh0 = dhT).  Output buffers must not alias
 * each other or any input.  The chunk length (64) does not change the result.
 *
 * Method.  KDA_BF16 with dk = dv = 128: the chunked form on the tensor cores
 * (chunks of 64 tokens; the chain rule through the chunked form's equations).
 * Its matrix products take bf16 operands with fp32 accumulation, as the forward's
 * do, so the gradients carry the bf16 bound of the forward (relative error
 * max|x - x_ref| / max|x_ref| of a few 1e-3, at most 1e-2).  The state and its
 * gradient are carried across chunks in fp32.  dq, dk, dv and dh0 are
 * reproducible bit for bit; dg and dbeta add a few per-chunk sums with
 * shared-memory atomics, so repeated calls may differ in their last bits.  Scratch:
 * 213,504 B per (chunk slot, head) (ceil(T/64) * B slots, ceil(T/64) + B when
 * packed).
 * Otherwise (KDA_F32, or a 64-wide head): the recurrent reverse sweep of
 * kda_chunk_bwd_recurrent below.
 * Scratch comes from the library's stream-ordered memory pool (released on the
 * stream at the end of the call).
 *
 * Returns KDA_OK, KDA_ERR_INVALID_ARG, KDA_ERR_UNSUPPORTED or KDA_ERR_CUDA
 * (also when the scratch cannot be allocated).
 */
KDA_API int kda_chunk_bwd(const void* q, const void* k, const void* v,
                          const float* g, const float* beta, const float* h0,
                          const int32_t* cu_seqlens, const void* dout, const float* dhT,
                          float* dq, float* dk, float* dv, float* dg, float* dbeta,
                          float* dh0, int B, int T, int H, int dk_dim, int dv_dim,
                          int in_dtype, void* stream);

/*
 * kda_chunk_bwd_recurrent -- the same gradients (g_group as in
 * kda_chunk_bwd_grouped; 1 = one decay per channel) by a recurrent reverse sweep
 * in fp32 on the CUDA cores, for any in_dtype and head size: accurate to fp32
 * rounding (relative error about 1e-6) where the chunked form is bf16-bounded.
 * The columns of the state evolve independently, so each warp runs the chain of
 * 4 state columns for one (sequence, head); the state is kept at every 64th token
 * and each chunk's states are recomputed once.  dv and dh0 are reproducible bit for
 * bit; dq, dk, dg and dbeta add the warps' parts with atomics, so repeated calls may
 * differ in the last bits (fp32 summation order).  Scratch: 4 * dk * dv bytes per
 * (chunk, head) plus 64 * 4 * dk * dv bytes per (sequence, head), from the library
 * pool.  Returns as kda_chunk_bwd.
 */
KDA_API int kda_chunk_bwd_recurrent(const void* q, const void* k, const void* v,
                                    const float* g, const float* beta, const float* h0,
                                    const int32_t* cu_seqlens, const void* dout,
                                    const float* dhT, float* dq, float* dk, float* dv, float* dg,
                                    float* dbeta, float* dh0, int B, int T, int H, int dk_dim,
                                    int dv_dim, int g_group, int in_dtype, void* stream);

/*
 * kda_chunk_bwd_grouped -- kda_chunk_bwd for grouped decay (one log-decay per
 * group of g_group consecutive key channels, the reading documented at
 * kda_chunk_fwd_grouped).  g and dg are [B, T, H, dk / g_group]; dg[.., m] is
 * the gradient of the shared value, i.e. the sum over the group's channels.
 * Everything else as in kda_chunk_bwd; g_group = 1 is exactly that call.
 * g_group must be a power of two, 1 <= g_group <= dk (else KDA_ERR_INVALID_ARG).
 */
KDA_API int kda_chunk_bwd_grouped(const void* q, const void* k, const void* v,
                                  const float* g, const float* beta, const float* h0,
                                  const int32_t* cu_seqlens, const void* dout,
                                  const float* dhT, float* dq, float* dk, float* dv, float* dg,
                                  float* dbeta, float* dh0, int B, int T, int H, int dk_dim,
                                  int dv_dim, int g_group, int in_dtype, void* stream);

/*
 * Caller-owned workspace.  kda_chunk_fwd and kda_chunk_bwd take their scratch from
 * a library-owned memory pool (see their Scratch notes).  The entry points below
 * take it from the caller instead and allocate nothing at all, so that the caller
 * owns every buffer: query the size, allocate it with the caller's allocator, and
 * pass it in.
 *
 * kda_workspace_size -- the workspace bytes one call needs.  Host only: no device
 * memory is read or allocated.
 *   op        KDA_OP_CHUNK_FWD (kda_chunk_fwd_ws) or KDA_OP_CHUNK_BWD (kda_chunk_bwd_ws)
 *   B, T, H, dk, dv, in_dtype   as the call will pass them
 *   packed    != 0 when the call passes cu_seqlens
 *   sms       streaming multiprocessors of the device the call will run on (the
 *             prefill splits long sequences into segments by it), or 0 for the
 *             current device (then the device's attribute is queried)
 *   *bytes    the size in bytes; 0 means the call needs no workspace
 * The forward's workspace is the chunk records, 74,240 B per (head, chunk slot)
 * with ceil(T/64) * B slots (ceil(T/64) + B when packed), followed, when the call
 * splits sequences into segments, by 2 * 64 KB per (segment slot, head), or
 * 4 * 64 KB when the split keeps half-way states (kda_prefill_plan gives the split;
 * segment slots = B * ceil(ceil(T/64) / G), or that count + B when packed).  KDA_F32
 * forward calls need none.  The backward's is, in its chunked form (KDA_BF16,
 * dk = dv = 128), 213,504 B per (chunk slot, head); otherwise 4 * dk * dv B per
 * (chunk slot + sequence, head) plus 64 * 4 * dk * dv B per (sequence, head).
 * Returns KDA_OK, KDA_ERR_INVALID_ARG (unknown op, bad sizes, NULL bytes),
 * KDA_ERR_UNSUPPORTED (head sizes) or KDA_ERR_CUDA (sms = 0 and no device).
 */
typedef enum {
  KDA_OP_CHUNK_FWD = 0,
  KDA_OP_CHUNK_BWD = 1
} kda_op_t;
KDA_API int kda_workspace_size(int op, int B, int T, int H, int dk, int dv, int packed,
                               int in_dtype, int sms, size_t* bytes);

/*
 * kda_chunk_fwd_ws -- kda_chunk_fwd (g_group = 1) or kda_chunk_fwd_grouped (g_group
 * channels per decay value, as documented there) on caller workspace.
 * kda_chunk_bwd_ws -- kda_chunk_bwd / kda_chunk_bwd_grouped likewise.
 * Passages, arguments, layouts and results: those of the calls named, plus
 *   workspace        DEVICE memory of at least kda_workspace_size(op, ..., sms = 0)
 *                    bytes, 256-byte aligned (NULL when that size is 0), owned by
 *                    the caller.  Its contents on entry do not matter and are
 *                    undefined afterwards; it must not be used by anything else
 *                    until the call's work on `stream` has finished (calls that share
 *                    one workspace must be ordered on the device).
 *   workspace_bytes  its size.
 * These calls allocate nothing and take nothing from the library pool.  A
 * workspace that is too small or misaligned gives KDA_ERR_INVALID_ARG with
 * nothing launched.  Otherwise as the calls named.
 */
KDA_API int kda_chunk_fwd_ws(const void* q, const void* k, const void* v,
                             const float* g, const float* beta, const float* h0,
                             const int32_t* cu_seqlens, void* out, float* hT,
                             int B, int T, int H, int dk, int dv, int g_group, int in_dtype,
                             void* workspace, size_t workspace_bytes, void* stream);
KDA_API int kda_chunk_bwd_ws(const void* q, const void* k, const void* v,
                             const float* g, const float* beta, const float* h0,
                             const int32_t* cu_seqlens, const void* dout, const float* dhT,
                             float* dq, float* dk, float* dv, float* dg, float* dbeta,
                             float* dh0, int B, int T, int H, int dk_dim, int dv_dim,
                             int g_group, int in_dtype, void* workspace,
                             size_t workspace_bytes, void* stream);

/*
 * kda_pool_usage -- the most bytes the library's memory pool on the current device
 * has had in use at once, since the pool was created or since the last reset
 * (diagnostic).  reset != 0 restarts the count after reading it.  Creates the pool
 * if it does not exist yet (which allocates no memory).  Returns KDA_OK,
 * KDA_ERR_INVALID_ARG (NULL output) or KDA_ERR_CUDA.
 */
KDA_API int kda_pool_usage(int reset, unsigned long long* used_high_bytes);

/*
 * kda_device_status -- did a bounded device-side wait give up?
 *
 * Every wait of the library's kernels on an asynchronous copy or a tensor-core
 * operation polls a bounded number of times.  If a limit runs out (a completion
 * that never arrives), the kernel stops waiting -- its results are then invalid --
 * raises a device flag and finishes, so the GPU never hangs on the library.  This
 * call synchronizes the current device (cudaDeviceSynchronize), reads the flags and,
 * with reset != 0, clears them.  Returns KDA_OK (no wait gave up since the library
 * was loaded or since the last reset), KDA_ERR_TIMEOUT (at least one did) or
 * KDA_ERR_CUDA (the device could not be synchronized or read).
 */
KDA_API int kda_device_status(int reset);

/*
 * kda_selftest_bounded_wait -- exercise the path above: launch one thread that
 * waits, at most `polls` polls (1 .. 2^20), on an mbarrier phase that nothing
 * completes, and raises the flag kda_device_status reports.  Asynchronous on
 * `stream`; the device stays usable.  Returns KDA_OK, KDA_ERR_INVALID_ARG or
 * KDA_ERR_CUDA.
 */
KDA_API int kda_selftest_bounded_wait(unsigned polls, void* stream);

/* Human-readable name of a status code (static storage, never NULL). */
KDA_API const char* kda_status_string(int status);

/* Library ABI version: (major << 16) | minor. */
KDA_API int kda_version(void);

/* Number of CUDA kernels this library has launched in the calling process
 * since it was loaded (all threads, all devices).  Diagnostic only. */
KDA_API unsigned long long kda_launch_count(void);

/*
 * kda_prefill_plan -- the sequence split kda_chunk_fwd (KDA_BF16, dk, dv in
 * {64, 128}) chooses for B sequences of T tokens (packed != 0: T packed tokens in
 * B documents) over H heads on a device with `sms` streaming multiprocessors.
 * Host-only (no device access); diagnostic.  Writes *segment_chunks = G, the
 * chunks (of 64 tokens) per segment, 0 when sequences are not split, and
 * *half_chunks = Gh, the chunks of the first pass-C chain of a split middle
 * segment, 0 without half points.  Returns KDA_OK, or KDA_ERR_INVALID_ARG for
 * B, H or sms < 1, T < 0 or a NULL output pointer.
 */
KDA_API int kda_prefill_plan(int B, int T, int H, int packed, int sms, int* segment_chunks,
                             int* half_chunks);

/* Per-kernel timing (diagnostic; this library's own facility, with no
 * counterpart on the pages).  Between kda_timing_start() and
 * kda_timing_stop(), every kernel the library launches is bracketed by two CUDA
 * events recorded on the stream it is launched on (the events cost a few
 * hundred nanoseconds of stream time each; nothing else changes).
 * kda_timing_read(kind, ...) waits for the recorded events and returns the
 * number of launches of that kernel kind and their summed duration in
 * milliseconds since the last kda_timing_start().  At most 65536 launches are
 * recorded; later ones are counted in kda_launch_count() only.  Process-wide,
 * not thread-safe against concurrent start/stop.  Returns KDA_OK,
 * KDA_ERR_INVALID_ARG for an unknown kind or null outputs, KDA_ERR_CUDA if an
 * event could not be created or read. */
typedef enum {
  KDA_KERNEL_PREP = 0,          /* per-chunk prep of the split prefill            */
  KDA_KERNEL_STATE = 1,         /* state pass of the split prefill                */
  KDA_KERNEL_COMBINE = 2,       /* segment combine                                */
  KDA_KERNEL_FUSED = 3,         /* single-kernel tensor-core prefill              */
  KDA_KERNEL_SIMT = 4,          /* CUDA-core prefill (fp32, d = 64)               */
  KDA_KERNEL_DECODE = 5,        /* decode step                                    */
  KDA_KERNEL_BWD = 6,           /* prefill backward, recurrent sweep              */
  KDA_KERNEL_BWD_PREP = 7,      /* chunked backward: per-chunk prep               */
  KDA_KERNEL_BWD_CHAIN = 8,     /* chunked backward: forward and reverse chains   */
  KDA_KERNEL_BWD_GRAD = 9,      /* chunked backward: per-chunk gradients          */
  KDA_KERNEL_KINDS = 10
} kda_kernel_kind_t;
KDA_API int kda_timing_start(void);
KDA_API int kda_timing_stop(void);
KDA_API int kda_timing_read(int kind, unsigned long long* launches, double* total_ms);

#ifdef __cplusplus
}
#endif

#endif /* KDA_H_ */
