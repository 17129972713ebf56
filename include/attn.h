/*
 * Skip Softmax attention for NVIDIA B200 (sm_100a): C ABI of libattn.so.
 *
 * The operation is fused scaled-dot-product attention, softmax(Q K^T/sqrt(d)) V,
 * evaluated block-wise (key tiles in ascending order, online softmax) with the
 * Skip Softmax block-skip rule: a key tile is skipped -- its exponentials, its
 * P*V product and its V load -- iff for EVERY query row of the row block the
 * tile's local maximum score is strictly below that row's running maximum
 * minus the threshold tau.  Source: "Accelerating Long-Context Inference with
 * Skip Softmax in NVIDIA TensorRT-LLM", Key Points and Detailed Analysis (the
 * page's comparison value is garbled in its transcript and is read as
 * m_i - tau; tau is the user-set speed/accuracy knob of the same sections).
 * Scores are S = Q K^T / sqrt(d) (natural-log units); tau is in those units.
 *
 * Conventions shared by every entry point
 *   - Tensors are bf16, contiguous, head dimension fastest:
 *       Q, O  [B, Hq,  N, d]      K, V  [B, Hkv, N, d]     (prefill)
 *       q, o  [B, Hq,  d]         K, V  [B, Hkv, L, d]     (decode)
 *     Query head h reads KV head floor(h / (Hq/Hkv)) (grouped-query attention).
 *   - Every tensor pointer is a DEVICE pointer on the current CUDA device,
 *     16-byte aligned.  The caller owns all buffers; the library never frees
 *     or keeps a caller pointer past the call's completion on the stream.
 *   - tau >= 0; tau = +INFINITY gives exact attention (nothing is skipped).
 *     NaN or negative tau is rejected.  Inputs must be finite.
 *   - Calls are asynchronous on the stream they are given (the plain forms
 *     use the stream set with attn_set_stream, default the legacy stream).
 *     The returned status covers argument validation and launch errors only;
 *     a kernel that gave up on a bounded internal wait is reported later by
 *     attn_sync_status().
 *   - There is no CPU fallback: without an sm_100 device every compute call
 *     returns ATTN_ERR_UNSUPPORTED.
 *   - The library caches, per device ordinal, the device addresses of its
 *     own __device__ variables (the status word, the no-alloc scratch) in
 *     the device's primary context.  Use it only from the primary context
 *     (the CUDA runtime's default), and not across cudaDeviceReset: after a
 *     reset the cached addresses would be stale.
 */
#ifndef SKIP_SOFTMAX_ATTN_H
#define SKIP_SOFTMAX_ATTN_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define ATTN_API __attribute__((visibility("default")))
#else
#define ATTN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  ATTN_OK = 0,
  ATTN_ERR_INVALID_ARG = 1, /* bad pointer, size, tau, tile or alignment   */
  ATTN_ERR_UNSUPPORTED = 2, /* no sm_100 device, or a shape beyond limits  */
  ATTN_ERR_CUDA = 3,        /* a CUDA runtime/driver call failed           */
  ATTN_ERR_TIMEOUT = 4      /* a kernel gave up on a bounded wait          */
} attn_status;

/* Device status word values written by kernels that gave up (internal). */
#define ATTN_DEVICE_TIMEOUT_BASE 0x100

/*
 * Prefill (self-attention over N tokens), Skip Softmax rule above.
 *   causal   0: every query sees every key.  1: top-left aligned causal mask,
 *            query i sees keys k <= i; key tiles wholly above the diagonal of
 *            a row block are not visited.
 *   Br, Bc   row-block and key-tile sizes of the skip rule:
 *            (64,64), (128,64) or (128,128).  d in {64, 128}.
 *   Errors: ATTN_ERR_INVALID_ARG for null/misaligned pointers, B/Hq/Hkv/N <= 0,
 *   Hq % Hkv != 0, unsupported d/Br/Bc, NaN or negative tau.
 */
ATTN_API int attn_prefill(const void* Q, const void* K, const void* V, void* O, int B, int Hq, int Hkv,
                 int N, int d, int causal, float tau, int Br, int Bc);

/*
 * As attn_prefill, on an explicit stream (a cudaStream_t passed as void*,
 * NULL = legacy stream), optionally writing the skip decisions:
 *   skip_mask  nullable device buffer uint8 [B, Hq, ceil(N/Br), ceil(N/Bc)]:
 *              0 tile kept, 1 tile skipped, 2 tile not visited (causal).
 */
ATTN_API int attn_prefill_ex(const void* Q, const void* K, const void* V, void* O, int B, int Hq, int Hkv,
                    int N, int d, int causal, float tau, int Br, int Bc, void* stream,
                    uint8_t* skip_mask);

/*
 * Prefill over a batch of sequences of different lengths packed one after
 * another ("varlen"), the layout serving engines batch prompts in:
 *   Q, O  [total_tokens, Hq, d] and K, V [total_tokens, Hkv, d], bf16, d
 *         fastest; sequence b is tokens [cu_seqlens[b], cu_seqlens[b+1]).
 *   cu_seqlens  device int32 [B + 1], non-decreasing, cu_seqlens[B] <=
 *         total_tokens; lengths above max_seqlen are cut to max_seqlen.  A
 *         malformed table cannot make the kernel read or write outside the
 *         tensors (offsets and lengths are clamped to [0, total_tokens]).
 *   Each sequence attends only to itself (causal: top-left aligned within
 *   the sequence), with the skip rule of attn_prefill.  Br must be 128
 *   (Bc 64 or 128).  Rows of O outside every sequence are not written.
 *   skip_mask (nullable): [B, Hq, ceil(max_seqlen/128), ceil(max_seqlen/Bc)];
 *   tiles and row blocks past a sequence's end are marked 2.
 *   Errors: as attn_prefill_ex, plus ATTN_ERR_INVALID_ARG for a null or
 *   unaligned cu_seqlens, total_tokens or max_seqlen <= 0, or Br != 128.
 */
ATTN_API int attn_prefill_varlen(const void* Q, const void* K, const void* V, void* O,
                                 const int32_t* cu_seqlens, int B, int max_seqlen,
                                 int total_tokens, int Hq, int Hkv, int d, int causal, float tau,
                                 int Br, int Bc, void* stream, uint8_t* skip_mask);

/*
 * e4m3 quantisation (for attn_prefill_qk8).  x is a device tensor of
 * groups * group_elems bf16 values, cut into `groups` contiguous groups
 * (one head slab [N, d] each for Q [B, Hq, N, d] or K [B, Hkv, N, d]).
 * Group g gets the scale s = 2^k, k the smallest integer >= -126 with
 * max|x| <= 448 * 2^k (448: the largest finite e4m3 value); a group of zeros
 * gets 1, a group holding inf or NaN gets NaN.  q[i] = e4m3(x[i] / s), rounded
 * to nearest, ties to even (OCP FP8 E4M3: bias 7, no infinities).  Since s is
 * a power of two, q * s is exactly representable in bf16.
 *   x: const bf16*, 16-byte aligned.  q: uint8_t* of the same element count,
 *   16-byte aligned.  scales: float* [groups], 4-byte aligned.  All device
 *   memory owned by the caller; the call is asynchronous on `stream`.
 *   Errors: ATTN_ERR_INVALID_ARG for null or unaligned pointers, groups or
 *   group_elems <= 0, or group_elems not a multiple of 16;
 *   ATTN_ERR_UNSUPPORTED off sm_100 or beyond 2^31 blocks; ATTN_ERR_CUDA.
 */
ATTN_API int attn_quantize_e4m3(const void* x, void* q, float* scales, long long groups,
                                long long group_elems, void* stream);

/*
 * Prefill with S = Q K^T from e4m3 operands on the FP8 tensor cores (kind
 * f8f6f4, fp32 accumulation); P*V stays bf16.  Q8 [B, Hq, N, d] and K8
 * [B, Hkv, N, d] hold one byte per element as written by attn_quantize_e4m3
 * with one group per head slab; head (b, h) of Q means Q8 * q_scales[b*Hq+h]
 * and head (b, h) of K means K8 * k_scales[b*Hkv+h].  The result is attention
 * (with the skip rule of attn_prefill) over those dequantised Q and K.
 * V, O and skip_mask as attn_prefill_ex.  d = 128 and Br = 128 only.
 *   Errors: as attn_prefill_ex, plus ATTN_ERR_INVALID_ARG for null or
 *   unaligned scale pointers, d != 128 or Br != 128.
 */
ATTN_API int attn_prefill_qk8(const void* Q8, const void* K8, const float* q_scales,
                              const float* k_scales, const void* V, void* O, int B, int Hq,
                              int Hkv, int N, int d, int causal, float tau, int Br, int Bc,
                              void* stream, uint8_t* skip_mask);

/*
 * int8 quantisation (for attn_prefill_qki8): as attn_quantize_e4m3, with the
 * scale s = 2^k, k the smallest integer >= -126 such that max|x| <= 127 * 2^k,
 * and q[i] = the integer nearest x[i] / s, ties to even, as a signed byte
 * (|q| <= 127).  q * s is exactly representable in bf16.  Same arguments,
 * ownership and errors as attn_quantize_e4m3.
 */
ATTN_API int attn_quantize_i8(const void* x, void* q, float* scales, long long groups,
                              long long group_elems, void* stream);

/*
 * Prefill with S = Q K^T from signed int8 operands on the tensor cores (kind
 * i8, int32 accumulation, exact); P*V stays bf16.  Q8 and K8 as written by
 * attn_quantize_i8 with one group per head slab; otherwise as
 * attn_prefill_qk8 (d = 128 and Br = 128 only, same errors).
 */
ATTN_API int attn_prefill_qki8(const void* Q8, const void* K8, const float* q_scales,
                               const float* k_scales, const void* V, void* O, int B, int Hq,
                               int Hkv, int N, int d, int causal, float tau, int Br, int Bc,
                               void* stream, uint8_t* skip_mask);

/*
 * Prefill with part of the exponentials computed in software on the FMA pipes
 * instead of the exponential unit (MUFU): the SAS idea of "TurboAttention:
 * Efficient Attention Approximation for High-Throughput LLM Serving"
 * (Technical Deep Dive: SAS), written for base 2 and bf16 probabilities.
 * 2^x is split into an integer part j = rint(x), added to the exponent field
 * of the bf16 result, and a degree-3 minimax polynomial of the fraction
 * f = x - j in [-1/2, 1/2]; the bf16 result is within one ulp of 2^x
 * correctly rounded.  poly_pairs of every 16 pairs of key columns take the
 * polynomial (0, 4 or 8; 0 computes every exponential on MUFU and equals
 * attn_prefill_ex bit for bit); the row sum adds the same bf16 values the
 * P*V product multiplies, whichever unit made them.  Otherwise as
 * attn_prefill_ex, for d = 128 and Br = Bc = 128 only.
 *   Errors: as attn_prefill_ex, plus ATTN_ERR_INVALID_ARG for poly_pairs not
 *   in {0, 4, 8} or another d, Br or Bc.
 */
ATTN_API int attn_prefill_poly(const void* Q, const void* K, const void* V, void* O, int B, int Hq,
                               int Hkv, int N, int d, int causal, float tau, int Br, int Bc,
                               int poly_pairs, void* stream, uint8_t* skip_mask);

/*
 * Prefill with the inputs and the output in host memory: the batch is cut
 * into chunks of `chunk` KV-head groups (a group is one KV head of one
 * sequence and the Hq/Hkv query heads that read it, B*Hkv groups in all;
 * 0: an eighth of them, rounded up) that flow through two library-owned
 * device buffer sets on two library streams, so the copy of
 * one chunk to the device overlaps the kernel and the copy back of the
 * previous one.  Qh, Kh, Vh, Oh are host pointers with the layouts of
 * attn_prefill; page-locked (pinned) memory is needed for the copies to
 * overlap.  The call is asynchronous and ordered on `stream` (cudaStream_t as
 * void*, NULL = legacy stream) like a kernel launch: work queued on `stream`
 * before the call happens before it, and Oh is complete once `stream`
 * reaches the point after the call (e.g. after cudaStreamSynchronize).  The
 * host buffers must stay valid and unmodified until then.  One call at a
 * time per process (calls from several host threads are serialised, their
 * device work may overlap only through their own streams' order).  The
 * device buffers (about 2 chunks of Q, K, V and O) are kept for the next call
 * and freed by attn_shutdown().  Errors: as attn_prefill, plus
 * ATTN_ERR_INVALID_ARG for null host pointers or chunk < 0.
 */
ATTN_API int attn_prefill_host(const void* Qh, const void* Kh, const void* Vh, void* Oh, int B,
                               int Hq, int Hkv, int N, int d, int causal, float tau, int Br, int Bc,
                               int chunk, void* stream);

/*
 * Decode: one new query token per (batch, query head) against L cached keys,
 * no mask.  The rows of the skip test are the g = Hq/Hkv query heads that
 * share one KV head (they share the V tile that a skip avoids loading).  The
 * key range of each (batch, KV head) is cut into splits of
 * attn_decode_split_len(B, Hkv, L) keys; inside a split, tiles of 64 keys are
 * visited in ascending order and the running maximum starts at -inf.  The
 * split results are merged exactly (log-sum-exp).
 * d in {64, 128}; g in {1, 2, 4, 8}.
 * The plain form allocates (once, and grows when needed) a device workspace
 * that attn_shutdown() frees.
 */
ATTN_API int attn_decode(const void* q, const void* K, const void* V, void* o, int B, int Hq, int Hkv,
                int L, int d, float tau);

/*
 * As attn_decode on an explicit stream with a caller-provided workspace of at
 * least attn_decode_workspace_bytes(B, Hq, Hkv, L, d) bytes (256-byte
 * aligned device memory; ws may be NULL only if ws_bytes is 0, in which case
 * the library's own workspace is used).  skip_mask: nullable device buffer
 * uint8 [B, Hkv, ceil(L/64)] (0 kept, 1 skipped).
 */
ATTN_API int attn_decode_ex(const void* q, const void* K, const void* V, void* o, int B, int Hq, int Hkv,
                   int L, int d, float tau, void* stream, uint8_t* skip_mask, void* ws,
                   size_t ws_bytes);

/*
 * Decode rule variants (bits of `rule` in attn_decode_rule).  The Skip
 * Softmax page compares a block's local maximum with the running maximum of
 * each row and says nothing on which rows of a decode step must agree, or
 * where a split of the key range starts its running maximum:
 *   ATTN_DECODE_RULE_GROUP (0): the rule of attn_decode above.
 *   ATTN_DECODE_RULE_PER_HEAD: every query head takes the test on its own row
 *     and skips its own exponentials and value sums; the V tile is still
 *     loaded iff some head of the group keeps the tile.  skip_mask is then
 *     [B, Hq, ceil(L/64)] (1 = that head skipped the tile).
 *   ATTN_DECODE_RULE_SINK_SEED: the running maximum of every split but the
 *     first starts at each row's maximum over keys [0, 64) of the sequence
 *     (where attention sinks sit) instead of -inf, so a split's first tiles
 *     can be skipped too.  With a single split this changes nothing.
 */
#define ATTN_DECODE_RULE_GROUP 0
#define ATTN_DECODE_RULE_PER_HEAD 1
#define ATTN_DECODE_RULE_SINK_SEED 2

/*
 * attn_decode_ex with a rule variant (a combination of the bits above; other
 * bits: ATTN_ERR_INVALID_ARG).  rule = 0 is exactly attn_decode_ex.
 */
ATTN_API int attn_decode_rule(const void* q, const void* K, const void* V, void* o, int B, int Hq,
                              int Hkv, int L, int d, float tau, int rule, void* stream,
                              uint8_t* skip_mask, void* ws, size_t ws_bytes);

/*
 * Decode from a paged KV cache (the layout serving engines keep: fixed-size
 * pages in one pool, a per-sequence table of page ids, ragged lengths).
 *   K_pages, V_pages  page pools, bf16 [num_pages, Hkv, 64, d]: page p holds
 *                     64 consecutive keys of every KV head of one sequence.
 *   block_table       device int32 [B, max_pages_per_seq]: entry (b, t) is the
 *                     page holding keys [64 t, 64 t + 64) of sequence b.
 *                     Only entries t < ceil(len_b / 64) are read.
 *   seq_lens          device int32 [B]: len_b, the keys of sequence b; used as
 *                     min(len_b, max_seq_len).  len_b must be >= 1 (a row with
 *                     no key has no softmax; its output is NaN).
 *   max_seq_len       the longest sequence (<= 64 * max_pages_per_seq); the
 *                     split layout is that of attn_decode_ex with L = max_seq_len.
 *   Keys past len_b inside the last page may hold anything (NaN included);
 *   they are masked.  A page id outside [0, num_pages) reads zeros (no fault).
 *   skip_mask (nullable): [B, Hkv, ceil(max_seq_len/64)], or [B, Hq, ...] with
 *   ATTN_DECODE_RULE_PER_HEAD; tiles past len_b are marked 2 (not visited).
 *   Other arguments and errors as attn_decode_rule; ATTN_ERR_INVALID_ARG also
 *   for null or unaligned block_table / seq_lens, num_pages or
 *   max_pages_per_seq <= 0, and max_seq_len > 64 * max_pages_per_seq.
 */
ATTN_API int attn_decode_paged(const void* q, const void* K_pages, const void* V_pages,
                               const int32_t* block_table, const int32_t* seq_lens, void* o, int B,
                               int Hq, int Hkv, int num_pages, int max_pages_per_seq,
                               int max_seq_len, int d, float tau, int rule, void* stream,
                               uint8_t* skip_mask, void* ws, size_t ws_bytes);

/*
 * Decode that allocates nothing, for callers that cannot allocate device
 * memory (a serving engine that has reserved all of HBM for its own pools, a
 * latency-critical loop that must not meet the implicit synchronisation of
 * cudaMalloc/cudaFree, a minimal binding that can only pass q, K, V and o).
 * The pages have no counterpart: this is a deployment variant of attn_decode.
 *   Same arguments, layouts and results as attn_decode_ex; the per-split
 *   scratch lives in a fixed 16 MiB array in device global memory, reserved
 *   on every GPU that loads the library and kept until the process exits.
 *   The first call on a device looks up that array's device address; make
 *   that first call before any stream capture.  Every call shares the array
 *   and leaves its contents behind (nothing in it needs clearing: each entry
 *   read is written earlier in the same call, also when a bounded wait gives
 *   up, in which case o is 0 for the affected rows and attn_sync_status()
 *   reports ATTN_ERR_TIMEOUT), so calls that overlap on the GPU -- on
 *   different streams, or from different threads -- race.
 *   Errors: as attn_decode_ex, plus ATTN_ERR_UNSUPPORTED when the problem
 *   needs more than 16 MiB of scratch (about B*Hq*splits*(d+1)*4 bytes).
 *   Calls no cudaMalloc, cudaFree or allocating library routine.
 */
ATTN_API int attn_decode_noalloc(const void* q, const void* K, const void* V, void* o, int B,
                                 int Hq, int Hkv, int L, int d, float tau, void* stream,
                                 uint8_t* skip_mask);

/* Split length in keys (a multiple of 64) used by decode: a deterministic
 * function of (B, Hkv, L) only.  Returns -1 for non-positive arguments. */
ATTN_API int attn_decode_split_len(int B, int Hkv, int L);

/* Key-tile size of the decode skip test (64). */
ATTN_API int attn_decode_tile(void);

/* Workspace bytes attn_decode_ex needs; 0 for invalid arguments. */
ATTN_API size_t attn_decode_workspace_bytes(int B, int Hq, int Hkv, int L, int d);

/* Stream used by the plain forms (cudaStream_t as void*; NULL = legacy). */
ATTN_API int attn_set_stream(void* stream);

/* Synchronise the current device, then report and clear the device status
 * word: ATTN_OK, or ATTN_ERR_TIMEOUT if a kernel gave up on a bounded wait
 * (attn_last_timeout_site() then names the wait), or ATTN_ERR_CUDA. */
ATTN_API int attn_sync_status(void);

/* Site code of the last wait that gave up (0 if none), for diagnostics. */
ATTN_API int attn_last_timeout_site(void);

/* Limit, in milliseconds, of every bounded wait inside the kernels
 * (default 2000).  Values < 1 are rejected. */
ATTN_API int attn_set_wait_limit_ms(int ms);

/* Test support for the timeout path (no fault, trap or hang is involved).
 * which = 1: every CTA of the following attn_decode / attn_decode_ex calls
 * withholds the copy of its first V tile, so every wait for that tile runs
 * out after the limit set by attn_set_wait_limit_ms; the kernel then records
 * ATTN_DEVICE_TIMEOUT_BASE + 20 in the status word, leaves no copy in flight
 * and returns, and attn_sync_status() reports ATTN_ERR_TIMEOUT.  The output
 * of such a call is undefined.  which = 0 restores normal operation (the
 * default).  Other values: ATTN_ERR_INVALID_ARG.  Not thread-safe with
 * respect to calls in flight on other host threads. */
ATTN_API int attn_test_withhold_copy(int which);

/* Human-readable name of a status code (static string). */
ATTN_API const char* attn_status_string(int status);

/* Free the library-owned decode workspace on every device it was allocated. */
ATTN_API void attn_shutdown(void);

#ifdef __cplusplus
}
#endif

#endif /* SKIP_SOFTMAX_ATTN_H */
