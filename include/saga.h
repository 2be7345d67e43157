/*
 * saga.h - C ABI of libsaga: the SAGA + Atop-N single-token decode-attention
 * step on NVIDIA B200 (sm_100a).
 *
 * Source of the operation: "More Value per Key: Asymmetric Sparse Attention
 * for Faster LLM Decoding" (Elata, Lamprecht, Shechter, Ohayon, Hubara,
 * Soudry).  One decode step of one attention layer:
 *   - append the new token's key and value rows to the KV cache;
 *   - score the token's queries against every cached key,
 *     A = q K^T / sqrt(d)                                      (eq. 2);
 *   - keep the positions whose score is at least a per-query-head threshold
 *     (Atop-N step 1); every R steps that threshold is recomputed exactly as
 *     the N-th largest score of the row and reused in between (Atop-N step 2);
 *   - O = softmax(A[i]) V[i] over the kept positions i          (eq. 7);
 *   - key and value head counts are independent, h_k != h_v     (SAGA).
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are DEVICE pointers owned by the caller.  The
 *     library never allocates, frees or synchronizes; every call only
 *     enqueues work on `stream` (a cudaStream_t passed as void*, NULL = the
 *     legacy default stream) and returns.
 *   - bf16 means IEEE bfloat16 stored as 16-bit words; fp32 is IEEE binary32.
 *   - Layouts are dense and row-major in the order written:
 *       q        bf16 [B, h_q, d]
 *       k_cache  bf16 [B, h_k, l_cap, d]   (one buffer per layer)
 *       v_cache  bf16 [B, h_v, l_cap, d]   (one buffer per layer)
 *       k_new    bf16 [B, h_k, d]
 *       v_new    bf16 [B, h_v, d]
 *       tau      fp32 [B, h_q]
 *       out      fp32 or bf16 [B, h_q, d]
 *     Base addresses must be 16-byte aligned.
 *   - Query head j reads key head floor(j*h_k/h_q) and value head
 *     floor(j*h_v/h_q) (contiguous groups).  Requires h_q % h_k == 0,
 *     h_q % h_v == 0 and (h_v % h_k == 0 or h_k % h_v == 0);
 *     1 <= h_q/h_k <= 64 (<= 32 when d = 128); d in {64, 128}; h_v/h_k <= 32.
 *   - Sequence length: `seq_len` is the number of valid cached tokens,
 *     including the token appended this step (1 <= seq_len <= l_cap).  If
 *     `seq_len_dev` is not NULL the kernels read the length from that device
 *     int instead, when they run (use this inside CUDA graphs, where the
 *     length changes between replays); `seq_len` must then still be a valid
 *     host-side estimate: it sizes the launch and places the context-split
 *     boundaries, and the last split also covers any tokens beyond it (so a
 *     graph captured at length P stays correct for every later length; pass
 *     the capture-time length).  A device length outside [1, l_cap] is
 *     clamped and flagged in the workspace status word.
 *   - The kernels are launched with programmatic dependent launch
 *     (cudaLaunchAttributeProgrammaticStreamSerialization): each may start
 *     while the previous kernel on the stream finishes, but reads and writes
 *     nothing that kernel can touch before it has completed (its early work
 *     is barrier and TMEM setup and an L2 prefetch of key rows).  Set
 *     SAGA_PDL=0 in the environment for plain stream order.
 *   - Reads of the caches: key rows are loaded in 32-row units, so rows up
 *     to the next multiple of 32 past seq_len - 1 (always below l_cap) may be
 *     read and are ignored.
 *   - Inputs must be finite (no NaN/Inf in q or the caches).
 *   - Return value: SAGA_OK or a negative SAGA_ERR_* code.  Arguments are
 *     validated before anything is enqueued; on an error nothing is
 *     launched and saga_last_error() describes it.  SAGA_ERR_CUDA reports a
 *     launch failure seen by cudaGetLastError after enqueueing.
 */
#ifndef SAGA_H
#define SAGA_H

#include <stddef.h>

#if defined(__GNUC__)
#define SAGA_API __attribute__((visibility("default")))
#else
#define SAGA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

#define SAGA_OK 0
#define SAGA_ERR_ARG (-1)         /* bad pointer, shape, length, N, R or dtype */
#define SAGA_ERR_UNSUPPORTED (-2) /* valid but not implemented (e.g. d = 96)   */
#define SAGA_ERR_WORKSPACE (-3)   /* workspace NULL or smaller than required    */
#define SAGA_ERR_CUDA (-4)        /* CUDA runtime/driver error while enqueueing */

#define SAGA_OUT_F32 0
#define SAGA_OUT_BF16 1

/* Bits of the workspace status word (see saga_get_status). */
#define SAGA_STATUS_LEN_CLAMPED 0x1u /* a device-side length was outside [1, l_cap] */
#define SAGA_STATUS_TIMEOUT 0x2u     /* a pipeline wait gave up (the result is invalid) */

typedef struct saga_shape {
  int batch; /* B */
  int h_q;   /* query heads */
  int h_k;   /* key heads   (SAGA: fewer key heads ...) */
  int h_v;   /* value heads (... than value heads) */
  int d;     /* head dimension: 64 or 128 */
  int l_cap; /* capacity of each cache head, in tokens */
} saga_shape;

/* Bytes of scratch that atopn_refresh_threshold and saga_decode_attn need for
 * this shape on the current device (split partials, the score rows of a
 * refresh step, per-split index lists, a status word).
 * The buffer is caller-owned device memory, 256-byte aligned, zero-filled
 * once before first use; calls on one workspace must not overlap in time.
 * Returns 0 for an invalid shape. */
SAGA_API size_t saga_workspace_bytes(const saga_shape* s);

/* KV cache append (the "KV cache" of the explainer's jargon list): writes
 * k_new into k_cache[:, :, pos, :] and v_new into v_cache[:, :, pos, :].
 * If seq_len_dev is not NULL, pos is read on the device as (*seq_len_dev - 1)
 * and the host `pos` only needs to be in range.  0 <= pos < l_cap. */
SAGA_API int saga_kv_append(const saga_shape* s, void* k_cache, void* v_cache, const void* k_new, const void* v_new, int pos,
                   const int* seq_len_dev, void* stream);

/* Decode-step query/key/value projection fused with the KV cache append
 * (eq. 1 of "More Value per Key: Asymmetric Sparse Attention for Faster LLM
 * Decoding", Attention Mechanism Formalization, with the decoupled head counts
 * of Methodology > SAGA Architecture: h_k key heads, h_v value heads).
 *   x      bf16 [batch, hidden], the new token's hidden state per batch row;
 *   w_qkv  bf16 [(h_q + h_k + h_v) * d, hidden], row-major; row n holds the
 *          weights of output column n: rows [0, h_q d) are W_Q's columns
 *          (query head n / d, dimension n % d), then h_k d rows of W_K, then
 *          h_v d rows of W_V;
 *   q_out  bf16 [batch, h_q, d] (written);
 *   k_cache bf16 [batch, h_k, l_cap, d], v_cache bf16 [batch, h_v, l_cap, d]:
 *          row pos of every head written, nothing else touched.
 * Products accumulate in fp32 (batch 1 on CUDA cores; batch 2 .. 16 on the
 * tensor cores, the hidden dimension split across CTAs and the fp32 partials
 * added in a fixed order, so results are reproducible run to run); each
 * output is rounded once to bf16 (nearest even).  If seq_len_dev is not NULL,
 * pos is read on the device as (*seq_len_dev - 1), clamped into [0, l_cap)
 * (the clamp is not flagged in the status word: the attention call that
 * reads the same device length flags it), and the host pos only needs to be
 * in range.  Requirements: 1 <= batch <=
 * 16, hidden a positive multiple of 8, 0 <= pos < l_cap, all tensor pointers
 * device memory 16-byte aligned, q_out and the cache rows not overlapping x
 * or w_qkv.  workspace: device memory of saga_qkv_workspace_bytes(s, hidden)
 * bytes, 256-byte aligned, zero-filled once before first use (every call
 * leaves it ready for the next); word 0 is a sticky status word read by
 * saga_get_status (SAGA_STATUS_TIMEOUT if a bounded wait gave up); calls on
 * one workspace must not overlap in time.  The caller owns every buffer.
 * The kernels start loading w_qkv before their programmatic dependency wait
 * (the weight stream overlaps the end of the preceding kernel): w_qkv must
 * not be written by work that can still be running when this call's kernels
 * start, i.e. by a kernel launched earlier on the stream that releases its
 * dependents early (programmatic launch completion).  Weights written by a
 * copy, by an ordinary kernel or on another synchronized stream are fine; x,
 * the caches and the device length are read after the wait.
 * Errors: SAGA_ERR_ARG / SAGA_ERR_UNSUPPORTED / SAGA_ERR_WORKSPACE before
 * anything is enqueued; SAGA_ERR_CUDA if the launch fails. */
SAGA_API int saga_qkv_project(const saga_shape* s, int hidden, const void* x, const void* w_qkv, void* q_out,
                              void* k_cache, void* v_cache, int pos, const int* seq_len_dev, void* workspace,
                              size_t ws_bytes, void* stream);

/* Workspace bytes saga_qkv_project needs for this shape and hidden size on
 * the current device (0 for invalid arguments or without a device). */
SAGA_API size_t saga_qkv_workspace_bytes(const saga_shape* s, int hidden);

/* Atop-N threshold refresh (Atop-N step 1-2, "computed once every n
 * tokens"): tau[b, j] = the n_top-th largest of the fp32 scores
 * A[b, j, 0..seq_len) (eq. 2), counted with multiplicity; -inf when
 * n_top >= seq_len.  Exact: radix selection over order-preserving 32-bit
 * images of the scores, no sort.  n_top >= 1.
 * tau is in/out: its incoming values (the stale thresholds of the last
 * refresh) only steer the work - the selection keeps the scores from the
 * stale threshold's top-byte bin up while it counts the top digit - and any
 * value, NaN and +-inf included, gives the same result bits. */
SAGA_API int atopn_refresh_threshold(const saga_shape* s, const void* q, const void* k_cache, int seq_len,
                            const int* seq_len_dev, int n_top, float* tau, void* workspace, size_t ws_bytes,
                            void* stream);

/* The exact N-th-largest selection alone, over caller-provided fp32 rows:
 * tau[r] = the n_top-th largest of scores[r*row_stride + 0 .. row_len), with
 * multiplicity; -inf when n_top >= row_len.  rows >= 1, 1 <= row_len <=
 * row_stride, row_stride % 4 == 0.  Workspace: at least
 * atopn_select_workspace_bytes(rows). */
SAGA_API size_t atopn_select_workspace_bytes(int rows);
SAGA_API int atopn_select_threshold(const float* scores, int rows, int row_len, long long row_stride, int n_top, float* tau,
                           void* workspace, size_t ws_bytes, void* stream);

/* One decode step of one layer (eqs. 2 and 7 with the Atop-N threshold).
 *   step: decode step index t >= 0; when t % refresh_interval == 0 the
 *         threshold is first recomputed exactly from this step's scores and
 *         written to tau; otherwise tau is read (it must hold the threshold of
 *         the last refresh step).
 *   n_top: N >= 1.  n_top >= seq_len selects every token (dense attention);
 *         pass n_top = l_cap for attention without a threshold.
 *   out_dtype: SAGA_OUT_F32 or SAGA_OUT_BF16 (round to nearest even).
 *   sel_count (nullable): int32 [B, h_q], number of kept positions.
 *   sel_idx (nullable, needs sel_count): int32 [B, h_q, l_cap]; the first
 *         sel_count[b, j] entries are the kept positions in ascending order.
 * The new token's rows must already be in the caches at seq_len - 1
 * (saga_kv_append), or use saga_decode_step. */
SAGA_API int saga_decode_attn(const saga_shape* s, const void* q, const void* k_cache, const void* v_cache, int seq_len,
                     const int* seq_len_dev, int n_top, int refresh_interval, long long step, float* tau, void* out,
                     int out_dtype, int* sel_count, int* sel_idx, void* workspace, size_t ws_bytes, void* stream);

/* Append and attend in one call: saga_kv_append(k_new, v_new, pos =
 * seq_len - 1) followed by saga_decode_attn, with the append done inside
 * the attention kernels (the context split that holds row seq_len - 1
 * writes the key and value rows before it loads them), so a decode step of
 * a layer costs no separate launch for it.  Same arguments and results as
 * saga_decode_attn plus k_new bf16 [B, h_k, d] and v_new bf16 [B, h_v, d];
 * the caches are written. */
SAGA_API int saga_decode_step(const saga_shape* s, const void* q, const void* k_new, const void* v_new, void* k_cache,
                     void* v_cache, int seq_len, const int* seq_len_dev, int n_top, int refresh_interval,
                     long long step, float* tau, void* out, int out_dtype, int* sel_count, int* sel_idx,
                     void* workspace, size_t ws_bytes, void* stream);

/* Tracing: the next saga_decode_attn (or saga_decode_step) call made on this host thread records
 * ev_start on its stream just before its context-split attention kernels
 * (after nothing else of that call) and ev_end just after them, before the
 * cross-split combine.  On a reuse step that is the one fused split kernel;
 * on a refresh step it spans score dump, radix select and the compare/gather
 * pass.  The events are cudaEvent_t handles created by the caller (timing
 * enabled); under stream capture they become external event-record nodes, so
 * graph replays record them too.  One-shot: cleared by that call.  Passing
 * NULLs cancels a pending request. */
SAGA_API int saga_trace_next_attention(void* ev_start, void* ev_end);

/* Allocation-free variant of saga_decode_attn (the paper has no counterpart:
 * this is an integration aid).  Same arguments and results, without the
 * workspace: the scratch is a fixed array of SAGA_NOALLOC_SCRATCH_BYTES in
 * the library's device image, which every device that loads the library
 * holds until the process exits.  For callers that cannot allocate device
 * memory around the call (their memory is owned by another allocator, or an
 * allocation is not allowed at that point).
 *   - Shapes whose saga_workspace_bytes exceeds the scratch are rejected with
 *     SAGA_ERR_WORKSPACE and a message; use saga_decode_attn for those.
 *   - Allocates nothing (no cudaMalloc/cudaFree, no allocating library call).
 *   - The scratch's device address comes from cudaGetSymbolAddress, looked up
 *     on each call made outside stream capture; a call made during capture
 *     uses the address an earlier call found, so make the first call on a
 *     device before any stream capture (else SAGA_ERR_CUDA).
 *   - Arguments are checked first; only then is the scratch's status word
 *     cleared on the stream, ahead of the kernels.
 *   - Every call on a device shares the one scratch array, which keeps the
 *     previous call's contents.  Calls whose work overlaps on the GPU (other
 *     streams, other host threads) race on the scratch: serialize them.
 * saga_noalloc_last_error() describes the last failure of this entry point;
 * saga_noalloc_get_status() reads the status word of the last call on the
 * current device (after synchronizing `stream`). */
#define SAGA_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)
SAGA_API size_t saga_noalloc_scratch_bytes(void);
SAGA_API int saga_decode_attn_noalloc(const saga_shape* s, const void* q, const void* k_cache, const void* v_cache,
                                      int seq_len, const int* seq_len_dev, int n_top, int refresh_interval,
                                      long long step, float* tau, void* out, int out_dtype, int* sel_count,
                                      int* sel_idx, void* stream);
SAGA_API int saga_noalloc_get_status(void* stream, unsigned* status);
SAGA_API const char* saga_noalloc_last_error(void);

/* Test hook for failure detection (no counterpart in the paper).  The next
 * saga_decode_attn / saga_decode_step call on this host thread, if it is a
 * reuse step (step % R != 0) run by the context-split attention kernel,
 * makes that kernel's epilogue wait, for at most limit_ns, on a barrier
 * that nothing arrives at, instead of running.  The wait gives up, the
 * kernel's pipeline unwinds (in-flight copies drained, TMEM freed) and
 * SAGA_STATUS_TIMEOUT is set in the status word; the call's results are then
 * invalid and the context stays usable.  One-shot: consumed by that next
 * call whatever its kind; limit_ns = 0 cancels a pending request. */
SAGA_API int saga_test_expire_next_wait(unsigned limit_ns);

/* ---------------------------------------------------------------------------
 * Closed-form GQA-to-SAGA key-head merge ("More Value per Key", Methodology >
 * GQA-to-SAGA Conversion > Stage 1).  A teacher with h_k key heads is merged
 * into h_k / 2 key heads: for every pair (a, b) of teacher heads, the merged
 * key projection minimising the squared logit error of eq. 13,
 *   L_ab(M) = sum_{j of a} ||Q^j (X M)^T - Q^j (X W_K^a)^T||_F^2 + (same over b),
 * is M(a, b) = (W_K^a S_a + W_K^b S_b)(S_a + S_b)^+ with S_r = sum_{j of r}
 * Q^j^T Q^j (Lemma 4.1, eq. 15); the pairing is the minimum-weight perfect
 * matching with weights w(a, b) = L_ab(M(a, b)) (Theorem 4.2, eq. 14).
 *
 * Inputs (device memory, caller-owned, 16-byte aligned):
 *   x     bf16 [tokens, hidden]   calibration hidden states X (rows = tokens)
 *   q     bf16 [tokens, h_q, d]   the teacher's queries Q^j on the same tokens
 *   w_k   fp32 [h_k, hidden, d]   teacher key projections (keys = X W_K^r)
 * Query head j belongs to key head floor(j * h_k / h_q) (contiguous groups).
 * Outputs:
 *   pair_loss  fp32 [h_k, h_k]        w(a, b), symmetric, zero diagonal
 *   pairing    int32 [h_k]            partner of every teacher head
 *   w_k_merged fp32 [h_k/2, hidden, d] M(a, b) of the chosen pairs, ordered
 *                                      by their smaller head
 * Arithmetic: G = X^T X and the S_r are formed on the tensor cores (bf16
 * products, fp32 sums); the pseudoinverse (Jacobi eigen-decomposition,
 * eigenvalues below 1e-5 of the largest count as zero), M and the losses are
 * fp64.  Ties between pairings go to the first in the order that pairs the
 * lowest unmatched head with each remaining head in ascending order.
 * Constraints: d in {64, 128}; h_k even, 2 <= h_k <= 16 (the matching is
 * exhaustive); h_q % h_k == 0.  Errors as for the decode calls; the
 * workspace (saga_merge_workspace_bytes, 256-byte aligned) starts with a
 * status word readable by saga_get_status.  saga_merge_last_error()
 * describes the last failure of these two calls. */
typedef struct saga_merge_shape {
  int tokens; /* T: calibration tokens */
  int hidden; /* D: rows of each key projection */
  int d;      /* head dimension */
  int h_q;    /* teacher query heads */
  int h_k;    /* teacher key heads (merged in pairs) */
} saga_merge_shape;
SAGA_API size_t saga_merge_workspace_bytes(const saga_merge_shape* s);
SAGA_API int saga_key_head_merge(const saga_merge_shape* s, const void* x, const void* q, const float* w_k,
                                 float* pair_loss, int* pairing, float* w_k_merged, void* workspace,
                                 size_t ws_bytes, void* stream);
SAGA_API const char* saga_merge_last_error(void);

/* Measurement aid (no counterpart in the paper): one streaming read of
 * `bytes` of device memory at buf (16-byte aligned; the last bytes % 16 are
 * not read), 16-byte loads with four in flight per thread over a grid of up
 * to four CTAs per SM.  Timed by the caller (events on `stream`), it gives
 * the pure-read HBM ceiling that the read-dominated attention kernels are
 * held to.  sink: device array of at least saga_read_probe_sink_words()
 * words (written, so no load is dropped).  Errors: SAGA_ERR_ARG for a NULL
 * or misaligned pointer or bytes < 16, SAGA_ERR_CUDA for a launch error. */
SAGA_API size_t saga_read_probe_sink_words(void);
SAGA_API int saga_read_probe(const void* buf, size_t bytes, unsigned* sink, void* stream);

/* Reads the workspace status word (SAGA_STATUS_* bits ORed by the kernels
 * since the workspace was zeroed) after synchronizing `stream`. */
SAGA_API int saga_get_status(const void* workspace, void* stream, unsigned* status);

/* Text of the last error reported on this host thread ("" if none). */
SAGA_API const char* saga_last_error(void);

/* ABI version (major * 100 + minor). */
SAGA_API int saga_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SAGA_H */
