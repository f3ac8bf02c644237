/*
 * rtp.h -- C ABI of the B200 (sm_100a) RTPurbo sparse-attention library (librtp.so).
 *
 * What is computed (one attention layer at inference time):
 *   - retrieval heads: a 16-dim token indexer scores every cached key,
 *       s_j = (P q) . (P k_j) / 4,
 *     each query keeps the smallest set of keys whose softmax-over-s mass
 *     reaches p (dynamic top-p; keys ordered by score descending, ties to the
 *     lower position), and exact 128-dim attention runs over that set only;
 *   - local heads: causal sliding-window attention over the last W keys.
 *   The pages this follows: "Full Attention Strikes Back: Transferring Full
 *   Attention into Sparse within Hundred Training Steps (RTPurbo)", TL;DR;
 *   "RTPurbo: Turning Dense LLMs into Sparse Attention Models with Just a Few
 *   Hundred Training Steps", "Three Key Insights" 1-3 and "The RTPurbo
 *   Method" 2.  The 1/4 score scale, the tie rule and the window bounds are
 *   this library's readings of what the pages leave open.
 *
 * Conventions shared by every call
 *   - Tensors are described by rtp_tensor: 4-D, strides in elements, the last
 *     dimension contiguous (stride[3] == 1), base address and every other
 *     stride 16-byte aligned.  Layout [B, H, N or T, D] ("head major"); any
 *     other memory order is expressed through the strides.  An empty tensor
 *     (a zero among its first three dimensions) may have a NULL base.
 *   - Every pointer is a DEVICE pointer on the current device, allocated and
 *     owned by the caller.  The library allocates nothing on any call: calls
 *     that need scratch take a caller workspace (256-byte aligned) whose size
 *     the matching *_workspace_size() reports.  A workspace must be
 *     zero-filled once before its first use (e.g. cudaMemsetAsync); every call
 *     leaves it ready for the next call.  Calls that share a workspace must
 *     not overlap on the GPU (use one stream, or one workspace per stream).
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream).  Arguments are validated on the host before any
 *     launch; on an error status nothing is launched and nothing is written.
 *   - Query head h reads KV head h / (Hq / Hk) (grouped-query attention).
 *   - Sequence lengths: `lens` is an optional device int32[B]; sequence b
 *     holds lens[b] keys (positions 0 .. lens[b]-1, clamped to [0, N]); NULL
 *     means N for every sequence.  The T queries of sequence b are its last T
 *     tokens: query t sits at position lens[b] - T + t.  A query whose
 *     position is negative has no keys and gets an all-zero output.
 *   - Scores, top-p masses and softmax statistics are fp32; top-p masses are
 *     accumulated in 64-bit fixed point so the selected set does not depend
 *     on thread scheduling.  Attention accumulates in fp32.
 */
#ifndef RTP_H_
#define RTP_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define RTP_API __attribute__((visibility("default")))
#else
#define RTP_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ------------------------------------------------------ */
typedef int32_t rtp_status;
#define RTP_OK               0
#define RTP_ERR_INVALID_ARG  1  /* null pointer, p not in (0, inf), W < 1, bad scale */
#define RTP_ERR_SHAPE        2  /* inconsistent or unsupported shapes (D != 128, d != 16, Hq % Hk, G > 8) */
#define RTP_ERR_DTYPE        3  /* unsupported dtype combination */
#define RTP_ERR_ALIGNMENT    4  /* base or stride not 16-byte aligned, or stride[3] != 1 */
#define RTP_ERR_WORKSPACE    5  /* workspace NULL or smaller than *_workspace_size() */
#define RTP_ERR_CUDA         6  /* a CUDA runtime call failed; see rtp_last_cuda_error() */
#define RTP_ERR_UNSUPPORTED  7  /* valid but outside what this build implements (e.g. N too large) */

typedef int32_t rtp_dtype;
#define RTP_F32   0
#define RTP_BF16  1

/* Opaque CUDA stream (binary compatible with cudaStream_t). */
typedef struct CUstream_st* rtp_stream_t;

typedef struct rtp_tensor {
  void*   data;       /* device pointer */
  int32_t dtype;      /* RTP_F32 or RTP_BF16 */
  int32_t ndim;       /* must be 4 */
  int64_t shape[4];
  int64_t stride[4];  /* elements */
} rtp_tensor;

/*
 * Per-query result of the top-p cut (one entry per query row r, with
 * r = (b * Hq + h) * T + t over the q_idx tensor's [B, Hq, T] dims).
 *   key j of query r is selected  iff  s_j > tau  or  (s_j == tau and j <= tiepos)
 * where tau is the fp32 value with bit pattern tau_bits[r].
 *   tau_bits  uint32[R]  bit pattern of the cut score (tau); -inf when p >= 1
 *   tiepos    int32[R]   last selected position among keys scoring exactly tau
 *                        (-1 for a query with no candidates)
 *   count     int32[R]   number of selected keys
 *   mask      uint32[R, mask_words] or NULL: bit (j % 32) of word j / 32 is set
 *             iff key j is selected; bits at positions >= lens[b] are 0.
 *             Required by rtp_sparse_attn_decode; optional elsewhere.
 *   mask_words  row stride of `mask` in words, >= ceil(N / 32).
 */
typedef struct rtp_selection {
  uint32_t* tau_bits;
  int32_t*  tiepos;
  int32_t*  count;
  uint32_t* mask;
  int64_t   mask_words;
} rtp_selection;

/* ---- a1: the 16-dim token indexer projection ---------------------------
 * x_idx[b, h, n, :] = P[h / (H / HP)] @ x[b, h, n, :]
 *   x      [B, H, N, 128]   f32 or bf16, post-rotary keys or queries
 *   P      [HP, 16, 128]    f32, contiguous; H must be a multiple of HP
 *   x_idx  [B, H, N, 16]    f32 or bf16 (output; fp32 dot, rounded to nearest even)
 * Cites: "RTPurbo: Turning Dense LLMs ...", "Three Key Insights" 2 (a 16-dim
 * low-frequency projection ranks tokens); "The RTPurbo Method" 2 (learned P).
 */
RTP_API rtp_status rtp_index_project(const rtp_tensor* x, const rtp_tensor* P, const rtp_tensor* x_idx,
                             rtp_stream_t stream);

/* ---- a2 + a3: indexer scores and the dynamic top-p cut -----------------
 *   q_idx  [B, Hq, T, 16]   f32 or bf16 (projected queries)
 *   k_idx  [B, Hk, N, 16]   same dtype (projected keys); Hq multiple of Hk
 *   lens   int32[B] device or NULL
 *   p      top-p mass, > 0; p >= 1 selects every candidate
 *   out    rtp_selection (device arrays sized for B*Hq*T rows)
 * Query (b, h, t) ranks keys 0 .. pos by s = (q_idx . k_idx[j]) / 4 (fp32, fixed
 * summation order), weights exp(s - max s), and keeps the shortest prefix of
 * the (s desc, position asc) order whose weight reaches p * Z.
 * T == 1 (decode) is implemented for N <= 2097152 (past 524288 keys the
 * workspace holds the scores the chip cannot keep: 4 bytes per key and query
 * beyond 524288); T > 1 (prefill) uses the tensor-core score tiles.
 * Workspace: rtp_topp_select_workspace_size() (0 for prefill and short caches).
 * Cites: "RTPurbo: Turning Dense LLMs ...", "Three Key Insights" 3 (cumulative
 * top-p per query); "Full Attention Strikes Back ... (RTPurbo)", Key findings.
 */
RTP_API rtp_status rtp_topp_select(const rtp_tensor* q_idx, const rtp_tensor* k_idx, const int32_t* lens,
                           float p, const rtp_selection* out, void* workspace, size_t workspace_bytes,
                           rtp_stream_t stream);
RTP_API size_t rtp_topp_select_workspace_size(int64_t B, int64_t Hq, int64_t T, int64_t Hk, int64_t N);

/* ---- a3 variant: a fixed top-k cut through the same selection -------------
 * Decode form (T == 1) only; arguments and results as rtp_topp_select, with k
 * in place of p: query (b, h) keeps the min(k, n) keys of highest indexer
 * score s (ties to the lower position), n = lens[b] (or N).  k < 1 is
 * RTP_ERR_INVALID_ARG, T != 1 RTP_ERR_UNSUPPORTED.  The kernel is the top-p
 * selection's with every key weighing 1, so its passes count keys.
 * Cites: "Full Attention Strikes Back ... (RTPurbo)", Key findings (dynamic
 * top-p set against a fixed top-k budget); "RTPurbo: Turning Dense LLMs ...",
 * "Three Key Insights" 3.  Workspace: rtp_topp_select_workspace_size().
 */
RTP_API rtp_status rtp_topk_select(const rtp_tensor* q_idx, const rtp_tensor* k_idx, const int32_t* lens,
                                   int32_t k, const rtp_selection* out, void* workspace, size_t workspace_bytes,
                                   rtp_stream_t stream);

/* ---- cache maintenance: appending new tokens --------------------------------
 *   k_new, v_new [B, H, T, 128]  bf16 or f32, post-rotary keys / values of the
 *                T new tokens of each sequence (all H KV heads)
 *   pos          int32[B] device: position of new token 0 in sequence b
 *   R            the first R KV heads are retrieval heads (0 <= R <= H)
 *   P            [R, 16, 128] f32 (unused, may be NULL, when R == 0)
 *   k_cache, v_cache [B, R, N, 128]  full caches of the retrieval heads:
 *                row pos+t receives token t (tokens outside [0, N) are dropped)
 *   k_idx        [B, R, N, 16]  projected keys: row pos+t receives P k_t,
 *                bit-identical to rtp_index_project of that row
 *   k_ring, v_ring [B, H - R, W, 128]  local heads' rings of W rows: token at
 *                position p goes to row p mod W (of the T tokens only the last
 *                W are written)
 *   lens_out     int32[B] device or NULL (not the pos buffer): receives pos + T,
 *                clamped to [0, N] when R > 0, i.e. the sequence length after the
 *                append and the `pos` of the next one
 *   ring_lens    int32[B] device or NULL (must be NULL when R == H): receives
 *                min(pos + T, W), the number of ring rows in use, i.e. the
 *                `lens` of rtp_window_attn over the ring with window W (after
 *                in-order appends the ring holds exactly the keys of the newest
 *                token's window, in slot order; attention does not depend on
 *                the order of its keys)
 * Caches, rings and P are NULL-able only for the head group that is empty.  All
 * tensors share the dtype of k_new (P is f32).  pos[b] + T must fit in int32.
 * pos, lens_out and ring_lens are three distinct buffers.  One launch, one pass
 * over the new rows.
 * Errors: INVALID_ARG (NULL pos, R outside [0, H], aliased length buffers),
 * SHAPE / DTYPE / ALIGNMENT as for the other calls; nothing is written then.
 * Cites: "RTPurbo: Turning Dense LLMs ...", "Three Key Insights" 1 (retrieval
 * heads keep the full cache, local heads a local window); "Full Attention
 * Strikes Back ... (RTPurbo)", TL;DR (a lightweight token indexer).
 */
RTP_API rtp_status rtp_kv_append(const rtp_tensor* k_new, const rtp_tensor* v_new, const int32_t* pos, int32_t R,
                                 const rtp_tensor* P, const rtp_tensor* k_cache, const rtp_tensor* v_cache,
                                 const rtp_tensor* k_idx, const rtp_tensor* k_ring, const rtp_tensor* v_ring,
                                 int32_t* lens_out, int32_t* ring_lens, rtp_stream_t stream);

/* ---- a4 (decode): exact attention over each query's selected keys -------
 *   q      [B, Hq, 1, 128]  bf16 or f32 (retrieval query heads)
 *   k, v   [B, Hk, N, 128]  same dtype (full KV cache of the retrieval heads)
 *   sel    selection from rtp_topp_select on the same [B, Hq, 1] rows; its
 *          mask is required
 *   scale  softmax scale (1/sqrt(128) for the usual attention)
 *   o      [B, Hq, 1, 128]  f32 or bf16 output
 * o = sum_{j in S} softmax_j(scale * q.k_j) v_j (empty S gives 0).  Each K/V
 * row selected by any head of a GQA group is read once for the group.
 * Hq / Hk <= 8.  Workspace: rtp_sparse_attn_decode_workspace_size().
 * Cites: "Full Attention Strikes Back ... (RTPurbo)", TL;DR (full KV cache for
 * retrieval heads, sparse attention over the indexed tokens).
 */
RTP_API rtp_status rtp_sparse_attn_decode(const rtp_tensor* q, const rtp_tensor* k, const rtp_tensor* v,
                                  const int32_t* lens, const rtp_selection* sel, float scale,
                                  const rtp_tensor* o, void* workspace, size_t workspace_bytes,
                                  rtp_stream_t stream);
RTP_API size_t rtp_sparse_attn_decode_workspace_size(int64_t B, int64_t Hq, int64_t Hk, int64_t N);

/* ---- a4 (decode) over one key range of longer sequences ------------------
 * For a sequence whose keys are split by position across devices (each holds
 * the K/V rows of one contiguous range and the full selection): attention of
 * each query over its selected keys inside this range, plus the log-sum-exp
 * that rtp_attn_combine needs to merge the ranges.
 *   q, sel, scale  as for rtp_sparse_attn_decode (sel covers the whole
 *          sequence; keys past mask_words * 32 count as not selected, so the
 *          last range may run past the sequence's end)
 *   k, v   [B, Hk, N, 128]  rows 0 .. N-1 hold keys key_lo .. key_lo + N - 1
 *   lens   int32[B] device or NULL: whole-sequence lengths (keys at or past
 *          lens[b] are not attended); NULL means key_lo + N
 *   key_lo global position of row 0; a multiple of 64, >= 0
 *   o      [B, Hq, 1, 128] f32 or bf16: attention over the range's selected
 *          keys, normalised within the range (0 when it has none)
 *   lse    [B, Hq] f32 (last dim contiguous): ln sum_j exp(scale * q.k_j) over
 *          those keys (-inf when none)
 * Workspace: rtp_sparse_attn_decode_workspace_size(B, Hq, Hk, N).  Errors as
 * rtp_sparse_attn_decode, plus INVALID_ARG for a bad key_lo or a NULL lse.
 * Cites: "Full Attention Strikes Back ... (RTPurbo)", TL;DR (retrieval heads
 * attend the indexed tokens of the full cache); softmax over a union of
 * disjoint key sets is the lse-weighted mean of the per-set results.
 */
RTP_API rtp_status rtp_sparse_attn_decode_range(const rtp_tensor* q, const rtp_tensor* k, const rtp_tensor* v,
                                                const int32_t* lens, const rtp_selection* sel, int64_t key_lo,
                                                float scale, const rtp_tensor* o, const rtp_tensor* lse,
                                                void* workspace, size_t workspace_bytes, rtp_stream_t stream);

/* ---- merge of key-range partials ---------------------------------------------
 *   o_parts   [S, B, Hq, 128] f32: S partial outputs (rtp_sparse_attn_decode_range
 *             or any attention normalised over its own key set)
 *   lse_parts [S, B, Hq] f32 (last dim contiguous): their log-sum-exps
 *   o         [B, Hq, 1, 128] f32 or bf16
 * o = sum_s exp(lse_s - M) o_s / sum_s exp(lse_s - M), M = max_s lse_s; rows
 * whose partials are all empty (lse = -inf) get 0.  A partial with lse = 0
 * and every other -inf passes through unchanged (used for heads that one
 * device computes alone).  One launch, one warp per row.
 */
RTP_API rtp_status rtp_attn_combine(const rtp_tensor* o_parts, const rtp_tensor* lse_parts, const rtp_tensor* o,
                                    rtp_stream_t stream);

/* ---- a4 (decode) without a caller workspace ------------------------------
 * The pages have no counterpart to this call: it is a library-level variant
 * of rtp_sparse_attn_decode (same arguments and results, minus the
 * workspace) for callers that cannot allocate device memory -- for example a
 * plugin inside a host framework that owns every device allocation and gives
 * its plugins no allocator, or a runtime that reserves all device memory at
 * start-up and forbids allocation afterwards.
 *   - The split-K scratch lives in a fixed device array inside librtp.so,
 *     RTP_NOALLOC_SCRATCH_BYTES long, which every GPU that loads the library
 *     keeps until the process exits.  Shapes whose scratch would exceed it
 *     (rtp_sparse_attn_decode_workspace_size() > RTP_NOALLOC_SCRATCH_BYTES)
 *     return RTP_ERR_UNSUPPORTED.
 *   - The first call in a CUDA context (on a device, with that context
 *     current) looks up the array's device address; make that first call
 *     before any stream capture.  After a device reset, or in another context
 *     on the same device, the next call looks it up again.
 *   - Every argument is checked first: an error status means nothing was
 *     enqueued and the array was not touched.
 *   - All calls on a device share the array: calls that overlap on the GPU
 *     race.  Order them on one stream.  Each call clears the part of the array
 *     that must start at zero; the rest keeps the previous call's contents.
 *   - Nothing is allocated: no cudaMalloc, cudaFree or allocating routine.
 */
#define RTP_NOALLOC_SCRATCH_BYTES (4u << 20)
RTP_API rtp_status rtp_sparse_attn_decode_noalloc(const rtp_tensor* q, const rtp_tensor* k, const rtp_tensor* v,
                                                  const int32_t* lens, const rtp_selection* sel, float scale,
                                                  const rtp_tensor* o, rtp_stream_t stream);

/* ---- a4 (prefill): causal attention over each query's selected keys ----
 *   q      [B, Hq, T, 128]  bf16;  k, v [B, Hk, N, 128] bf16
 *   q_idx  [B, Hq, T, 16], k_idx [B, Hk, N, 16]  bf16 (the inputs the selection used)
 *   sel    threshold form (tau_bits, tiepos) from rtp_topp_select on q_idx/k_idx
 *   o      [B, Hq, T, 128]  f32 or bf16
 * Key j is attended by query t iff j <= pos_t and it is selected: the kernel
 * recomputes s_j with the same tensor-core instruction as the selection, so
 * the predicate is evaluated on bit-identical scores.
 * Cites: as rtp_sparse_attn_decode, plus "Three Key Insights" 3.
 */
RTP_API rtp_status rtp_sparse_attn_prefill(const rtp_tensor* q, const rtp_tensor* k, const rtp_tensor* v,
                                   const rtp_tensor* q_idx, const rtp_tensor* k_idx,
                                   const int32_t* lens, const rtp_selection* sel, float scale,
                                   const rtp_tensor* o, void* workspace, size_t workspace_bytes,
                                   rtp_stream_t stream);
RTP_API size_t rtp_sparse_attn_prefill_workspace_size(int64_t B, int64_t Hq, int64_t T, int64_t Hk, int64_t N);

/* ---- a5: causal sliding-window attention (local heads) -----------------
 *   q      [B, Hq, T, 128]  bf16 or f32;  k, v [B, Hk, N, 128] same dtype
 *   W      window, >= 1: query at position i attends keys max(0, i-W+1) .. i
 *   o      [B, Hq, T, 128]  f32 or bf16
 * T == 1 is the decode form.  Workspace: rtp_window_attn_workspace_size().
 * Cites: "RTPurbo: Turning Dense LLMs ...", "Three Key Insights" 1 (local heads
 * keep only a local window).
 */
RTP_API rtp_status rtp_window_attn(const rtp_tensor* q, const rtp_tensor* k, const rtp_tensor* v,
                           const int32_t* lens, int32_t W, float scale, const rtp_tensor* o,
                           void* workspace, size_t workspace_bytes, rtp_stream_t stream);
RTP_API size_t rtp_window_attn_workspace_size(int64_t B, int64_t Hq, int64_t T, int64_t Hk, int64_t N, int32_t W);

/* ---- device-side errors -------------------------------------------------
 * Kernels that wait on asynchronous copies or tensor-core completions give up
 * after about two seconds instead of hanging, and record a code in a device
 * word.  rtp_poll_device_error synchronises the device, stores that code in
 * *code (0: nothing happened; RTP_DEVICE_ERR_TIMEOUT: a wait gave up and the
 * affected outputs are invalid) and clears it.
 */
#define RTP_DEVICE_ERR_TIMEOUT 1
RTP_API rtp_status rtp_poll_device_error(int32_t* code);
/* Budget, in GPU clock cycles, of each bounded device wait in the prefill
 * kernels launched after this call (process-wide).  0 restores the default
 * (4e9 cycles, about two seconds); a negative value is RTP_ERR_INVALID_ARG.
 * A diagnostic knob: a tiny budget makes waits give up on purpose, which is
 * how the give-up path is tested; the results of such a launch are invalid,
 * the error word reports RTP_DEVICE_ERR_TIMEOUT, and the next launch with the
 * default budget is unaffected (a kernel that gives up still waits for the
 * copies and tensor-core operations it issued before it exits). */
RTP_API rtp_status rtp_set_wait_budget_cycles(int64_t cycles);

/* ---- utilities ---------------------------------------------------------- */
RTP_API const char* rtp_status_string(rtp_status s);   /* static string, never NULL */
RTP_API int32_t rtp_last_cuda_error(void);              /* cudaError_t of the last RTP_ERR_CUDA on this thread */
RTP_API int32_t rtp_version(void);                      /* major * 10000 + minor * 100 + patch */

#ifdef __cplusplus
}
#endif
#endif /* RTP_H_ */
