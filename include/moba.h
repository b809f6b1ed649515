/*
 * moba.h — C ABI of the MoBA (Mixture of Block Attention) causal-prefill
 * forward for NVIDIA B200 (sm_100a).
 *
 * Method: "MoBA: Mixture of Block Attention for Long-Context LLMs"
 * (arXiv 2502.13189).  Section names below are those of the paper-graph
 * summary page of that paper ([summary]); [note] is the research-hub concept
 * note "MoBA (Mixture of Block Attention)", "Key math / How it works"; [review]
 * is the paperhub.cn OpenReview discussion page of the paper (reviews and
 * author rebuttals).
 *
 * The forward pass is three calls on one CUDA stream:
 *   moba_block_meanpool  pooled key of every size-B block      ([summary] §3
 *                        "Affinity Scoring"; Algorithm 1 Step 1)
 *   moba_gate_topk       causal top-k block selection per query head plus the
 *                        query-per-block index                  ([summary] §3
 *                        "Top-k Gating", "Causality Enforcement"; Algorithm 1
 *                        Steps 1-2)
 *   moba_attn_fwd        softmax attention over the union of the selected
 *                        blocks, causal inside the current block, with the
 *                        online-softmax merge                   ([summary] §3
 *                        "The Core MoBA Attention Equation"; Algorithm 1
 *                        Steps 3-4)
 *
 * Conventions shared by every call
 *   - Tensors are dense and contiguous: q and out [batch, seqlen, hq, head_dim],
 *     k and v [batch, seqlen, hkv, head_dim].  q, k, v and out share the dtype
 *     (bf16 or fp32).  All pointers are DEVICE pointers on the current device,
 *     16-byte aligned.
 *   - The caller owns all memory.  The library never allocates or frees device
 *     memory, keeps no state between calls and never synchronises: every call
 *     only enqueues work on `stream` and returns.
 *   - Arguments are validated before anything is enqueued.  A bad argument
 *     returns MOBA_ERR_INVALID_ARG / MOBA_ERR_UNSUPPORTED / MOBA_ERR_WORKSPACE
 *     and launches nothing.  A launch failure returns MOBA_ERR_CUDA (the CUDA
 *     error code is available from moba_last_cuda_error()).  Errors that
 *     happen later on the device surface through the stream as usual.
 *   - topk counts the current block: each query attends to its own block
 *     (causally) plus the top (topk-1) earlier blocks by unscaled <q, mean K>.
 *     Equal scores go to the lower block index.  Future blocks are never
 *     selected.  With fewer than topk-1 earlier blocks, all are selected.
 *   - GQA: query head h uses kv head h / (hq / hkv); every query head selects
 *     its own blocks ([review] rebuttal W1 on the OpenReview discussion page).
 *   - seqlen need not be a multiple of block: the last block is shorter.
 *   - scale <= 0 selects 1/sqrt(head_dim).  lse is the natural-log
 *     log-sum-exp of the scaled logits.
 *   - Sizes: seqlen*hq*batch < 2^31, head_dim in {64, 128},
 *     1 <= topk <= MOBA_MAX_TOPK, and at most 65535 blocks and 65535 batch
 *     entries (MOBA_ERR_UNSUPPORTED beyond).
 */
#ifndef MOBA_H_
#define MOBA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define MOBA_API __attribute__((visibility("default")))
#else
#define MOBA_API
#endif

typedef struct CUstream_st* moba_stream_t; /* a cudaStream_t; NULL = legacy default stream */

#define MOBA_MAX_TOPK 16

typedef enum {
  MOBA_OK = 0,
  MOBA_ERR_INVALID_ARG = 1,  /* null pointer, misaligned pointer, bad shape   */
  MOBA_ERR_UNSUPPORTED = 2,  /* valid but not implemented (e.g. head_dim 96) */
  MOBA_ERR_WORKSPACE = 3,    /* workspace smaller than the *_workspace_size  */
  MOBA_ERR_CUDA = 4,         /* a CUDA runtime call or launch failed         */
  MOBA_ERR_INTERNAL = 5,
  MOBA_ERR_TIMEOUT = 6       /* a bounded device-side wait expired; written to a
                                device status word, never returned by a call    */
} moba_status_t;

typedef enum { MOBA_BF16 = 0, MOBA_F32 = 1 } moba_dtype_t;

typedef struct {
  int32_t batch;       /* independent sequences                                   */
  int32_t seqlen;      /* N: tokens per sequence                                  */
  int32_t hq;          /* query heads                                             */
  int32_t hkv;         /* key/value heads; hq % hkv == 0                          */
  int32_t head_dim;    /* d: 64 or 128                                            */
  int32_t block;       /* B: tokens per KV block                                  */
  int32_t topk;        /* blocks attended per query, counting the current block  */
  int32_t dtype;       /* moba_dtype_t of q, k, v and out                         */
  float scale;         /* softmax scale; <= 0 selects 1/sqrt(head_dim)           */
  int32_t query_chunk; /* tokens per attention pass; 0 = automatic (see below)   */
} moba_shape_t;

/* ---- sizes (host only, no CUDA calls) --------------------------------- */

/* MOBA_OK if the shape is supported, else the status moba_* calls return. */
MOBA_API moba_status_t moba_check_shape(const moba_shape_t* shape);

/* n = ceil(seqlen / block). */
MOBA_API int64_t moba_num_blocks(const moba_shape_t* shape);

/* Tokens per attention pass C.  The query range is processed in passes of C
 * tokens (for every batch entry at once) so that the per-block partial
 * results of one pass fit a bounded workspace.  query_chunk > 0 (a multiple
 * of 128) is used as given; 0 picks the largest power of two >= 128 whose
 * partials fit 8 GiB, capped at seqlen rounded up to 128 (a partial takes
 * 2 * head_dim + 4 bytes on the tensor-core path, bf16 with head_dim 128 or
 * 64, and 4 * (head_dim + 1) bytes for fp32; 65536 tokens at 1M, 524288 at
 * 10M). */
MOBA_API int64_t moba_query_chunk(const moba_shape_t* shape);

/* Number of passes: ceil(seqlen / C). */
MOBA_API int64_t moba_num_chunks(const moba_shape_t* shape);

/* Elements of meank: batch * n * hkv * head_dim (fp32). */
MOBA_API int64_t moba_meank_elems(const moba_shape_t* shape);

/* Elements of sel: batch * seqlen * hq * topk (int32). */
MOBA_API int64_t moba_sel_elems(const moba_shape_t* shape);

/* Elements of offsets: num_chunks * batch * hkv * n + 1 (int32). */
MOBA_API int64_t moba_offsets_elems(const moba_shape_t* shape);

/* Exact number of rows entries: batch * hq * sum_t min(topk-1, t / block). */
MOBA_API int64_t moba_rows_elems(const moba_shape_t* shape);

/* Device scratch bytes needed by moba_gate_topk / moba_attn_fwd. */
MOBA_API size_t moba_gate_workspace_size(const moba_shape_t* shape);
MOBA_API size_t moba_attn_workspace_size(const moba_shape_t* shape);

/* The scratch of one layer's gate and attention as one allocation:
 * moba_gate_workspace_size + moba_attn_workspace_size (both multiples of 256).
 * Pass ws to moba_gate_topk and ws + moba_gate_workspace_size(shape) to
 * moba_attn_fwd.  0 for an invalid shape. */
MOBA_API size_t moba_workspace_size(const moba_shape_t* shape);

/* Capacity the rows array needs: an upper bound of the entries any gate
 * writes for this shape, batch * hq * sum_t min(topk-1, t / block).  For the
 * plain gate it is the exact count (moba_rows_elems); for the pooled variant's
 * wide shape the gate fills offsets[last] <= capacity entries.  -1 for an
 * invalid shape. */
MOBA_API int64_t moba_rows_capacity(const moba_shape_t* shape);

/* ---- the three steps --------------------------------------------------- */

/* Block mean-pool ([summary] §3 "Affinity Scoring": the block representation
 * mean_pool(K[I_i]), computed once per layer; Algorithm 1 Step 1).
 *   k      [batch, seqlen, hkv, head_dim]  dtype     (read)
 *   meank  [batch, n, hkv, head_dim]       fp32      (written)
 * meank[b,j,g,:] is the mean of k[b, t, g, :] over the rows t of block j
 * (a shorter last block is averaged over its own rows). */
MOBA_API moba_status_t moba_block_meanpool(const moba_shape_t* shape, const void* k, float* meank,
                                           moba_stream_t stream);

/* Gate ([summary] §3 "Top-k Gating" g_i = 1[s_i in Topk], "Causality
 * Enforcement" mechanism 1, the current block as a shared expert; Algorithm 1
 * Step 1 S = Q meanK^T with the causal mask, and Step 2 grouping queries by
 * block).
 *   q        [batch, seqlen, hq, head_dim]  dtype   (read)
 *   meank    output of moba_block_meanpool          (read)
 *   sel      [batch, seqlen, hq, topk] int32        (written) selected blocks
 *            of each query head, ascending; the current block is the last
 *            valid entry; unused entries are -1.
 *   offsets  [moba_offsets_elems] int32             (written) exclusive
 *            prefix over groups (chunk, b, kv head g, block j) in that order:
 *            rows[offsets[i] .. offsets[i+1]) are the query rows of pass
 *            `chunk` that selected earlier block j and read kv head g.
 *   rows     [moba_rows_elems] int32                (written) query row ids
 *            r = (b * seqlen + t) * hq + h (the row of q viewed as
 *            [batch*seqlen*hq, head_dim]); within a group the order is
 *            unspecified.
 *   ws       >= moba_gate_workspace_size bytes of device scratch.  After the
 *            call completes on the stream, the int32 at byte offset
 *            moba_gate_workspace_size - 256 holds 0, or MOBA_ERR_TIMEOUT if a
 *            bounded device-side wait of the tensor-core scoring kernel expired
 *            (the results are then invalid). */
MOBA_API moba_status_t moba_gate_topk(const moba_shape_t* shape, const void* q, const float* meank,
                                      int32_t* sel, int32_t* offsets, int32_t* rows, void* ws,
                                      size_t ws_bytes, moba_stream_t stream);

/* Block-sparse attention ([summary] §3 "The Core MoBA Attention Equation"
 * MoBA(q,K,V) = Softmax(q K[I]^T) V[I]; "Causality Enforcement" mechanism 2,
 * causal inside the current block; Algorithm 1 Step 3 (history without mask,
 * grouped by block so each block's K/V serves all its queries) and Step 4
 * (online-softmax merge of the partial results)).
 *   q, k, v            as above                              (read)
 *   sel, offsets, rows outputs of moba_gate_topk             (read)
 *   out   [batch, seqlen, hq, head_dim] dtype                (written)
 *   lse   [batch, hq, seqlen] fp32, natural log, or NULL     (written)
 *   ws    >= moba_attn_workspace_size bytes of device scratch.  After the call
 *         completes on the stream, the first int32 of ws holds 0, or
 *         MOBA_ERR_TIMEOUT if a bounded device-side wait of a tensor-core
 *         kernel expired (out is then invalid).  Every wait in these kernels is
 *         bounded (2 s), so a fault in the pipeline cannot hang the GPU. */
MOBA_API moba_status_t moba_attn_fwd(const moba_shape_t* shape, const void* q, const void* k,
                                     const void* v, const int32_t* sel, const int32_t* offsets,
                                     const int32_t* rows, void* out, float* lse, void* ws,
                                     size_t ws_bytes, moba_stream_t stream);

/* ---- backward ---------------------------------------------------------- */

/* Device scratch bytes moba_attn_bwd needs for `shape`; 0 for an invalid shape. */
MOBA_API size_t moba_attn_bwd_workspace_size(const moba_shape_t* shape);

/* Gradients of the attention step ([summary] §3 "The Core MoBA Attention
 * Equation" differentiated with the gate's selection held fixed: a top-k of
 * scores is piecewise constant, so no gradient flows through the routing; the
 * pages print no backward formula).  For a row r with logits
 * z_u = scale <q_r, k_u> over its key set and the forward's lse L_r:
 *   p = exp(z - L_r), D_r = <dout_r, out_r>, ds = p (<dout_r, v_u> - D_r),
 *   dq_r = scale sum_u ds k_u, dk_u = scale sum_r ds q_r, dv_u = sum_r p dout_r
 * (query heads of a GQA group add into their kv head's dk, dv).
 *   q, k, v, sel, offsets, rows  as for moba_attn_fwd                (read)
 *   out   [batch, seqlen, hq, head_dim] dtype: the forward's output  (read)
 *   dout  [batch, seqlen, hq, head_dim] dtype: dL/d(out)             (read)
 *   lse   [batch, hq, seqlen] fp32: the forward's lse (natural log)  (read)
 *   dq    [batch, seqlen, hq, head_dim] dtype                        (written)
 *   dk, dv [batch, seqlen, hkv, head_dim] dtype                      (written)
 *   ws    >= moba_attn_bwd_workspace_size bytes of device scratch; its first
 *         int32 is a status word (0) like the forward's.
 * dk and dv are written once per key (for one gate index they are bitwise
 * reproducible; they sum over a group's rows in the order of `rows`).  bf16
 * with head_dim 128 runs on tensor cores and accumulates dq in fp32 with one
 * vector reduction per row and selected block, so its last fp32 bits may
 * depend on the order in which blocks arrive; the other layers write dq once. */
MOBA_API moba_status_t moba_attn_bwd(const moba_shape_t* shape, const void* q, const void* k,
                                     const void* v, const void* out, const void* dout, const float* lse,
                                     const int32_t* sel, const int32_t* offsets, const int32_t* rows,
                                     void* dq, void* dk, void* dv, void* ws, size_t ws_bytes,
                                     moba_stream_t stream);

/* ---- the whole layer from host buffers ---------------------------------- */

/* Device bytes moba_prefill_host needs for `shape` (with_lse: whether an lse
 * output will be requested); 0 for an invalid shape. */
MOBA_API size_t moba_prefill_host_workspace_size(const moba_shape_t* shape, int with_lse);

/* One MoBA prefill layer (Algorithm 1, Steps 1-4: mean-pool, gate, block-sparse
 * attention, merge; the same kernels and results as moba_block_meanpool +
 * moba_gate_topk + moba_attn_fwd) from and to HOST buffers, with the copies
 * overlapped with the computation.  The paper has no counterpart: this is the
 * library's host-side runtime around the three steps.
 *   q, k, v  host [batch, seqlen, hq|hkv, head_dim] dtype   (read)
 *   out      host [batch, seqlen, hq, head_dim] dtype       (written)
 *   lse      host [batch, hq, seqlen] fp32 natural log, or NULL (written)
 *   status   host int[2], or NULL: after the stream completes, the gate's and
 *            the attention's device status words (0, or MOBA_ERR_TIMEOUT)
 *   ws       >= moba_prefill_host_workspace_size(shape, lse != NULL) bytes of
 *            device memory, 16-byte aligned; it holds the device copies of the
 *            tensors and every intermediate array
 * q, k and v arrive one query pass (moba_query_chunk tokens) at a time on a
 * second stream (every step of a pass reads only tokens before the pass's
 * end); the mean-pool of the blocks a pass completes, its gate and its
 * attention start as soon as its rows are in, and each pass's output returns
 * on a third stream while the next pass computes.  The device copies of k and
 * v are cleared first.  The call only enqueues: `stream` (the compute stream)
 * completes when the last output byte is in host memory.  The copies overlap
 * only from page-locked host memory (cudaHostAlloc / cudaHostRegister);
 * pageable buffers give the same results with copies that block the calling
 * thread.  The call creates and releases two streams and 2 * passes + 2
 * events; it does no device allocation.  If a CUDA call fails after copies
 * were queued, it waits for them before returning MOBA_ERR_CUDA. */
MOBA_API moba_status_t moba_prefill_host(const moba_shape_t* shape, const void* q, const void* k,
                                         const void* v, void* out, float* lse, int* status,
                                         void* ws, size_t ws_bytes, moba_stream_t stream);

/* ---- gate variant: mean-, max- and min-pooled block keys ----------------- */

/* [review], the authors' rebuttals to W1 (block representation; the comparison
 * with QUEST): an ablation that, besides the blocks the mean-pooled gate
 * selects, also selects the top blocks under max pooling and under min pooling
 * of the keys.  The page gives no formula.  The reading implemented here: a
 * query at position t (current block c) attends
 *     the top (topk - 1) earlier blocks by <q, mean K_j>   (the plain gate)
 *   U the top `extra` earlier blocks by <q, max K_j>
 *   U the top `extra` earlier blocks by <q, min K_j>
 *   U {c},
 * max and min taken channel-wise over the block's key rows, each ranking over
 * the blocks j < c with equal scores going to the lower block index.  With
 * extra = 0 this is the plain gate.  A row attends between min(topk, c + 1)
 * and min(topk + 2 extra, c + 1) blocks.
 *
 * Buffers of the variant are sized by the WIDE shape: `shape` with topk
 * replaced by W = topk + 2 extra (moba_pooled_wide_shape).  For it
 * moba_sel_elems, moba_offsets_elems, moba_query_chunk, moba_num_chunks,
 * moba_gate_workspace_size and moba_attn_workspace_size give the variant's
 * sizes; moba_rows_elems gives an upper bound of its rows entries (the gate
 * writes offsets[last] of them). */

/* The wide shape of the variant: *wide = *shape with topk + 2 extra.  Returns
 * MOBA_ERR_INVALID_ARG for extra < 0 and MOBA_ERR_UNSUPPORTED when
 * topk + 2 extra > MOBA_MAX_TOPK; host only. */
MOBA_API moba_status_t moba_pooled_wide_shape(const moba_shape_t* shape, int32_t extra,
                                              moba_shape_t* wide);

/* Channel-wise max and min of every block's keys.
 *   k      [batch, seqlen, hkv, head_dim]  dtype     (read)
 *   maxk   [batch, n, hkv, head_dim]       fp32      (written)
 *   mink   [batch, n, hkv, head_dim]       fp32      (written)
 * Exact (no rounding): maxk/mink hold the inputs' own values. */
MOBA_API moba_status_t moba_block_maxminpool(const moba_shape_t* shape, const void* k, float* maxk,
                                             float* mink, moba_stream_t stream);

/* The variant's gate.  Scores are fp32 dot products of q with the three pooled
 * keys (bf16 with head_dim 128 and ceil((n - 1) / 32) <= W: tensor cores, one
 * pass per ranking, each exact up to fp32 accumulation; otherwise CUDA cores).
 *   q, meank        as for moba_gate_topk                              (read)
 *   maxk, mink      outputs of moba_block_maxminpool                   (read)
 *   sel      [batch, seqlen, hq, W] int32 (written): the chosen earlier blocks
 *            ascending, then the current block, then -1
 *   offsets, rows   as for moba_gate_topk, for the wide shape          (written)
 *   ws       >= moba_gate_workspace_size(wide) bytes of device scratch */
MOBA_API moba_status_t moba_gate_pooled(const moba_shape_t* shape, int32_t extra, const void* q,
                                        const float* meank, const float* maxk, const float* mink,
                                        int32_t* sel, int32_t* offsets, int32_t* rows, void* ws,
                                        size_t ws_bytes, moba_stream_t stream);

/* Attention over the variant's selections: the kernels of moba_attn_fwd for
 * the wide shape, plus one kernel per pass that marks the partial-result slots
 * of rows that chose fewer blocks as empty before the merge.
 *   arguments as for moba_attn_fwd; sel, offsets, rows from moba_gate_pooled
 *   ws   >= moba_attn_workspace_size(wide) bytes; first int32 = status word
 * The variant's backward is moba_attn_bwd called with the wide shape and this
 * gate's sel, offsets and rows: its kernels read variable-length selections
 * through them (rows entries up to offsets[last]). */
MOBA_API moba_status_t moba_attn_fwd_pooled(const moba_shape_t* shape, int32_t extra, const void* q,
                                            const void* k, const void* v, const int32_t* sel,
                                            const int32_t* offsets, const int32_t* rows, void* out,
                                            float* lse, void* ws, size_t ws_bytes,
                                            moba_stream_t stream);

/* ---- index validation ---------------------------------------------------- */

/* Checks the query-per-block index on the device before an attention or
 * backward call uses it (an index from another gate, or a changed gate; the
 * paper has no counterpart).  The attention kernels index K, V, partials and
 * outputs with these values unchecked.
 *   shape    as for the gate that wrote the index (the wide shape for the
 *            pooled variant)
 *   exact    nonzero: every sel row holds exactly min(topk, c + 1) blocks (the
 *            plain gate); 0: between 1 and min(topk, c + 1) (the pooled variant)
 *   sel, offsets   (read; rewritten only if a check fails)
 *   rows     moba_rows_capacity(shape) entries                   (read)
 *   status   device int32                                        (written)
 * Checks: each sel row strictly ascending in [0, c] with c (the query's block)
 * last, then -1; offsets[0] = 0, non-decreasing, offsets[last] <= the rows
 * capacity; every rows entry a row id of the shape whose batch entry, kv head
 * and pass are those of its group (pass, b, g, j), with j < its block and j in
 * its sel row.  Duplicate rows entries are not detected.  After the stream
 * completes, *status is 0, or MOBA_ERR_INTERNAL if a check failed; then the
 * index has been made inert (offsets all 0, every sel row {c, -1, ...}), so
 * a later moba_attn_fwd / moba_attn_bwd reads no invalid index (its outputs
 * are then not meaningful).  Nothing faults or traps. */
MOBA_API moba_status_t moba_check_index(const moba_shape_t* shape, int32_t exact, int32_t* sel,
                                        int32_t* offsets, const int32_t* rows, int* status,
                                        moba_stream_t stream);

/* ---- diagnostics ------------------------------------------------------- */

/* Static description of a status code. */
MOBA_API const char* moba_status_string(moba_status_t status);

/* The cudaError_t behind the last MOBA_ERR_CUDA returned on this thread. */
MOBA_API int moba_last_cuda_error(void);

/* Number of kernel launches the last moba_* call on this thread enqueued. */
MOBA_API int moba_last_launch_count(void);

/* Self-test of the failure path shared by the tensor-core kernels (the paper
 * has no counterpart): one kernel waits, with the same bounded wait, on an
 * mbarrier that nothing arrives at.  After about 2 s it gives up and writes
 * MOBA_ERR_TIMEOUT to *status (a device int32); the context stays usable.
 * Nothing faults, traps or hangs. */
MOBA_API moba_status_t moba_selftest_bounded_wait(int* status, moba_stream_t stream);

/* ---- gate without caller-provided scratch ----------------------------- */

/* Groups (offsets entries minus one) the allocation-free gate can index. */
#define MOBA_GATE_NOALLOC_MAX_GROUPS (1 << 19)

/* moba_gate_topk for callers that cannot hand the library any device scratch:
 * for example a plain C host program that has no device allocator of its own,
 * or a serving runtime that reserves all device memory when it starts and
 * forbids allocations afterwards.  The paper has no counterpart: this is a
 * packaging variant of the gate, not a step of the method.
 *
 * Same arguments, results and layouts as moba_gate_topk, minus ws/ws_bytes.
 * The scratch (two int32 counters per group) lives in a fixed array inside
 * the library: 2 * MOBA_GATE_NOALLOC_MAX_GROUPS + 64 int32 (4 MiB), held on every
 * GPU that loads the library until the process exits.  Shapes with more than
 * MOBA_GATE_NOALLOC_MAX_GROUPS groups (moba_offsets_elems - 1) are rejected
 * with MOBA_ERR_UNSUPPORTED before anything is enqueued.
 *   - Nothing is allocated: no cudaMalloc/cudaFree and no allocating library
 *     routine.  The counters are cleared on `stream` at the start of every call.
 *   - The first call on each device looks up that device's address of the
 *     array (with the device current); make that first call before any stream
 *     capture on the device.
 *   - All calls on a device share the one array: calls that overlap on the GPU
 *     (different streams without ordering between them) race and give wrong
 *     results.  Order them on one stream or with events.
 *   - The device status word (0, or MOBA_ERR_TIMEOUT when a bounded wait of the
 *     tensor-core scoring kernel gave up and sel/offsets/rows are not valid) is
 *     in the same array, at a fixed place; moba_gate_noalloc_status reads it. */
MOBA_API moba_status_t moba_gate_topk_noalloc(const moba_shape_t* shape, const void* q,
                                              const float* meank, int32_t* sel, int32_t* offsets,
                                              int32_t* rows, moba_stream_t stream);

/* Status word of the last moba_gate_topk_noalloc call on the current device:
 * enqueues on `stream` a copy of the word into *status, HOST memory (pinned or
 * pageable; with pageable memory the copy completes before this call returns).
 * Read *status after `stream` has synchronised.  The word is cleared at the
 * start of every moba_gate_topk_noalloc call, so order this call after the gate
 * call it reports on (the same stream does that).  Allocates nothing.
 * Returns MOBA_ERR_INVALID_ARG for a null pointer, MOBA_ERR_CUDA if the copy
 * cannot be enqueued. */
MOBA_API moba_status_t moba_gate_noalloc_status(int* status, moba_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* MOBA_H_ */
