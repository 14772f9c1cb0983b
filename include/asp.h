/*
 * asp.h -- C ABI of libasp: predicted-query token-level sparse decode attention
 * for NVIDIA B200 (sm_100a).
 *
 * The method (AsyncSpade, "Efficient Test-Time Scaling with Asynchronous Sparse
 * Decoding") removes KV selection from the decoding loop's critical path: while
 * step t attends over the tokens chosen for it, the selection for step t+1 is
 * made from a *predicted* query (abstract, components (1) and (2); research-map
 * summary, "Approach").  The pages print no API; these calls follow that problem
 * statement:
 *
 *   asp_predict_query   step 1: next query from the last W queries (ridge + softmax
 *                       coefficients + multi-window average pooling)
 *   asp_score_keys      step 2: every cached key of a KV head scored with its
 *                       group's predicted queries
 *   asp_select_topk     step 3: the C best tokens per (sequence, KV head)
 *   asp_sparse_attend   step 4: single-token attention over the selected K/V only,
 *                       with the true current query
 *   asp_decode_step     steps 1-4 for one decode step: attention of step t on one
 *                       stream, the selection for step t+1 on a side stream
 *   asp_quest_*         the page-level comparison path (min/max page metadata)
 *
 * Conventions for every call:
 *   - Pointers named as device memory must be device memory of the current CUDA
 *     device; they stay owned by the caller.  The library never allocates device
 *     or host memory for these calls and keeps no host-side state between calls.
 *   - Work is enqueued asynchronously on the stream(s) given; a call returns once
 *     the work is enqueued.  Stream and event handles are plain CUDA runtime
 *     handles (cudaStream_t / cudaEvent_t); NULL stream means the legacy default
 *     stream.
 *   - Arguments are validated on the host before anything is enqueued.  On an
 *     invalid argument the call returns a status other than ASP_OK and enqueues
 *     nothing.  A failed launch returns ASP_ERR_CUDA.  No C++ exception crosses
 *     this boundary.
 *   - Device-side checks never trap: an out-of-range token index or page id is
 *     skipped, a bounded wait that runs out stops its warp, and either event sets
 *     the library's device status word, read with asp_device_status().
 *   - Layouts are row-major; "[a, b, c]" lists dimensions outermost first.
 *   - GQA: query head hq belongs to KV head hq / G, G = n_q_heads / n_kv_heads.
 */
#ifndef ASP_H_
#define ASP_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define ASP_ABI_VERSION 5

#if defined(__GNUC__)
#define ASP_API __attribute__((visibility("default")))
#else
#define ASP_API
#endif

/* ABI-compatible with cudaStream_t / cudaEvent_t. */
typedef struct CUstream_st* asp_stream_t;
typedef struct CUevent_st* asp_event_t;

typedef enum {
  ASP_OK = 0,
  ASP_ERR_INVALID_ARG = 1,  /* null pointer, bad size or inconsistent shapes */
  ASP_ERR_UNSUPPORTED = 2,  /* valid but not built: head_dim, group size, dtype combination */
  ASP_ERR_WORKSPACE = 3,    /* workspace missing or smaller than the matching *_workspace_bytes() */
  ASP_ERR_CUDA = 4,         /* a CUDA runtime call or launch failed */
  ASP_ERR_TIMEOUT = 5,      /* asp_wait_selection: the event did not complete in time */
  ASP_ERR_DEVICE = 6        /* asp_device_status: a kernel recorded a device-side fault */
} asp_status;

typedef enum { ASP_F32 = 0, ASP_BF16 = 1 } asp_dtype;

/* How the ridge coefficients of one window become weights (softmax is the
 * method's softmax normalisation; RAW keeps the coefficients). */
typedef enum { ASP_COEF_SOFTMAX = 0, ASP_COEF_RAW = 1 } asp_coef_mode;

/* What "multi-window average pooling" averages.  PREDICTIONS (the reading the
 * library follows by default): one ridge fit per window on that window's lagged
 * queries, the windows' predictions averaged.  FEATURES (the recorded
 * alternative): each window w pools the history into one feature, the mean of the
 * w most recent vectors; one ridge fit on the windows' features one step back
 * gives a weight per window (normalised as `coef` says), applied to the current
 * features. */
typedef enum { ASP_POOL_PREDICTIONS = 0, ASP_POOL_FEATURES = 1 } asp_pool_mode;

/* Device status word bits (asp_device_status). */
#define ASP_DEV_BAD_INDEX  0x1   /* a selected index outside [0, T_b) was skipped */
#define ASP_DEV_BAD_PAGE   0x2   /* a page-table entry outside [0, n_pages) was skipped */
#define ASP_DEV_WAIT_LIMIT 0x4   /* a bounded shared-memory barrier wait ran out */
#define ASP_DEV_TAIL_LIMIT 0x8   /* a tail longer than max_tail was truncated */
#define ASP_DEV_SELECT     0x10  /* a selection output position past C was skipped (a first-digit
                                    histogram that does not match the scores) */
#define ASP_DEV_NAN_SCORE  0x20  /* the selection read a NaN score: invalid input, the chosen set
                                    is then unspecified (it never holds more than C tokens) */

/* The KV cache of one layer.
 *   page_size == 0: k, v are [batch, n_kv_heads, t_max, head_dim] (contiguous).
 *   page_size  > 0: k, v are [n_pages, n_kv_heads, page_size, head_dim]; token j of
 *                   sequence b lives in page page_table[b * max_pages + j / page_size]
 *                   at row j % page_size.  page_size must be a multiple of 16, at most 256.
 * seq_lens[b] = T_b, the number of valid tokens of sequence b (device int32 [batch],
 * 0 <= T_b <= t_max; larger values are clamped to t_max).  NULL means T_b = t_max.
 * Paged caches require seq_lens and page_table (device int32 [batch, max_pages]),
 * t_max <= max_pages * page_size.  k, v must be 16-byte aligned. */
typedef struct {
  int batch;
  int n_kv_heads;
  int head_dim;          /* 64 or 128 */
  int t_max;             /* token capacity of a sequence; row stride of score buffers */
  asp_dtype kv_dtype;    /* ASP_F32 or ASP_BF16 */
  const void* k;
  const void* v;
  int page_size;
  const int32_t* page_table;
  int max_pages;
  int n_pages;           /* physical pages in the pool (paged only) */
  const int32_t* seq_lens;
} asp_kv;

/* Predictor configuration (host memory). */
typedef struct {
  int W;                 /* lags; the history holds W + 1 vectors, 1 <= W <= 32 */
  const int* windows;    /* pooling windows, each in [1, W], 1 to 8 of them */
  int n_windows;
  float lambda;          /* ridge parameter, > 0, added to the Gram diagonal unscaled */
  asp_coef_mode coef;
  asp_pool_mode pool;    /* ASP_POOL_PREDICTIONS unless comparing the readings */
} asp_pred_cfg;

/* ---------------------------------------------------------------------------
 * Step 1 -- predicted query.
 * Source: abstract, component (1) (a light-weight temporal-regressive module
 * predicts the next query from a short window of recent queries); research-map
 * summary, "Approach" (softmax-normalized ridge regression with multi-window
 * average pooling); reproduction card, claim C5 (one-step-ahead fit, 16-query
 * window).  For each query head and each window w: ridge-fit q_t on the lags
 * q_{t-w}..q_{t-1} over the head_dim channels, a = (X X^T + lambda I)^-1 X q_t,
 * turn a into weights (softmax or raw), apply weight i to q_{t-w+i}; average
 * the window predictions.  The Gram matrix and right-hand side are formed in fp32,
 * the Cholesky factorisation and both substitutions run in fp64, the softmax of
 * the coefficients in fp32.
 *
 * qhist : device fp32 ring [batch, n_q_heads, W+1, head_dim].  Slot
 *         (ring_start + s) % (W+1) holds the s-th oldest vector (s = 0..W).
 * q_new : NULL, or device [batch, n_q_heads, head_dim] of q_new_dtype.  When given,
 *         the oldest slot (ring_start) is first overwritten with q_new (as fp32),
 *         so the window becomes slots ring_start+1 .. ring_start+W+1; the caller
 *         then advances its ring_start by one.  Without it qhist is only read.
 * qpred : device fp32 [batch, n_q_heads, head_dim], written.
 * Errors: ASP_ERR_INVALID_ARG (null pointers, sizes <= 0, windows outside [1, W],
 * lambda <= 0, ring_start outside [0, W]); ASP_ERR_UNSUPPORTED (head_dim not 64/128,
 * W > 32). */
ASP_API asp_status asp_predict_query(float* qhist, int ring_start, const void* q_new, asp_dtype q_new_dtype,
                             int batch, int n_q_heads, int head_dim, const asp_pred_cfg* cfg,
                             float* qpred, asp_stream_t stream);

/* ---------------------------------------------------------------------------
 * Step 2 -- score every cached key.
 * Source: abstract (query-aware, token-level KV selection replacing page
 * filtering); research-map summary, "Key results" (Qwen3 GQA models).
 * scores[b, h, j] = max over the G query heads g of KV head h of
 *                   (qpred[b, h*G + g, :] . k[b, h, j, :]) / sqrt(head_dim),  j < T_b.
 * Entries j >= T_b of a row are not written.  fp32 arithmetic.
 * qpred  : device fp32 [batch, n_q_heads, head_dim].
 * scores : device fp32 [batch, n_kv_heads, t_max], written.
 * Errors: ASP_ERR_INVALID_ARG; ASP_ERR_UNSUPPORTED (G not in {1,2,4,8}, head_dim
 * not 64/128, batch > 8192). */
ASP_API asp_status asp_score_keys(const float* qpred, int n_q_heads, const asp_kv* kv, float* scores,
                          asp_stream_t stream);

/* Step 2 on the CUDA cores whatever the key type: the scan asp_score_keys runs for
 * fp32 keys and page sizes other than 16, and for bf16 keys the comparison of its
 * tensor-core scan (same arguments, errors and results within the score tolerance;
 * the tensor-core path replaced it for bf16 keys because it reaches the copy
 * bandwidth where this one is bound by instruction issue). */
ASP_API asp_status asp_score_keys_cuda_cores(const float* qpred, int n_q_heads, const asp_kv* kv, float* scores,
                                             asp_stream_t stream);

/* ---------------------------------------------------------------------------
 * Step 3 -- top-C token selection.
 * Source: research-map summary, "Key results" (2k selected tokens); reproduction
 * card, "Key finding" (C = 2k tokens).  Per row (b, h): the C largest of
 * scores[b, h, 0:T_b] under IEEE order (-0.0 == +0.0; +-inf allowed; NaN is not
 * allowed), ties at the threshold going to the lowest token index.  The chosen
 * indices are written in ascending order; count = min(C, T_b); entries past count
 * are -1.
 * scores   : device fp32 [batch, n_kv_heads, t_max] (only j < T_b is read).
 * seq_lens : device int32 [batch] or NULL (T_b = t_max).
 * idx      : device int32 [batch, n_kv_heads, C], written.
 * count    : device int32 [batch, n_kv_heads], written.
 * Errors: ASP_ERR_INVALID_ARG; ASP_ERR_UNSUPPORTED (batch * n_kv_heads > 65535). */
ASP_API asp_status asp_select_topk(const float* scores, const int32_t* seq_lens, int batch, int n_kv_heads,
                           int t_max, int C, int32_t* idx, int32_t* count, asp_stream_t stream);

/* ---------------------------------------------------------------------------
 * Step 4 -- single-token attention over the selected tokens.
 * Source: abstract (attention over the selected KV; selection decoupled from the
 * decoding loop); reproduction card, "Key finding" (both methods attend to the
 * same 2k tokens).  For query head hq of KV head h, with S = {idx[b,h,0:count]} u
 * [tail_begin[b], T_b):
 *   out[b, hq] = sum_{j in S} softmax_j(q[b,hq] . k_j / sqrt(d)) v_j,
 *   lse[b, hq] = ln sum_{j in S} exp(q[b,hq] . k_j / sqrt(d)).
 * The query is the true current query.  Selected indices >= tail_begin[b] are
 * covered by the tail and skipped; indices outside [0, T_b) are skipped and flagged.
 * An empty S gives out = 0 and lse = -inf.  Split-K over S with a log-sum-exp merge;
 * fp32 accumulation.
 * q          : device [batch, n_q_heads, head_dim] of q_dtype (bf16 or fp32).
 * idx, count : as written by asp_select_topk (idx row stride C); the first count
 *              entries of a row must be distinct.  May be NULL when C == 0.
 * tail_begin : device int32 [batch] or NULL (no tail); max_tail bounds T_b - tail_begin
 *              (longer tails are truncated and flagged).  max_tail = t_max with
 *              tail_begin = 0 and count = 0 gives dense attention.
 * out        : device [batch, n_q_heads, head_dim] in kv_dtype, written.
 * lse        : device fp32 [batch, n_q_heads] or NULL.
 * workspace  : device scratch of at least asp_attend_workspace_bytes(...) bytes,
 *              16-byte aligned; contents need no initialisation.  May be NULL when
 *              asp_attend_workspace_bytes(...) is 0.
 * Errors: ASP_ERR_INVALID_ARG; ASP_ERR_UNSUPPORTED; ASP_ERR_WORKSPACE. */
ASP_API asp_status asp_sparse_attend(const void* q, asp_dtype q_dtype, int n_q_heads, const asp_kv* kv,
                             const int32_t* idx, const int32_t* count, int C,
                             const int32_t* tail_begin, int max_tail,
                             void* out, float* lse, void* workspace, size_t workspace_bytes,
                             asp_stream_t stream);

/* Bytes of workspace asp_sparse_attend needs for these sizes (a pure function of
 * its arguments; 0 for invalid sizes). */
ASP_API size_t asp_attend_workspace_bytes(int batch, int n_q_heads, int n_kv_heads, int head_dim, int C,
                                  int max_tail);

/* Bytes of workspace asp_decode_step needs (attention partials plus the
 * selection's first-digit histogram, which the key scan builds); a pure function
 * of its arguments, 0 for invalid sizes. */
ASP_API size_t asp_decode_workspace_bytes(int batch, int n_q_heads, int n_kv_heads, int head_dim, int C,
                                          int max_tail);

/* Bytes of one predictor-factor buffer of asp_decode_step (pred_factor_cur / _next):
 * per query head the scaled rows of the lag Gram's Cholesky factor and its inverse
 * diagonal, fp64.  0 for invalid arguments. */
ASP_API size_t asp_pred_factor_bytes(int batch, int n_q_heads, const asp_pred_cfg* cfg);

/* ---------------------------------------------------------------------------
 * Step 4 without a caller-provided workspace.  No counterpart in the paper: this
 * entry point exists for callers that cannot allocate device memory -- for example
 * a plug-in inside an engine that owns all device memory and hands the plug-in only
 * the tensors of the call, or a latency-critical decode loop that must not call
 * cudaMalloc (it can synchronise the device).  It computes exactly what
 * asp_sparse_attend computes, with the same arguments minus the workspace.
 * The split-K partials live in one fixed array inside the library, of
 * ASP_NOALLOC_SCRATCH_BYTES bytes (2 MiB), that every GPU which loads the library
 * holds until the process exits.  Sizes whose partials would not fit (compare
 * asp_attend_workspace_bytes) return ASP_ERR_WORKSPACE and enqueue nothing; with
 * the current split plan the partials stay below 1.9 MB for every valid size.
 * The first call on a device looks up the array's device address on that device
 * (the device must be current); make that first call before any stream capture.
 * All calls share the one array and it keeps the last call's contents; nothing in
 * it has to start at zero (every partial the merge reads is written earlier in the
 * same call).  Calls whose kernels overlap on the GPU (different streams without
 * ordering between them) race on the array and give wrong results. */
#define ASP_NOALLOC_SCRATCH_BYTES ((size_t)2 << 20)
ASP_API asp_status asp_sparse_attend_noalloc(const void* q, asp_dtype q_dtype, int n_q_heads, const asp_kv* kv,
                                             const int32_t* idx, const int32_t* count, int C,
                                             const int32_t* tail_begin, int max_tail, void* out, float* lse,
                                             asp_stream_t stream);

/* ---------------------------------------------------------------------------
 * The new token's K and V appended to the cache (the cache management that
 * surrounds the steps; reproduction card, "Key finding", and abstract,
 * component (2): the cache side keeps the KV cache current while decoding).
 * k_new, v_new : device [batch, n_kv_heads, head_dim] in kv_dtype, 16-byte aligned.
 * For every sequence b the token goes to position T = seq_lens[b] (contiguous:
 * row T of [b, h]; paged: row T % page_size of page page_table[b][T / page_size],
 * which the caller has allocated), then tail_begin_out[b] = T (when not NULL: the
 * start of the tail that the next attention covers in full) and seq_lens[b] = T + 1.
 * kv->seq_lens is read and written on the device and must not be NULL.
 * quest_meta : NULL, or page bounds as in asp_quest_build_meta (pages of
 *              quest_page tokens) that are kept current: a token that opens a page
 *              sets the page's bounds, later tokens widen them.
 * A sequence at capacity (T == t_max, or past its pages) or whose page is not
 * valid is left unchanged and ASP_DEV_BAD_PAGE is recorded (asp_device_status).
 * Asynchronous on `stream`. */
ASP_API asp_status asp_append_kv(const asp_kv* kv, const void* k_new, const void* v_new, int32_t* tail_begin_out,
                                 void* quest_meta, int quest_page, asp_stream_t stream);

/* ---------------------------------------------------------------------------
 * One asynchronous decode step (steps 1-4).
 * Source: abstract, component (2) (KV selection decoupled from the decoding loop
 * and overlapped with the forward computation).  On one GPU the two ranks of the
 * pages become two streams:
 *   s_main : waits for ev_sel_done (the previous step's selection, i.e. idx_cur),
 *            then attends q_t over idx_cur/count_cur (+ tail) -> out, lse.
 *   s_side : waits for ev_fork (recorded on s_main at entry), pushes q_t into the
 *            ring, predicts qpred, scores every key, selects idx_next/count_next,
 *            then records ev_sel_done.
 * The side chain is the step's critical path: s_side should be a stream of higher
 * priority than s_main, so that its kernels get SMs before the attention's.
 * The caller swaps idx_cur/idx_next (and count_*) between steps, advances
 * ring_start by one, and must not reuse q_t, qpred, scores or idx_next before
 * ev_sel_done completes.  While s_main is being captured (CUDA graphs) the step
 * leaves out its wait for ev_sel_done: the caller then orders the graph launches on
 * one stream, and ends each capture with s_main waiting for ev_sel_done, so that
 * the graph joins both streams.  workspace: at least asp_decode_workspace_bytes(...)
 * bytes, 256-byte aligned, no initialisation needed (ASP_ERR_WORKSPACE otherwise).  timing: NULL, or 8 events recorded around the kernels
 * (begin/end of predict, score, select on s_side; attend on s_main) for profiling. */
typedef struct {
  const void* q_t;              /* device [batch, n_q_heads, head_dim] */
  asp_dtype q_dtype;
  int n_q_heads;
  float* qhist;                 /* ring, see asp_predict_query */
  int ring_start;
  const asp_pred_cfg* pred;
  const asp_kv* kv;
  int C;
  const int32_t* idx_cur;       /* [batch, n_kv_heads, C] */
  const int32_t* count_cur;     /* [batch, n_kv_heads] */
  const int32_t* tail_begin;    /* [batch] or NULL */
  int max_tail;
  float* qpred;                 /* [batch, n_q_heads, head_dim] scratch */
  float* scores;                /* [batch, n_kv_heads, t_max] scratch */
  int32_t* idx_next;            /* [batch, n_kv_heads, C] */
  int32_t* count_next;          /* [batch, n_kv_heads] */
  void* out;                    /* [batch, n_q_heads, head_dim] kv dtype */
  float* lse;                   /* [batch, n_q_heads] or NULL */
  void* workspace;
  size_t workspace_bytes;
  asp_stream_t s_main;
  asp_stream_t s_side;
  asp_event_t ev_fork;
  asp_event_t ev_sel_done;
  asp_event_t* timing;          /* NULL or asp_event_t[8] */
  /* Optional: the step first appends the new token (asp_append_kv) on s_main, so
   * that this step's attention, scan and selection all see it.  With k_new set,
   * kv->seq_lens is advanced on the device and tail_begin (which must then be set,
   * with max_tail >= 1) is overwritten with the lengths before the append. */
  const void* k_new;            /* [batch, n_kv_heads, head_dim] kv dtype, or NULL */
  const void* v_new;
  void* quest_meta;             /* NULL, or page bounds kept current (see asp_append_kv) */
  int quest_page;
  /* Optional: the predictor's lag factorisation moved off the critical path.  The
   * lag Gram that step t+1 solves holds q_t and the W - 1 queries before it, all
   * known at step t, so step t factorises it into pred_factor_next on s_main once
   * its key scan is done (ev_fork is then recorded again on s_side after the scan),
   * beside the selection, and step t+1's predictor only forms the right-hand side
   * and substitutes.  Both buffers hold asp_pred_factor_bytes(...) bytes (8-byte
   * aligned, distinct); the caller swaps them between steps like idx_cur/idx_next
   * and sets pred_factor_valid = 1 once pred_factor_cur holds the factor the
   * previous decode step wrote for this ring (0 on a first step or after the ring
   * was changed otherwise: the step then factorises in full).  NULL pointers turn
   * the precomputation off.  It is also off (every step factorises in full, the
   * buffers untouched) when the selection's CTAs (batch * n_kv_heads) and the
   * factorisation's (one per 4 query heads) do not fit on the GPU's SMs together,
   * for windows that are not powers of two filling at most 32 lags, and for the
   * pooled-features reading. */
  double* pred_factor_cur;
  int pred_factor_valid;
  double* pred_factor_next;
  /* Optional: recorded on s_main as soon as this step's out and lse are written
   * (before the main stream's later work of the step, such as the factorisation),
   * so that a caller can copy the output back while the selection still runs.
   * NULL: not recorded. */
  asp_event_t ev_attend_done;
} asp_decode_args;

ASP_API asp_status asp_decode_step(const asp_decode_args* args);

/* CUDA graphs of decode steps (no counterpart in the pages: launch plumbing).
 * graph: a cudaGraph_t captured from asp_decode_step calls (see above).  The graph
 * is instantiated so that each kernel keeps the priority of the stream it was
 * captured from: the selection chain then stays ahead of the attention, as in
 * eager steps (a plain instantiation runs every node at the launch stream's
 * priority).  The caller keeps the graph alive while it uses the instantiation,
 * and frees the instantiation with asp_graph_destroy. */
ASP_API asp_status asp_graph_instantiate(void* graph, void** exec_out);
ASP_API asp_status asp_graph_launch(void* exec, asp_stream_t stream);
ASP_API asp_status asp_graph_destroy(void* exec);

/* Host wait for a selection with a time limit (polls the event; never blocks past
 * timeout_us).  Returns ASP_OK, ASP_ERR_TIMEOUT or ASP_ERR_CUDA. */
ASP_API asp_status asp_wait_selection(asp_event_t ev_sel_done, long timeout_us);

/* ---------------------------------------------------------------------------
 * Page-level comparison path (Quest-style).
 * Source: abstract and research-map summary, "Problem" (query-aware page-level
 * filtering that waits for the current query); reproduction card, "Key finding"
 * (its page-scan term 2 q h T/P).  Pages of quest_page tokens (a multiple of 16;
 * for a paged cache it must equal kv->page_size).
 * meta : device [batch, n_kv_heads, ceil(t_max / quest_page), 2, head_dim] in kv_dtype:
 *        per page and channel the minimum (index 0) and maximum (index 1) key value
 *        over the page's valid tokens. */
ASP_API asp_status asp_quest_build_meta(const asp_kv* kv, int quest_page, void* meta, asp_stream_t stream);

/* The page scores alone (the first half of asp_quest_select): page_scores
 * [batch, n_kv_heads, ceil(t_max / quest_page)] fp32 get u_p (defined below) for
 * every page holding a valid token; entries past a sequence's pages are not
 * written.  Same arguments and errors as asp_quest_select, less the selection's. */
ASP_API asp_status asp_quest_page_scores(const void* q, asp_dtype q_dtype, int n_q_heads, const asp_kv* kv,
                                         const void* meta, int quest_page, float* page_scores,
                                         asp_stream_t stream);

/* Page score u_p = max over the group's query heads of
 * sum_c max(q_c kmin_c, q_c kmax_c) / sqrt(d) with the current query q; the
 * ceil(C / quest_page) best pages (lowest page index on ties) are kept and their
 * valid tokens written ascending to idx [batch, n_kv_heads, ceil(C/quest_page)*quest_page]
 * (-1 padded), count [batch, n_kv_heads].
 * page_scores : device fp32 scratch [batch, n_kv_heads, ceil(t_max / quest_page)]. */
ASP_API asp_status asp_quest_select(const void* q, asp_dtype q_dtype, int n_q_heads, const asp_kv* kv,
                            const void* meta, int quest_page, int C, float* page_scores,
                            int32_t* idx, int32_t* count, asp_stream_t stream);

/* ---------------------------------------------------------------------------
 * Utilities. */

/* Check of the device-side failure detection (no counterpart in the pages).  One
 * warp waits on a shared-memory barrier that nothing arrives on, with the bounded
 * wait every kernel of the library uses cut to `tries` attempts (each at most about
 * 1 us); it gives up, records ASP_DEV_WAIT_LIMIT (read it with asp_device_status)
 * and writes 1 to *returned (device int32) before it exits -- 2 would mean the wait
 * succeeded.  No fault, trap or hang is involved.  Errors: ASP_ERR_INVALID_ARG
 * (returned NULL, tries outside [1, 2^20]). */
ASP_API asp_status asp_check_wait_limit(int tries, int32_t* returned, asp_stream_t stream);

/* Reads and clears the device status word (ASP_DEV_* bits) after synchronising
 * `stream`.  Returns ASP_ERR_DEVICE when a bit was set, else ASP_OK/ASP_ERR_CUDA. */
ASP_API asp_status asp_device_status(asp_stream_t stream, int32_t* bits_out);

ASP_API const char* asp_status_string(asp_status status);
ASP_API int asp_abi_version(void);

#ifdef __cplusplus
}
#endif
#endif /* ASP_H_ */
