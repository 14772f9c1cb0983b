// asp_api.cu -- the C ABI of libasp: host-side validation, dispatch to the
// kernels, the two-stream decode step and small utilities.  Nothing here
// allocates memory; every error is reported as an asp_status.
#include <chrono>
#include <cmath>
#include <map>
#include <mutex>
#include <thread>
#include <tuple>

#include "asp_common.cuh"
#include "asp_internal.h"

namespace asp {

int sm_count() {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (cache[dev] <= 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && n > 0) cache[dev] = n;
  }
  return cache[dev] > 0 ? cache[dev] : 148;
}

int prepare_kernel(const void* kern, size_t smem, int threads) {
  // The dynamic shared-memory limit is one attribute per kernel: keep it at the
  // largest size requested so far, so that every cached configuration stays valid.
  static std::mutex mu;
  static std::map<std::pair<const void*, int>, size_t> limit;
  static std::map<std::tuple<const void*, int, size_t, int>, int> occupancy;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  std::lock_guard<std::mutex> lock(mu);
  size_t& cur = limit[std::make_pair(kern, dev)];
  if (smem > cur) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess) {
      (void)cudaGetLastError();
      return 0;
    }
    cur = smem;
  }
  const auto key = std::make_tuple(kern, dev, smem, threads);
  auto it = occupancy.find(key);
  if (it != occupancy.end()) return it->second;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, smem) != cudaSuccess) {
    (void)cudaGetLastError();
    return 0;
  }
  occupancy[key] = per_sm;
  return per_sm;
}

}  // namespace asp

namespace {

using asp::KvView;

constexpr int kMaxGridY = 65535;
constexpr int kMaxScoreBatch = 8192;   // the key scan keeps per-sequence offsets in shared memory

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool group_ok(int n_q_heads, int n_kv) {
  if (n_kv <= 0 || n_q_heads <= 0 || n_q_heads % n_kv) return false;
  const int g = n_q_heads / n_kv;
  return g == 1 || g == 2 || g == 4 || g == 8;
}

// Validates a KV description; need_v: the call reads v too.
asp_status check_kv(const asp_kv* kv, bool need_v) {
  if (!kv) return ASP_ERR_INVALID_ARG;
  if (kv->batch <= 0 || kv->n_kv_heads <= 0 || kv->t_max <= 0) return ASP_ERR_INVALID_ARG;
  if (kv->kv_dtype != ASP_F32 && kv->kv_dtype != ASP_BF16) return ASP_ERR_INVALID_ARG;
  if (kv->head_dim != 64 && kv->head_dim != 128) return ASP_ERR_UNSUPPORTED;
  if (!kv->k || (need_v && !kv->v)) return ASP_ERR_INVALID_ARG;
  if (!aligned16(kv->k) || (need_v && !aligned16(kv->v))) return ASP_ERR_INVALID_ARG;
  if ((long)kv->batch * kv->n_kv_heads > kMaxGridY) return ASP_ERR_UNSUPPORTED;
  if (kv->page_size < 0) return ASP_ERR_INVALID_ARG;
  if (kv->page_size > 0) {
    if (kv->page_size % 16 || kv->page_size > 256) return ASP_ERR_UNSUPPORTED;
    if (!kv->page_table || !kv->seq_lens || kv->max_pages <= 0 || kv->n_pages <= 0) return ASP_ERR_INVALID_ARG;
    if ((long)kv->max_pages * kv->page_size < kv->t_max) return ASP_ERR_INVALID_ARG;
  }
  return ASP_OK;
}

KvView view_of(const asp_kv* kv) {
  KvView v;
  v.k = kv->k;
  v.v = kv->v;
  v.kv_f32 = kv->kv_dtype == ASP_F32;
  v.batch = kv->batch;
  v.n_kv = kv->n_kv_heads;
  v.head_dim = kv->head_dim;
  v.t_max = kv->t_max;
  v.page_size = kv->page_size;
  v.max_pages = kv->page_size ? kv->max_pages : 0;
  v.n_pages = kv->page_size ? kv->n_pages : 0;
  v.page_table = kv->page_size ? kv->page_table : nullptr;
  v.seq_lens = kv->seq_lens;
  return v;
}

asp_status check_pred(const asp_pred_cfg* cfg, int ring_start) {
  if (!cfg) return ASP_ERR_INVALID_ARG;
  if (cfg->W < 1) return ASP_ERR_INVALID_ARG;
  if (cfg->W > 32) return ASP_ERR_UNSUPPORTED;
  if (!cfg->windows || cfg->n_windows < 1 || cfg->n_windows > 8) return ASP_ERR_INVALID_ARG;
  for (int i = 0; i < cfg->n_windows; ++i)
    if (cfg->windows[i] < 1 || cfg->windows[i] > cfg->W) return ASP_ERR_INVALID_ARG;
  if (!(cfg->lambda > 0.0f) || !std::isfinite(cfg->lambda)) return ASP_ERR_INVALID_ARG;
  if (cfg->coef != ASP_COEF_SOFTMAX && cfg->coef != ASP_COEF_RAW) return ASP_ERR_INVALID_ARG;
  if (cfg->pool != ASP_POOL_PREDICTIONS && cfg->pool != ASP_POOL_FEATURES) return ASP_ERR_INVALID_ARG;
  if (ring_start < 0 || ring_start > cfg->W) return ASP_ERR_INVALID_ARG;
  return ASP_OK;
}

asp_status cuda_status(cudaError_t e) { return e == cudaSuccess ? ASP_OK : ASP_ERR_CUDA; }

// asp_decode_step's workspace: the attention's split-K partials, then (256-byte
// aligned) the key-score histogram [batch * n_kv, 2048] int32 of the selection.
// The decode step's attention runs beside the selection chain: one CTA per SM
// leaves room for the key scan's CTA on every SM.
constexpr int kDecodeAttendCtasPerSm = 1;

size_t decode_hist_offset(int batch, int n_q_heads, int n_kv_heads, int head_dim, int C, int max_tail) {
  const size_t att =
      asp::attend_plan(batch, n_q_heads, n_kv_heads, head_dim, C, max_tail, kDecodeAttendCtasPerSm).workspace_bytes;
  return ((att + 255) / 256) * 256;
}

asp::PredictArgs predict_args(float* qhist, int ring_start, const void* q_new, asp_dtype q_new_dtype, int batch,
                              int n_q_heads, int head_dim, const asp_pred_cfg* cfg, float* qpred) {
  asp::PredictArgs a;
  a.zero = nullptr;
  a.zero_words = 0;
  a.qhist = qhist;
  a.ring_start = ring_start;
  a.q_new = q_new;
  a.q_new_f32 = q_new_dtype == ASP_F32;
  a.n_heads = batch * n_q_heads;
  a.W = cfg->W;
  a.head_dim = head_dim;
  a.n_win = cfg->n_windows;
  a.wmax = 0;
  for (int i = 0; i < 8; ++i) a.windows[i] = 0;
  for (int i = 0; i < cfg->n_windows; ++i) {
    a.windows[i] = cfg->windows[i];
    if (cfg->windows[i] > a.wmax) a.wmax = cfg->windows[i];
  }
  a.lam = (double)cfg->lambda;
  a.coef_raw = cfg->coef == ASP_COEF_RAW;
  a.pool_features = cfg->pool == ASP_POOL_FEATURES;
  a.qpred = qpred;
  a.mode = 0;
  a.factor_in = nullptr;
  a.factor_out = nullptr;
  return a;
}

asp_status check_attend(const void* q, asp_dtype q_dtype, int n_q_heads, const asp_kv* kv, const int32_t* idx,
                        const int32_t* count, int C, const int32_t* tail_begin, int max_tail, void* out,
                        void* workspace, size_t workspace_bytes, asp::AttendPlan* plan, int ctas_per_sm = 0) {
  asp_status st = check_kv(kv, true);
  if (st != ASP_OK) return st;
  if (!q || !out) return ASP_ERR_INVALID_ARG;
  if (q_dtype != ASP_F32 && q_dtype != ASP_BF16) return ASP_ERR_INVALID_ARG;
  if (n_q_heads <= 0 || n_q_heads % kv->n_kv_heads) return ASP_ERR_INVALID_ARG;
  if (!group_ok(n_q_heads, kv->n_kv_heads)) return ASP_ERR_UNSUPPORTED;
  if (C < 0 || (C > 0 && (!idx || !count))) return ASP_ERR_INVALID_ARG;
  const int mt = tail_begin ? max_tail : 0;
  if (mt < 0 || (long)C + mt < 1) return ASP_ERR_INVALID_ARG;
  if ((long)C + mt > (1L << 30)) return ASP_ERR_UNSUPPORTED;
  *plan = asp::attend_plan(kv->batch, n_q_heads, kv->n_kv_heads, kv->head_dim, C, mt, ctas_per_sm);
  if (plan->workspace_bytes) {
    if (!workspace || workspace_bytes < plan->workspace_bytes) return ASP_ERR_WORKSPACE;
    if (!aligned16(workspace)) return ASP_ERR_WORKSPACE;
  }
  return ASP_OK;
}

asp_status check_append(const asp_kv* kv, const void* k_new, const void* v_new, const void* meta, int quest_page) {
  asp_status st = check_kv(kv, true);
  if (st != ASP_OK) return st;
  if (!k_new || !v_new || !kv->seq_lens) return ASP_ERR_INVALID_ARG;
  if (!aligned16(k_new) || !aligned16(v_new)) return ASP_ERR_INVALID_ARG;
  if (meta) {
    if (quest_page <= 0 || !aligned16(meta)) return ASP_ERR_INVALID_ARG;
    if (quest_page % 16 || quest_page > 256) return ASP_ERR_UNSUPPORTED;
    if (kv->page_size && kv->page_size != quest_page) return ASP_ERR_UNSUPPORTED;
  }
  return ASP_OK;
}

}  // namespace

extern "C" {

int asp_abi_version(void) { return ASP_ABI_VERSION; }

const char* asp_status_string(asp_status s) {
  switch (s) {
    case ASP_OK: return "ok";
    case ASP_ERR_INVALID_ARG: return "invalid argument";
    case ASP_ERR_UNSUPPORTED: return "unsupported configuration";
    case ASP_ERR_WORKSPACE: return "workspace missing or too small";
    case ASP_ERR_CUDA: return "CUDA error";
    case ASP_ERR_TIMEOUT: return "timed out";
    case ASP_ERR_DEVICE: return "device-side fault recorded";
  }
  return "unknown status";
}

asp_status asp_predict_query(float* qhist, int ring_start, const void* q_new, asp_dtype q_new_dtype, int batch,
                             int n_q_heads, int head_dim, const asp_pred_cfg* cfg, float* qpred,
                             asp_stream_t stream) {
  if (!qhist || !qpred || batch <= 0 || n_q_heads <= 0) return ASP_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return ASP_ERR_UNSUPPORTED;
  if (q_new && q_new_dtype != ASP_F32 && q_new_dtype != ASP_BF16) return ASP_ERR_INVALID_ARG;
  if ((long)batch * n_q_heads > (1L << 28)) return ASP_ERR_UNSUPPORTED;
  asp_status st = check_pred(cfg, ring_start);
  if (st != ASP_OK) return st;
  const asp::PredictArgs a = predict_args(qhist, ring_start, q_new, q_new_dtype, batch, n_q_heads, head_dim, cfg, qpred);
  return cuda_status(asp::launch_predict(a, reinterpret_cast<cudaStream_t>(stream)));
}

asp_status asp_score_keys(const float* qpred, int n_q_heads, const asp_kv* kv, float* scores, asp_stream_t stream) {
  asp_status st = check_kv(kv, false);
  if (st != ASP_OK) return st;
  if (!qpred || !scores) return ASP_ERR_INVALID_ARG;
  if (n_q_heads <= 0 || n_q_heads % kv->n_kv_heads) return ASP_ERR_INVALID_ARG;
  if (!group_ok(n_q_heads, kv->n_kv_heads)) return ASP_ERR_UNSUPPORTED;
  if (kv->batch > kMaxScoreBatch) return ASP_ERR_UNSUPPORTED;
  return cuda_status(asp::launch_score(qpred, n_q_heads, view_of(kv), scores, reinterpret_cast<cudaStream_t>(stream)));
}

asp_status asp_score_keys_cuda_cores(const float* qpred, int n_q_heads, const asp_kv* kv, float* scores,
                                     asp_stream_t stream) {
  asp_status st = check_kv(kv, false);
  if (st != ASP_OK) return st;
  if (!qpred || !scores) return ASP_ERR_INVALID_ARG;
  if (n_q_heads <= 0 || n_q_heads % kv->n_kv_heads) return ASP_ERR_INVALID_ARG;
  if (!group_ok(n_q_heads, kv->n_kv_heads)) return ASP_ERR_UNSUPPORTED;
  if (kv->batch > kMaxScoreBatch) return ASP_ERR_UNSUPPORTED;
  return cuda_status(asp::launch_score_cuda_cores(qpred, n_q_heads, view_of(kv), scores,
                                                  reinterpret_cast<cudaStream_t>(stream)));
}

asp_status asp_select_topk(const float* scores, const int32_t* seq_lens, int batch, int n_kv_heads, int t_max, int C,
                           int32_t* idx, int32_t* count, asp_stream_t stream) {
  if (!scores || !idx || !count || batch <= 0 || n_kv_heads <= 0 || t_max <= 0 || C <= 0) return ASP_ERR_INVALID_ARG;
  if ((long)batch * n_kv_heads > kMaxGridY || !asp::select_supported(t_max, 1)) return ASP_ERR_UNSUPPORTED;
  asp::SelectArgs a;
  a.scores = scores;
  a.row_stride = t_max;
  a.seq_lens = seq_lens;
  a.t_max = t_max;
  a.rows_per_seq = n_kv_heads;
  a.n_rows = batch * n_kv_heads;
  a.c_units = C;
  a.expand = 1;
  a.idx = idx;
  a.count = count;
  a.hist0 = nullptr;
  return cuda_status(asp::launch_select(a, reinterpret_cast<cudaStream_t>(stream)));
}

size_t asp_decode_workspace_bytes(int batch, int n_q_heads, int n_kv_heads, int head_dim, int C, int max_tail) {
  if (batch <= 0 || n_q_heads <= 0 || n_kv_heads <= 0 || C < 1 || max_tail < 0) return 0;
  if (head_dim != 64 && head_dim != 128) return 0;
  return decode_hist_offset(batch, n_q_heads, n_kv_heads, head_dim, C, max_tail) +
         (size_t)batch * n_kv_heads * asp::kTopBins * 4;
}

size_t asp_pred_factor_bytes(int batch, int n_q_heads, const asp_pred_cfg* cfg) {
  if (batch <= 0 || n_q_heads <= 0 || check_pred(cfg, 0) != ASP_OK) return 0;
  int wmax = 0;
  for (int i = 0; i < cfg->n_windows; ++i) wmax = cfg->windows[i] > wmax ? cfg->windows[i] : wmax;
  return asp::predict_factor_bytes(batch * n_q_heads, wmax);
}

size_t asp_attend_workspace_bytes(int batch, int n_q_heads, int n_kv_heads, int head_dim, int C, int max_tail) {
  if (batch <= 0 || n_q_heads <= 0 || n_kv_heads <= 0 || C < 0 || max_tail < 0 || (long)C + max_tail < 1) return 0;
  if (head_dim != 64 && head_dim != 128) return 0;
  return asp::attend_plan(batch, n_q_heads, n_kv_heads, head_dim, C, max_tail).workspace_bytes;
}

asp_status asp_sparse_attend(const void* q, asp_dtype q_dtype, int n_q_heads, const asp_kv* kv, const int32_t* idx,
                             const int32_t* count, int C, const int32_t* tail_begin, int max_tail, void* out,
                             float* lse, void* workspace, size_t workspace_bytes, asp_stream_t stream) {
  asp::AttendPlan plan;
  asp_status st = check_attend(q, q_dtype, n_q_heads, kv, idx, count, C, tail_begin, max_tail, out, workspace,
                               workspace_bytes, &plan);
  if (st != ASP_OK) return st;
  return cuda_status(asp::launch_attend(q, q_dtype == ASP_F32, n_q_heads, view_of(kv), idx, count, C, tail_begin,
                                        max_tail, out, lse, workspace, plan, reinterpret_cast<cudaStream_t>(stream)));
}

asp_status asp_sparse_attend_noalloc(const void* q, asp_dtype q_dtype, int n_q_heads, const asp_kv* kv,
                                     const int32_t* idx, const int32_t* count, int C, const int32_t* tail_begin,
                                     int max_tail, void* out, float* lse, asp_stream_t stream) {
  // Same validation as asp_sparse_attend; the workspace check is satisfied with a
  // stand-in (never used: the partials go to the library's fixed scratch), and the
  // plan's workspace size is then checked against that scratch.
  asp::AttendPlan plan;
  void* const stand_in = reinterpret_cast<void*>(static_cast<uintptr_t>(256));
  asp_status st = check_attend(q, q_dtype, n_q_heads, kv, idx, count, C, tail_begin, max_tail, out, stand_in,
                               ~static_cast<size_t>(0), &plan);
  if (st != ASP_OK) return st;
  if (plan.workspace_bytes > ASP_NOALLOC_SCRATCH_BYTES) return ASP_ERR_WORKSPACE;
  return cuda_status(asp::launch_attend_noalloc(q, q_dtype == ASP_F32, n_q_heads, view_of(kv), idx, count, C,
                                                tail_begin, max_tail, out, lse, plan,
                                                reinterpret_cast<cudaStream_t>(stream)));
}

asp_status asp_decode_step(const asp_decode_args* a) {
  if (!a) return ASP_ERR_INVALID_ARG;
  asp::AttendPlan plan;
  asp_status st = check_attend(a->q_t, a->q_dtype, a->n_q_heads, a->kv, a->idx_cur, a->count_cur, a->C, a->tail_begin,
                               a->max_tail, a->out, a->workspace, a->workspace_bytes, &plan, kDecodeAttendCtasPerSm);
  if (st != ASP_OK) return st;
  if (a->C < 1 || !a->qhist || !a->qpred || !a->scores || !a->idx_next || !a->count_next) return ASP_ERR_INVALID_ARG;
  const int mt = a->tail_begin ? a->max_tail : 0;
  const size_t hist_off = decode_hist_offset(a->kv->batch, a->n_q_heads, a->kv->n_kv_heads, a->kv->head_dim, a->C, mt);
  const size_t hist_words = (size_t)a->kv->batch * a->kv->n_kv_heads * asp::kTopBins;
  if (!a->workspace || a->workspace_bytes < hist_off + hist_words * 4 ||
      (reinterpret_cast<uintptr_t>(a->workspace) & 255))
    return ASP_ERR_WORKSPACE;
  int32_t* hist = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(a->workspace) + hist_off);
  if (!a->ev_fork || !a->ev_sel_done) return ASP_ERR_INVALID_ARG;
  st = check_pred(a->pred, a->ring_start);
  if (st != ASP_OK) return st;
  if (!asp::select_supported(a->kv->t_max, 1) || a->kv->batch > kMaxScoreBatch) return ASP_ERR_UNSUPPORTED;
  if ((a->pred_factor_cur && (reinterpret_cast<uintptr_t>(a->pred_factor_cur) & 7)) ||
      (a->pred_factor_next && (reinterpret_cast<uintptr_t>(a->pred_factor_next) & 7)) ||
      (a->pred_factor_cur && a->pred_factor_cur == a->pred_factor_next))
    return ASP_ERR_INVALID_ARG;
  if (a->k_new) {   // the step appends the new token first: it writes seq_lens and tail_begin
    st = check_append(a->kv, a->k_new, a->v_new, a->quest_meta, a->quest_page);
    if (st != ASP_OK) return st;
    if (!a->tail_begin || a->max_tail < 1) return ASP_ERR_INVALID_ARG;
  }

  cudaStream_t sm = reinterpret_cast<cudaStream_t>(a->s_main);
  cudaStream_t ss = reinterpret_cast<cudaStream_t>(a->s_side);
  // The lag factorisation moves to the previous step when it can run beside the
  // selection without taking SMs from it: the selection's CTAs (one per row) and
  // the factorisation's (four heads each) fit on the GPU at once.  A pure function
  // of the sizes, so consecutive steps agree on it.
  bool use_factor = false;
  {
    asp::PredictArgs probe = predict_args(a->qhist, a->ring_start, a->q_t, a->q_dtype, a->kv->batch, a->n_q_heads,
                                          a->kv->head_dim, a->pred, a->qpred);
    const long rows = (long)a->kv->batch * a->kv->n_kv_heads;
    const long fctas = ((long)a->kv->batch * a->n_q_heads + 3) / 4;
    use_factor = asp::predict_factor_eligible(probe) && rows + fctas <= asp::sm_count();
  }
  cudaEvent_t fork = reinterpret_cast<cudaEvent_t>(a->ev_fork);
  cudaEvent_t done = reinterpret_cast<cudaEvent_t>(a->ev_sel_done);
  auto mark = [&](int i, cudaStream_t s) -> cudaError_t {
    return a->timing ? cudaEventRecord(reinterpret_cast<cudaEvent_t>(a->timing[i]), s) : cudaSuccess;
  };
  const KvView kv = view_of(a->kv);
  const int B = a->kv->batch;

  // idx_cur is the previous step's selection.  While s_main is being captured into
  // a graph the wait is left out: launches of the captured graph on one stream are
  // ordered, and each graph ends with both streams joined.
  cudaStreamCaptureStatus capture = cudaStreamCaptureStatusNone;
  cudaError_t e = cudaStreamIsCapturing(sm, &capture);
  if (e == cudaSuccess && capture == cudaStreamCaptureStatusNone) e = cudaStreamWaitEvent(sm, done, 0);
  if (e == cudaSuccess && a->k_new)   // before the fork: both streams see the new token
    e = asp::launch_append(kv, a->k_new, a->v_new, const_cast<int32_t*>(a->kv->seq_lens),
                           const_cast<int32_t*>(a->tail_begin), a->quest_meta, a->quest_page, sm);
  if (e == cudaSuccess) e = cudaEventRecord(fork, sm);
  // main stream: attention of this step, issued first so that its CTAs (one per
  // SM) are placed before the side chain's, in a captured graph as in a stream
  if (e == cudaSuccess) e = mark(6, sm);
  if (e == cudaSuccess)
    e = asp::launch_attend(a->q_t, a->q_dtype == ASP_F32, a->n_q_heads, kv, a->idx_cur, a->count_cur, a->C,
                           a->tail_begin, a->max_tail, a->out, a->lse, a->workspace, plan, sm);
  if (e == cudaSuccess) e = mark(7, sm);
  // out and lse are complete here: a caller may read them back from this point on
  if (e == cudaSuccess && a->ev_attend_done)
    e = cudaEventRecord(reinterpret_cast<cudaEvent_t>(a->ev_attend_done), sm);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(ss, fork, 0);
  // side stream: selection for the next step
  if (e == cudaSuccess) e = mark(0, ss);
  if (e == cudaSuccess) {
    asp::PredictArgs pa = predict_args(a->qhist, a->ring_start, a->q_t, a->q_dtype, B, a->n_q_heads,
                                       a->kv->head_dim, a->pred, a->qpred);
    pa.zero = hist;   // the score kernel accumulates the selection's first histogram here
    pa.zero_words = hist_words;
    if (use_factor && a->pred_factor_cur && a->pred_factor_valid) {
      pa.mode = 2;
      pa.factor_in = a->pred_factor_cur;
    }
    e = asp::launch_predict(pa, ss);
  }
  if (e == cudaSuccess) e = mark(1, ss);
  if (e == cudaSuccess) e = mark(2, ss);
  // the predictor is the scan's only producer in this stream: the scan may start
  // streaming keys while it runs
  if (e == cudaSuccess) e = asp::launch_score(a->qpred, a->n_q_heads, kv, a->scores, ss, hist, true);
  // main stream, once the scan is done: the next step's lag factorisation, on the SMs
  // the selection leaves free (it reads q_t and ring slots this step's push leaves
  // alone); ev_fork is reused to carry the scan's completion
  if (e == cudaSuccess && use_factor && a->pred_factor_next) {
    e = cudaEventRecord(fork, ss);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(sm, fork, 0);
    asp::PredictArgs fa = predict_args(a->qhist, a->ring_start, a->q_t, a->q_dtype, B, a->n_q_heads,
                                       a->kv->head_dim, a->pred, a->qpred);
    fa.mode = 1;
    fa.factor_out = a->pred_factor_next;
    if (e == cudaSuccess) e = asp::launch_predict(fa, sm);
  }
  if (e == cudaSuccess) e = mark(3, ss);
  if (e == cudaSuccess) e = mark(4, ss);
  if (e == cudaSuccess) {
    asp::SelectArgs sa;
    sa.scores = a->scores;
    sa.row_stride = a->kv->t_max;
    sa.seq_lens = a->kv->seq_lens;
    sa.t_max = a->kv->t_max;
    sa.rows_per_seq = a->kv->n_kv_heads;
    sa.n_rows = B * a->kv->n_kv_heads;
    sa.c_units = a->C;
    sa.expand = 1;
    sa.idx = a->idx_next;
    sa.count = a->count_next;
    sa.hist0 = hist;
    e = asp::launch_select(sa, ss);
  }
  if (e == cudaSuccess) e = mark(5, ss);
  if (e == cudaSuccess) e = cudaEventRecord(done, ss);
  return cuda_status(e);
}

asp_status asp_graph_instantiate(void* graph, void** exec_out) {
  if (!graph || !exec_out) return ASP_ERR_INVALID_ARG;
  cudaGraphExec_t ex = nullptr;
  const cudaError_t e = cudaGraphInstantiateWithFlags(&ex, static_cast<cudaGraph_t>(graph),
                                                      cudaGraphInstantiateFlagUseNodePriority);
  if (e != cudaSuccess) return ASP_ERR_CUDA;
  *exec_out = ex;
  return ASP_OK;
}

asp_status asp_graph_launch(void* exec, asp_stream_t stream) {
  if (!exec) return ASP_ERR_INVALID_ARG;
  return cuda_status(cudaGraphLaunch(static_cast<cudaGraphExec_t>(exec), reinterpret_cast<cudaStream_t>(stream)));
}

asp_status asp_graph_destroy(void* exec) {
  if (!exec) return ASP_ERR_INVALID_ARG;
  return cuda_status(cudaGraphExecDestroy(static_cast<cudaGraphExec_t>(exec)));
}

asp_status asp_wait_selection(asp_event_t ev_sel_done, long timeout_us) {
  if (!ev_sel_done || timeout_us < 0) return ASP_ERR_INVALID_ARG;
  const auto t0 = std::chrono::steady_clock::now();
  for (;;) {
    const cudaError_t e = cudaEventQuery(reinterpret_cast<cudaEvent_t>(ev_sel_done));
    if (e == cudaSuccess) return ASP_OK;
    if (e != cudaErrorNotReady) return ASP_ERR_CUDA;
    const long waited = (long)std::chrono::duration_cast<std::chrono::microseconds>(
                            std::chrono::steady_clock::now() - t0).count();
    if (waited >= timeout_us) return ASP_ERR_TIMEOUT;
    std::this_thread::sleep_for(std::chrono::microseconds(20));
  }
}

asp_status asp_append_kv(const asp_kv* kv, const void* k_new, const void* v_new, int32_t* tail_begin_out,
                         void* quest_meta, int quest_page, asp_stream_t stream) {
  asp_status st = check_append(kv, k_new, v_new, quest_meta, quest_page);
  if (st != ASP_OK) return st;
  return cuda_status(asp::launch_append(view_of(kv), k_new, v_new, const_cast<int32_t*>(kv->seq_lens), tail_begin_out,
                                        quest_meta, quest_page, reinterpret_cast<cudaStream_t>(stream)));
}

asp_status asp_quest_build_meta(const asp_kv* kv, int quest_page, void* meta, asp_stream_t stream) {
  asp_status st = check_kv(kv, false);
  if (st != ASP_OK) return st;
  if (!meta || quest_page <= 0) return ASP_ERR_INVALID_ARG;
  if (quest_page % 16 || quest_page > 256) return ASP_ERR_UNSUPPORTED;
  if (kv->page_size && kv->page_size != quest_page) return ASP_ERR_UNSUPPORTED;
  return cuda_status(asp::launch_quest_meta(view_of(kv), quest_page, meta, reinterpret_cast<cudaStream_t>(stream)));
}

namespace {
asp_status check_quest(const void* q, asp_dtype q_dtype, int n_q_heads, const asp_kv* kv, const void* meta,
                       int quest_page, float* page_scores) {
  asp_status st = check_kv(kv, false);
  if (st != ASP_OK) return st;
  if (!q || !meta || !page_scores || quest_page <= 0) return ASP_ERR_INVALID_ARG;
  if (q_dtype != ASP_F32 && q_dtype != ASP_BF16) return ASP_ERR_INVALID_ARG;
  if (n_q_heads <= 0 || n_q_heads % kv->n_kv_heads) return ASP_ERR_INVALID_ARG;
  if (!group_ok(n_q_heads, kv->n_kv_heads)) return ASP_ERR_UNSUPPORTED;
  if (quest_page % 16 || quest_page > 256) return ASP_ERR_UNSUPPORTED;
  if (kv->page_size && kv->page_size != quest_page) return ASP_ERR_UNSUPPORTED;
  return ASP_OK;
}
}  // namespace

asp_status asp_quest_page_scores(const void* q, asp_dtype q_dtype, int n_q_heads, const asp_kv* kv, const void* meta,
                                 int quest_page, float* page_scores, asp_stream_t stream) {
  asp_status st = check_quest(q, q_dtype, n_q_heads, kv, meta, quest_page, page_scores);
  if (st != ASP_OK) return st;
  return cuda_status(asp::launch_quest_score(q, q_dtype == ASP_F32, n_q_heads, view_of(kv), meta, quest_page,
                                             page_scores, reinterpret_cast<cudaStream_t>(stream)));
}

asp_status asp_quest_select(const void* q, asp_dtype q_dtype, int n_q_heads, const asp_kv* kv, const void* meta,
                            int quest_page, int C, float* page_scores, int32_t* idx, int32_t* count,
                            asp_stream_t stream) {
  asp_status st = check_quest(q, q_dtype, n_q_heads, kv, meta, quest_page, page_scores);
  if (st != ASP_OK) return st;
  if (!idx || !count || C <= 0) return ASP_ERR_INVALID_ARG;
  if (!asp::select_supported(kv->t_max, quest_page)) return ASP_ERR_UNSUPPORTED;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = asp::launch_quest_score(q, q_dtype == ASP_F32, n_q_heads, view_of(kv), meta, quest_page,
                                          page_scores, s);
  if (e != cudaSuccess) return ASP_ERR_CUDA;
  asp::SelectArgs sa;
  sa.scores = page_scores;
  sa.row_stride = (kv->t_max + quest_page - 1) / quest_page;
  sa.seq_lens = kv->seq_lens;
  sa.t_max = kv->t_max;
  sa.rows_per_seq = kv->n_kv_heads;
  sa.n_rows = kv->batch * kv->n_kv_heads;
  sa.c_units = (C + quest_page - 1) / quest_page;
  sa.expand = quest_page;
  sa.idx = idx;
  sa.count = count;
  sa.hist0 = nullptr;
  return cuda_status(asp::launch_select(sa, s));
}

asp_status asp_check_wait_limit(int tries, int32_t* returned, asp_stream_t stream) {
  if (!returned || tries < 1 || tries > (1 << 20)) return ASP_ERR_INVALID_ARG;
  return cuda_status(asp::launch_wait_limit_check(tries, returned, reinterpret_cast<cudaStream_t>(stream)));
}

asp_status asp_device_status(asp_stream_t stream, int32_t* bits_out) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int v = 0;
  cudaError_t e = cudaStreamSynchronize(s);
  if (e == cudaSuccess) e = asp::read_status_predict(s, &v);
  if (e == cudaSuccess) e = asp::read_status_score(s, &v);
  if (e == cudaSuccess) e = asp::read_status_select(s, &v);
  if (e == cudaSuccess) e = asp::read_status_attend(s, &v);
  if (e == cudaSuccess) e = asp::read_status_quest(s, &v);
  if (e == cudaSuccess) e = asp::read_status_score_tc(s, &v);
  if (e == cudaSuccess) e = asp::read_status_append(s, &v);
  if (bits_out) *bits_out = v;
  if (e != cudaSuccess) return ASP_ERR_CUDA;
  return v ? ASP_ERR_DEVICE : ASP_OK;
}

}  // extern "C"
