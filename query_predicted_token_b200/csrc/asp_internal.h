// asp_internal.h -- launchers shared between the libasp translation units.
// Each launcher assumes its arguments were validated by the C ABI layer
// (asp_api.cu) and returns the CUDA error of its launch.
#pragma once

#include <cstddef>
#include <cstdint>
#include <utility>
#include <cuda_runtime.h>

#include "asp.h"

namespace asp {

// Number of SMs of the current device (cached per device).
int sm_count();

// One-time launch setup per (kernel, device, dynamic shared memory): raises the
// kernel's dynamic shared-memory limit and returns its resident CTAs per SM
// (0 if the configuration cannot launch).  Cached, so launches stay cheap.
int prepare_kernel(const void* kern, size_t smem, int threads);

// Launches `kern` with programmatic stream serialisation: it may begin while the
// previous kernel on `s` finishes (the kernel orders its reads with pdl_wait()).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  // the stream's priority travels with the launch, so that a graph captured from
  // the stream keeps it per kernel
  int prio = 0;
  if (cudaStreamGetPriority(s, &prio) != cudaSuccess) prio = 0;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributePriority;
  attr[1].val.priority = prio;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// launch_pdl with thread-block clusters of `cluster_x` CTAs along x (grid.x a
// multiple of it).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl_cluster(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                               int cluster_x, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  int prio = 0;
  if (cudaStreamGetPriority(s, &prio) != cudaSuccess) prio = 0;
  cudaLaunchAttribute attr[3];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributePriority;
  attr[1].val.priority = prio;
  attr[2].id = cudaLaunchAttributeClusterDimension;
  attr[2].val.clusterDim.x = (unsigned)cluster_x;
  attr[2].val.clusterDim.y = 1;
  attr[2].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 3;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// A plain launch (no early start) that carries the stream's priority like launch_pdl.
template <typename... KArgs, typename... Args>
cudaError_t launch_prio(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  int prio = 0;
  if (cudaStreamGetPriority(s, &prio) != cudaSuccess) prio = 0;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributePriority;
  attr[0].val.priority = prio;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// Per-file device status readers (OR into *bits, then clear).
cudaError_t read_status_predict(cudaStream_t s, int* bits);
cudaError_t read_status_score(cudaStream_t s, int* bits);
cudaError_t read_status_select(cudaStream_t s, int* bits);
cudaError_t read_status_attend(cudaStream_t s, int* bits);
cudaError_t read_status_quest(cudaStream_t s, int* bits);
cudaError_t read_status_score_tc(cudaStream_t s, int* bits);
cudaError_t read_status_append(cudaStream_t s, int* bits);

// ---- step 1 -----------------------------------------------------------------
struct PredictArgs {
  int32_t* zero;          // optional buffer the kernel clears first (next step's key histogram)
  size_t zero_words;
  float* qhist;
  int ring_start;
  const void* q_new;      // may be null
  int q_new_f32;          // 1: fp32, 0: bf16
  int n_heads;            // batch * n_q_heads
  int W;
  int head_dim;
  int n_win;
  int windows[8];
  int wmax;
  double lam;
  int coef_raw;
  int pool_features;      // 1: regress on the windows' pooled features (the recorded alternative reading)
  float* qpred;
  int win_fast;           // set by launch_predict: windows sorted, powers of two, one round of lanes
  // decode loop: 0 factorise and predict; 1 only factorise the next step's lag Gram
  // into factor_out; 2 predict with factor_in (stored by the previous step's mode 1)
  int mode;
  const double* factor_in;
  double* factor_out;
};
cudaError_t launch_predict(const PredictArgs& a, cudaStream_t s);
// Whether the factor modes apply to these windows (powers of two in one round of
// lanes, not the pooled-features reading); otherwise mode 2 predicts in full and
// mode 1 launches nothing.
bool predict_factor_eligible(const PredictArgs& a);
size_t predict_factor_bytes(int n_heads, int wmax);

// ---- step 2 -----------------------------------------------------------------
struct KvView {
  const void* k;
  const void* v;
  int kv_f32;             // 1: fp32, 0: bf16
  int batch, n_kv, head_dim, t_max;
  int page_size, max_pages, n_pages;
  const int32_t* page_table;
  const int32_t* seq_lens;   // may be null (all t_max)
};
// The new token's K and V [batch, n_kv, head_dim] at position seq_lens[b]; then
// tail_begin[b] (optional) = the old length and seq_lens[b] += 1.  meta: optional
// page bounds [batch, n_kv, ceil(t_max / quest_page), 2, head_dim] kept current.
cudaError_t launch_append(const KvView& kv, const void* k_new, const void* v_new, int32_t* seq_lens,
                          int32_t* tail_begin, void* meta, int quest_page, cudaStream_t s);

// hist: optional [batch * n_kv, 2048] int32 counts of the scores' top 11 key bits
// (must be zero on entry); the selection then skips its own first pass.
// early: the previous kernel of the stream writes only qpred (and clears hist), and
// every other input was written before it started; the tensor-core scan then
// starts streaming keys before that kernel has finished.
cudaError_t launch_score(const float* qpred, int n_q_heads, const KvView& kv, float* scores, cudaStream_t s,
                         int32_t* hist = nullptr, bool early = false);

// The key scan on the CUDA cores whatever the key type (the path of fp32 keys and
// other page sizes; for bf16 keys the comparison of the tensor-core scan).
cudaError_t launch_score_cuda_cores(const float* qpred, int n_q_heads, const KvView& kv, float* scores,
                                    cudaStream_t s, int32_t* hist = nullptr);

// Tensor-core key scan (bf16 keys, head_dim 64/128, contiguous or 16-token pages,
// G in {1,2,4,8}, 16-byte aligned qpred); launch_score uses it when supported.
bool quest_tc_supported(const KvView& kv, int n_q_heads, const void* q);
cudaError_t launch_quest_score_tc(const void* q, int q_f32, int n_q_heads, const KvView& kv, const void* meta,
                                  int quest_page, float* page_scores, cudaStream_t s);
bool score_tc_supported(const KvView& kv, int n_q_heads, const float* qpred);
cudaError_t launch_score_tc(const float* qpred, int n_q_heads, const KvView& kv, float* scores, cudaStream_t s,
                            int32_t* hist, bool early = false);

// ---- step 3 -----------------------------------------------------------------
// Selects `c_units` units per row out of ceil(T_b / expand) scores (row stride
// `row_stride`) and writes each chosen unit u as the tokens u*expand + i (i <
// expand, tokens >= T_b written as -1), ascending; out row stride c_units*expand.
struct SelectArgs {
  const float* scores;
  int row_stride;
  const int32_t* seq_lens;  // may be null
  int t_max;
  int rows_per_seq;          // n_kv_heads
  int n_rows;                // batch * n_kv_heads
  int c_units;
  int expand;
  int32_t* idx;
  int32_t* count;
  const int32_t* hist0;      // optional first-pass histogram [n_rows, 2048] (expand == 1 only)
  int key_cap;               // set by launch_select: shared-memory slots per row (keys, or packed lists)
};
cudaError_t launch_select(const SelectArgs& a, cudaStream_t s);
bool select_supported(int t_max, int expand);

// ---- step 4 -----------------------------------------------------------------
struct AttendPlan {
  int splits;
  int rows_per_split;
  size_t workspace_bytes;
  int ctas;   // CTAs of the (persistent) tensor-core attention grid
  int lean;   // 1: the kernel form with fewer registers (one CTA per SM beside the key scan)
  int gather;           // 1: bf16 cache and query go through attend_gather_kernel
  int tiles_per_unit;   // gather: 16-row tiles planned per (sequence, KV head) unit
  int gather_ctas;      // gather: CTAs (at most one per SM)
};
// ctas_per_sm: resident CTAs per SM the grid is sized for (0: as many as fit).
AttendPlan attend_plan(int batch, int n_q_heads, int n_kv_heads, int head_dim, int C, int max_tail,
                       int ctas_per_sm = 0);
cudaError_t launch_attend(const void* q, int q_f32, int n_q_heads, const KvView& kv, const int32_t* idx,
                          const int32_t* count, int C, const int32_t* tail_begin, int max_tail, void* out,
                          float* lse, void* workspace, const AttendPlan& plan, cudaStream_t s);

// Launches step 4 with its split-K partials in the library's fixed scratch array
// (asp_sparse_attend_noalloc); `plan.workspace_bytes` must fit in it.
cudaError_t launch_attend_noalloc(const void* q, int q_f32, int n_q_heads, const KvView& kv, const int32_t* idx,
                                  const int32_t* count, int C, const int32_t* tail_begin, int max_tail, void* out,
                                  float* lse, const AttendPlan& plan, cudaStream_t s);

// ---- failure detection ----------------------------------------------------------
// One warp waits on a barrier nothing arrives on, bounded to `tries` attempts;
// *returned = 1 once it has given up (2 if the wait had succeeded).
cudaError_t launch_wait_limit_check(int tries, int32_t* returned, cudaStream_t s);

// ---- comparison path ----------------------------------------------------------
cudaError_t launch_quest_meta(const KvView& kv, int quest_page, void* meta, cudaStream_t s);
cudaError_t launch_quest_score(const void* q, int q_f32, int n_q_heads, const KvView& kv, const void* meta,
                               int quest_page, float* page_scores, cudaStream_t s);

}  // namespace asp
