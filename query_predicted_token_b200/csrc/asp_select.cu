// asp_select.cu -- step 3: top-C selection per (sequence, KV head).
//
// The C largest scores of scores[0:T_b] (IEEE order, -0.0 == +0.0), ties at the
// threshold to the lowest index, written ascending.
//
// One thread-block cluster of NC CTAs per row; each CTA keeps its segment of the
// row as 32-bit order keys in shared memory, so the row is read from L2/HBM once.
// NC is chosen so that the whole grid is resident in one wave.  Radix select
// from the most significant end with digits of 11, 11 and 10 bits: every CTA
// builds a histogram of its candidates (warp-aggregated with match/ballot, so a
// hot bin costs one shared atomic per warp), the cluster sums the NC histograms
// through distributed shared memory, and every CTA picks the same threshold
// digit.  Only keys that still match the threshold prefix take part in later
// passes, and a pass stops the search once the threshold bin holds exactly the
// number of tokens still needed (for continuous scores: after two passes).  The
// ascending write-out is a stable compaction: per 512-token tile, ballots give
// each token its rank among "above threshold" and "at threshold" tokens, with
// the counts of lower-ranked CTAs added from DSMEM.
#include <cooperative_groups.h>

#include "asp_common.cuh"
#include "asp_internal.h"

namespace cg = cooperative_groups;

namespace asp {
namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kSegMax = 32768;   // keys per CTA (128 KB of shared memory)
constexpr int kBins = 2048;      // widest digit: 11 bits
constexpr int kStaticSmem = 2 * kBins * 4 + 1024;

__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;   // -0.0 ties +0.0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Exclusive scan of one int per thread over the CTA; also returns the total.
__device__ __forceinline__ int cta_exclusive_scan(int x, int* wsum, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = x;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = lane < kWarps ? wsum[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    if (lane < kWarps) wsum[lane] = w;
  }
  __syncthreads();
  const int excl = incl - x + (warp > 0 ? wsum[warp - 1] : 0);
  *total = wsum[kWarps - 1];
  __syncthreads();
  return excl;
}

__global__ void __launch_bounds__(kThreads, 2) select_kernel(SelectArgs a) {
  cg::cluster_group cluster = cg::this_cluster();
  const int nc = (int)cluster.num_blocks();
  const int rank = (int)cluster.block_rank();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int row = blockIdx.y;
  const int b = row / a.rows_per_seq;

  extern __shared__ uint32_t keys[];
  __shared__ int hist[2][kBins];
  __shared__ int wsum[kWarps];
  __shared__ int wg[kWarps], we[kWarps];
  __shared__ int s_digit, s_above, s_bincnt, s_tile_gt, s_tile_eq, s_last_sel;
  __shared__ int s_cnt[2];

  int T = a.seq_lens ? a.seq_lens[b] : a.t_max;
  T = T < 0 ? 0 : (T > a.t_max ? a.t_max : T);
  const int E = a.expand;
  const int n_units = (T + E - 1) / E;
  const int out_stride = a.c_units * E;
  int32_t* out = a.idx + (size_t)row * out_stride;
  const int seg = (n_units + nc - 1) / nc;
  const int lo = min(n_units, rank * seg);
  const int hi = min(n_units, lo + seg);
  const int nloc = hi - lo;

  auto write_unit = [&](int u, int pos) {
    for (int e = 0; e < E; ++e) {
      const int tok = u * E + e;
      out[pos * E + e] = tok < T ? tok : -1;
    }
  };

  if (n_units <= a.c_units) {   // every unit chosen (uniform over the cluster)
    for (int u = lo + tid; u < hi; u += kThreads) write_unit(u, u);
    for (int i = n_units * E + rank * kThreads + tid; i < out_stride; i += nc * kThreads) out[i] = -1;
    if (rank == 0 && tid == 0) a.count[row] = T;
    return;
  }

  const float* srow = a.scores + (size_t)row * a.row_stride + lo;
  for (int i = tid; i < nloc; i += kThreads) keys[i] = order_key(srow[i]);
  __syncthreads();

  uint32_t prefix = 0u, mask = 0u;
  int krem = a.c_units;
#pragma unroll 1
  for (int pass = 0; pass < 3; ++pass) {
    const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
    const int nb = pass == 2 ? 1024 : 2048;
    const uint32_t dmask = (uint32_t)nb - 1u;
    int* h = hist[pass & 1];
    for (int i = tid; i < nb; i += kThreads) h[i] = 0;
    __syncthreads();
    for (int base = 0; base < nloc; base += kThreads) {
      const int i = base + tid;
      bool act = false;
      uint32_t dig = 0u;
      if (i < nloc) {
        const uint32_t key = keys[i];
        act = (key & mask) == prefix;
        dig = (key >> shift) & dmask;
      }
      const uint32_t am = __ballot_sync(0xffffffffu, act);
      if (act) {
        const uint32_t peers = __match_any_sync(am, dig);
        if (lane == __ffs(peers) - 1) atomicAdd(&h[dig], __popc(peers));
      }
    }
    cluster.sync();
    // thread t owns digits nb-1-(t*bpt .. t*bpt+bpt-1): thread order is descending digit order
    const int bpt = nb / kThreads;
    int v[kBins / kThreads];
    int local = 0;
#pragma unroll
    for (int j = 0; j < kBins / kThreads; ++j) {
      v[j] = 0;
      if (j < bpt) {
        const int d = nb - 1 - (tid * bpt + j);
        int sum = 0;
#pragma unroll
        for (int r = 0; r < 8; ++r)
          if (r < nc) sum += cluster.map_shared_rank(h, r)[d];
        v[j] = sum;
        local += sum;
      }
    }
    int total;
    const int excl = cta_exclusive_scan(local, wsum, &total);
    if (excl < krem && krem <= excl + local) {
      int run = excl;
      for (int j = 0; j < bpt; ++j) {
        if (run + v[j] >= krem) {
          s_digit = nb - 1 - (tid * bpt + j);
          s_above = run;
          s_bincnt = v[j];
          break;
        }
        run += v[j];
      }
    }
    __syncthreads();
    const int digit = s_digit;
    krem -= s_above;
    prefix |= (uint32_t)digit << shift;
    mask |= dmask << shift;
    const bool done = s_bincnt == krem;
    __syncthreads();
    if (done) break;
  }

  // counts of this CTA, published for the higher-ranked CTAs of the cluster
  int my_gt = 0, my_eq = 0;
  for (int i = tid; i < nloc; i += kThreads) {
    const uint32_t mk = keys[i] & mask;
    my_gt += mk > prefix;
    my_eq += mk == prefix;
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    my_gt += __shfl_xor_sync(0xffffffffu, my_gt, o);
    my_eq += __shfl_xor_sync(0xffffffffu, my_eq, o);
  }
  if (lane == 0) {
    wg[warp] = my_gt;
    we[warp] = my_eq;
  }
  __syncthreads();
  if (tid == 0) {
    int sg = 0, se = 0;
    for (int w = 0; w < kWarps; ++w) {
      sg += wg[w];
      se += we[w];
    }
    s_cnt[0] = sg;
    s_cnt[1] = se;
    s_last_sel = 0;
  }
  cluster.sync();
  int run_gt = 0, run_eq = 0;
  for (int r = 0; r < rank; ++r) {
    const int* rc = cluster.map_shared_rank(s_cnt, r);
    run_gt += rc[0];
    run_eq += rc[1];
  }

  const uint32_t lt_mask = (1u << lane) - 1u;
  for (int base = 0; base < nloc; base += kThreads) {
    const int i = base + tid;
    const bool valid = i < nloc;
    const uint32_t mk = valid ? (keys[i] & mask) : 0u;
    const bool gt = valid && mk > prefix;
    const bool eq = valid && mk == prefix;
    const uint32_t bg = __ballot_sync(0xffffffffu, gt);
    const uint32_t be = __ballot_sync(0xffffffffu, eq);
    if (lane == 0) {
      wg[warp] = __popc(bg);
      we[warp] = __popc(be);
    }
    __syncthreads();
    if (warp == 0) {
      int g = lane < kWarps ? wg[lane] : 0;
      int e = lane < kWarps ? we[lane] : 0;
      int gi = g, ei = e;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int yg = __shfl_up_sync(0xffffffffu, gi, o);
        const int ye = __shfl_up_sync(0xffffffffu, ei, o);
        if (lane >= o) {
          gi += yg;
          ei += ye;
        }
      }
      if (lane < kWarps) {
        wg[lane] = gi - g;
        we[lane] = ei - e;
      }
      if (lane == kWarps - 1) {
        s_tile_gt = gi;
        s_tile_eq = ei;
      }
    }
    __syncthreads();
    const int Gj = run_gt + wg[warp] + __popc(bg & lt_mask);
    const int Ej = run_eq + we[warp] + __popc(be & lt_mask);
    if (gt || (eq && Ej < krem)) {
      const int u = lo + i;
      write_unit(u, Gj + min(Ej, krem));
      if (u == n_units - 1) s_last_sel = 1;
    }
    run_gt += s_tile_gt;
    run_eq += s_tile_eq;
    __syncthreads();
  }
  if (tid == 0 && nloc > 0 && hi == n_units) {
    a.count[row] = out_stride - (s_last_sel ? (n_units * E - T) : 0);
  }
  cluster.sync();   // keep this CTA's shared memory alive until the cluster is done reading it
}

// Cluster size: the largest NC whose grid (rows * NC CTAs) is resident in one
// wave; if none is, the smallest NC whose segment fits in shared memory.
int pick_cluster(int rows, int len_max) {
  const int sms = sm_count();
  int best = 0;
  for (int nc = 1; nc <= 8; nc *= 2) {
    const int seg = (len_max + nc - 1) / nc;
    if (seg > kSegMax) continue;
    const int smem = seg * 4 + kStaticSmem;
    int per_sm = (227 * 1024) / smem;
    per_sm = per_sm > 2 ? 2 : per_sm;
    if ((long)rows * nc <= (long)sms * per_sm) best = nc;
    else if (!best) best = -nc;   // remembers the smallest fitting NC
  }
  if (best > 0) return best;
  return best < 0 ? -best : 8;
}

}  // namespace

bool select_supported(int t_max, int expand) {
  const int len = (t_max + expand - 1) / expand;
  return (len + 7) / 8 <= kSegMax;
}

cudaError_t launch_select(const SelectArgs& a, cudaStream_t s) {
  const int len_max = (a.t_max + a.expand - 1) / a.expand;
  const int nc = pick_cluster(a.n_rows, len_max);
  const int seg_max = (len_max + nc - 1) / nc;
  const size_t smem = (size_t)(seg_max > 0 ? seg_max : 1) * 4;
  if (prepare_kernel((const void*)select_kernel, smem, kThreads) < 1) return cudaErrorInvalidConfiguration;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(nc, a.n_rows, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = nc;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, select_kernel, a);
}

ASP_STATUS_READER(read_status_select)

}  // namespace asp
