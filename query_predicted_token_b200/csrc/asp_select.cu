// One thread-block cluster of NC CTAs per row; each CTA keeps its segment of the
// row as 32-bit order keys in shared memory, so the row is read from L2/HBM once
// (16-byte loads).  NC is chosen so that the whole grid is resident in one wave.
// Radix select from the most significant end with digits of 11, 11 and 10 bits.
// The first digit's histogram either comes with the scores (the key scan builds
// it with global atomics while it streams the cache) or is built while the keys
// are loaded.  Later passes count only keys that still match the threshold
// prefix (warp-aggregated with ballot/match, one shared atomic per distinct
// digit), the cluster sums its NC histograms through distributed shared memory,
// and every CTA picks the same threshold digit; the search stops once the
// threshold bin holds exactly the number of tokens still needed (for continuous
// scores: after the second digit).  The ascending write-out is a stable
// compaction: one sweep per warp over a contiguous run of keys packs the
// candidates (above or at the threshold) in order into shared memory, one scan
// over warps and, through DSMEM, over lower-ranked CTAs gives the offsets, and
// the packed lists are written out with the lowest-index rule for ties.
#include <cooperative_groups.h>

#include "asp_common.cuh"
#include "asp_internal.h"

namespace cg = cooperative_groups;

namespace asp {
namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kSegMax = 32768;   // keys per CTA (128 KB of shared memory)
constexpr int kBins = kTopBins;  // widest digit: 11 bits
constexpr int kBpt = kBins / kThreads;
constexpr int kStaticSmem = 2 * kBins * 4 + 1024;
constexpr uint32_t kEqTag = 0x80000000u;

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

// Sums bin d of the NC histograms of the cluster (all remote loads in flight at once).
template <int NC>
__device__ __forceinline__ int cluster_bin_sum(cg::cluster_group& cluster, int* h, int d) {
  int v[NC];
#pragma unroll
  for (int r = 0; r < NC; ++r) v[r] = cluster.map_shared_rank(h, r)[d];
  int s = 0;
#pragma unroll
  for (int r = 0; r < NC; ++r) s += v[r];
  return s;
}

__device__ __forceinline__ int bin_sum(cg::cluster_group& cluster, int nc, int* h, int d) {
  switch (nc) {
    case 1: return h[d];
    case 2: return cluster_bin_sum<2>(cluster, h, d);
    case 4: return cluster_bin_sum<4>(cluster, h, d);
    default: return cluster_bin_sum<8>(cluster, h, d);
  }
}

__global__ void __launch_bounds__(kThreads, 2) select_kernel(SelectArgs a) {
  cg::cluster_group cluster = cg::this_cluster();
  const int nc = (int)cluster.num_blocks();
  const int rank = (int)cluster.block_rank();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int row = blockIdx.y;
  const int b = row / a.rows_per_seq;

  extern __shared__ __align__(16) uint32_t keys[];
  __shared__ int hist[2][kBins];
  __shared__ int wsum[kWarps];
  __shared__ int wg[kWarps], we[kWarps], wn[kWarps];
  __shared__ int s_digit, s_above, s_bincnt, s_last_sel;
  __shared__ int s_cnt[2];

  int T = a.seq_lens ? a.seq_lens[b] : a.t_max;
  T = T < 0 ? 0 : (T > a.t_max ? a.t_max : T);
  const int E = a.expand;
  const int n_units = (T + E - 1) / E;
  const int out_stride = a.c_units * E;
  int32_t* out = a.idx + (size_t)row * out_stride;
  const int seg = (((n_units + nc - 1) / nc) + 3) & ~3;   // multiple of 4: 16-byte loads
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

  // ---- load the segment as order keys (and, without a given first histogram, count its top bits)
  const bool own_h0 = a.hist0 == nullptr;
  int* h0 = hist[0];
  if (own_h0) {
    for (int i = tid; i < kBins; i += kThreads) h0[i] = 0;
    __syncthreads();
  }
  const float* srow = a.scores + (size_t)row * a.row_stride + lo;
  auto count0 = [&](bool act, uint32_t key) {
    const uint32_t dig = key >> kTopShift;
    const uint32_t am = __ballot_sync(0xffffffffu, act);
    if (act) {
      const uint32_t peers = __match_any_sync(am, dig);
      if (lane == __ffs(peers) - 1) atomicAdd(&h0[dig], __popc(peers));
    }
  };
  if ((a.row_stride & 3) == 0 && (reinterpret_cast<uintptr_t>(a.scores) & 15) == 0) {
    const int n4 = (nloc + 3) >> 2;
    for (int base = 0; base < n4; base += kThreads) {
      const int i4 = base + tid;
      uint32_t k4[4] = {0u, 0u, 0u, 0u};
      bool v4[4] = {false, false, false, false};
      if (i4 < n4) {
        const float4 f = reinterpret_cast<const float4*>(srow)[i4];
        const float fv[4] = {f.x, f.y, f.z, f.w};
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          v4[c] = 4 * i4 + c < nloc;
          k4[c] = order_key(fv[c]);
        }
        *reinterpret_cast<uint4*>(&keys[4 * i4]) = make_uint4(k4[0], k4[1], k4[2], k4[3]);
      }
      if (own_h0) {
#pragma unroll
        for (int c = 0; c < 4; ++c) count0(v4[c], k4[c]);
      }
    }
  } else {
    for (int base = 0; base < nloc; base += kThreads) {
      const int i = base + tid;
      uint32_t key = 0u;
      if (i < nloc) {
        key = order_key(srow[i]);
        keys[i] = key;
      }
      if (own_h0) count0(i < nloc, key);
    }
  }
  __syncthreads();

  // ---- radix passes: 11, 11, 10 bits; later passes only count keys that still match
  uint32_t prefix = 0u, mask = 0u;
  int krem = a.c_units;
#pragma unroll 1
  for (int pass = 0; pass < 3; ++pass) {
    const int shift = pass == 0 ? kTopShift : (pass == 1 ? 10 : 0);
    const int nb = pass == 2 ? 1024 : 2048;
    const uint32_t dmask = (uint32_t)nb - 1u;
    int* h = hist[pass & 1];
    if (pass > 0) {
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
    }
    const bool global_h = pass == 0 && !own_h0;
    if (!global_h) cluster.sync();
    // thread t owns digits nb-1-(t*bpt .. t*bpt+bpt-1): thread order is descending digit order
    const int bpt = nb / kThreads;
    int v[kBpt];
    int local = 0;
    const int32_t* g0 = global_h ? a.hist0 + (size_t)row * kBins : nullptr;
#pragma unroll
    for (int j = 0; j < kBpt; ++j) {
      v[j] = 0;
      if (j < bpt) {
        const int d = nb - 1 - (tid * bpt + j);
        v[j] = global_h ? g0[d] : bin_sum(cluster, nc, h, d);
        local += v[j];
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

  // ---- stable compaction.  Warp w owns the contiguous keys [w0, w1): one sweep
  // packs the local indices of keys above (and, tagged, at) the threshold, in
  // order, into the front of that range of `keys` (writes never pass the read point).
  const int R = (((nloc + kWarps - 1) / kWarps) + 31) & ~31;
  const int w0 = min(nloc, warp * R), w1 = min(nloc, w0 + R);
  const uint32_t lt_mask = (1u << lane) - 1u;
  int c_gt = 0, c_eq = 0;
  for (int i0 = w0; i0 < w1; i0 += 32) {
    const int i = i0 + lane;
    const uint32_t mk = i < w1 ? (keys[i] & mask) : 0u;
    const bool gt = i < w1 && mk > prefix;
    const bool eq = i < w1 && mk == prefix;
    const uint32_t bg = __ballot_sync(0xffffffffu, gt);
    const uint32_t be = __ballot_sync(0xffffffffu, eq);
    const uint32_t bs = bg | be;
    if (gt || eq) keys[w0 + c_gt + c_eq + __popc(bs & lt_mask)] = (uint32_t)i | (eq ? kEqTag : 0u);
    c_gt += __popc(bg);
    c_eq += __popc(be);
  }
  if (lane == 0) {
    wg[warp] = c_gt;
    we[warp] = c_eq;
    wn[warp] = c_gt + c_eq;
  }
  __syncthreads();
  if (warp == 0) {
    const int g = lane < kWarps ? wg[lane] : 0;
    const int e = lane < kWarps ? we[lane] : 0;
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
      wg[lane] = gi - g;   // exclusive offsets of the warps
      we[lane] = ei - e;
    }
    if (lane == kWarps - 1) {
      s_cnt[0] = gi;   // this CTA's totals, read by the higher-ranked CTAs
      s_cnt[1] = ei;
    }
    if (lane == 0) s_last_sel = 0;
  }
  cluster.sync();
  int run_gt = wg[warp], run_eq = we[warp];
  if (rank > 0) {
    int rg[8], re[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      rg[r] = 0;
      re[r] = 0;
      if (r < rank) {
        const int* rc = cluster.map_shared_rank(s_cnt, r);
        rg[r] = rc[0];
        re[r] = rc[1];
      }
    }
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      run_gt += rg[r];
      run_eq += re[r];
    }
  }
  const int n_w = wn[warp];
  for (int k0 = 0; k0 < n_w; k0 += 32) {
    const int k = k0 + lane;
    const uint32_t e = k < n_w ? keys[w0 + k] : 0u;
    const bool is_eq = k < n_w && (e & kEqTag);
    const bool is_gt = k < n_w && !(e & kEqTag);
    const uint32_t bg = __ballot_sync(0xffffffffu, is_gt);
    const uint32_t be = __ballot_sync(0xffffffffu, is_eq);
    const int Gj = run_gt + __popc(bg & lt_mask);
    const int Ej = run_eq + __popc(be & lt_mask);
    if (is_gt || (is_eq && Ej < krem)) {
      const int u = lo + (int)(e & ~kEqTag);
      write_unit(u, Gj + min(Ej, krem));
      if (u == n_units - 1) s_last_sel = 1;
    }
    run_gt += __popc(bg);
    run_eq += __popc(be);
  }
  __syncthreads();
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
    const int seg = (((len_max + nc - 1) / nc) + 3) & ~3;
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
  return ((((len + 7) / 8) + 3) & ~3) <= kSegMax;
}

cudaError_t launch_select(const SelectArgs& a, cudaStream_t s) {
  const int len_max = (a.t_max + a.expand - 1) / a.expand;
  const int nc = pick_cluster(a.n_rows, len_max);
  const int seg_max = (((len_max + nc - 1) / nc) + 3) & ~3;
  const size_t smem = (size_t)(seg_max > 0 ? seg_max : 4) * 4;
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
