// asp_score.cu -- step 2: score every cached key with its group's predicted queries.
//
// scores[b, h, j] = max_g (qpred[b, h*G+g] . k[b, h, j]) / sqrt(d),  j < T_b.
//
// HBM-bound stream (one read of every key row).  Design for sm_100a:
//  * the (sequence, KV head, 16-row block) list is flattened and cut into one
//    contiguous range per warp of a persistent grid, so every warp streams a
//    contiguous region of the cache (or of its pages);
//  * each warp runs its own STAGES-deep pipeline of 1-D bulk copies (TMA) of one
//    16-row block each into shared memory, completion counted on an mbarrier,
//    with an L2 evict-first hint since every key is read once;
//  * compute reads 16-byte vectors from shared memory (conflict-free), each lane
//    owning 8 bf16 (or 4 fp32) channels of a row; the G partial dot products of
//    several rows are summed over the row's lanes with a warp reduce-scatter
//    (about one shuffle per (row, head) instead of log2 of the lane count);
//  * packed fp32x2 FMAs (FFMA2) halve the issue slots of the dot products.
#include <cfloat>

#include "asp_common.cuh"
#include "asp_internal.h"

namespace asp {
namespace {

constexpr int kRows = 16;   // rows per bulk copy / block

struct ScoreParams {
  const float* qpred;
  int n_q_heads;
  const uint8_t* k;
  int batch, n_kv, t_max, page_size, max_pages, n_pages;
  const int32_t* page_table;
  const int32_t* seq_lens;
  float* scores;
  int32_t* hist;   // optional per-row histogram of the top 11 key bits
  float scale;
};

struct Cursor {
  int b, h, blk, nblk, T;
};

template <typename KT, int D, int G, int WARPS, int STAGES>
__global__ void __launch_bounds__(WARPS * 32, 1) score_kernel(ScoreParams p) {
  using E = Elem<KT>;
  constexpr int ROW_BYTES = D * E::kBytes;
  constexpr int LPR = ROW_BYTES / 16;        // lanes per row
  constexpr int RPS = 32 / LPR;              // rows per warp step
  constexpr int CPL = E::kPerVec;            // channels per lane
  constexpr int NSTEP = kRows / RPS;
  constexpr int BLOCK_BYTES = kRows * ROW_BYTES;
  constexpr int SPP = (NSTEP * G <= 32) ? NSTEP : (32 / G);   // steps per reduce pass
  constexpr int NPASS = NSTEP / SPP;
  constexpr int NV = SPP * G;                // partial sums per lane per pass
  static_assert(LPR >= 2 && LPR <= 32 && 32 % LPR == 0, "row must span 2..32 lanes");
  static_assert(NSTEP % SPP == 0 && NV <= 32 && G * LPR >= NV, "reduce layout");

  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ int scratch[33];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint8_t* wbuf = smem + (size_t)warp * STAGES * BLOCK_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (size_t)WARPS * STAGES * BLOCK_BYTES) + warp * STAGES;
  int* pre = reinterpret_cast<int*>(smem + (size_t)WARPS * STAGES * BLOCK_BYTES + WARPS * STAGES * 8);
  int* lens = pre + p.batch + 1;

  pdl_wait();      // inputs may come from the previous kernel (the predicted queries, the cleared histogram)
  pdl_trigger();
  for (int b = threadIdx.x; b < p.batch; b += blockDim.x) {
    int t = p.seq_lens ? p.seq_lens[b] : p.t_max;
    lens[b] = t < 0 ? 0 : (t > p.t_max ? p.t_max : t);
  }
  __syncthreads();
  cta_prefix_sum(p.batch, pre, [&](int b) { return ((lens[b] + kRows - 1) / kRows) * p.n_kv; }, scratch);

  if (lane == 0) {
    for (int s = 0; s < STAGES; ++s) mbar_init(&bars[s], 1);
    mbar_init_fence();
  }
  __syncwarp();

  const int total = pre[p.batch];
  const int nw_total = gridDim.x * WARPS;
  const int gw = blockIdx.x * WARPS + warp;
  const int chunk = (total + nw_total - 1) / nw_total;
  const int i0 = min(total, gw * chunk);
  const int i1 = min(total, i0 + chunk);
  if (i0 >= i1) return;

  auto locate = [&](int i, Cursor& c) {
    int lo = 0, hi = p.batch;   // pre[lo] <= i < pre[hi]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (pre[mid] <= i) lo = mid; else hi = mid;
    }
    c.b = lo;
    c.T = lens[lo];
    c.nblk = (pre[lo + 1] - pre[lo]) / p.n_kv;
    const int r = i - pre[lo];
    c.h = r / c.nblk;
    c.blk = r - c.h * c.nblk;
  };
  auto advance = [&](Cursor& c) {
    if (++c.blk == c.nblk) {
      c.blk = 0;
      if (++c.h == p.n_kv) {
        c.h = 0;
        do { ++c.b; } while (c.b < p.batch && pre[c.b + 1] == pre[c.b]);
        if (c.b < p.batch) {
          c.T = lens[c.b];
          c.nblk = (pre[c.b + 1] - pre[c.b]) / p.n_kv;
        }
      }
    }
  };

  const uint64_t policy = l2_evict_first_policy();
  int pt_b = -1, pt_base = 0, pt_val = -1;   // page-table window cache: entry pt_base + lane of row pt_b

  auto issue = [&](int slot, const Cursor& c) {
    const int j0 = c.blk * kRows;
    const uint8_t* src = nullptr;
    uint32_t bytes = 0;
    if (p.page_size == 0) {
      const int rows = min(kRows, c.T - j0);
      src = p.k + ((size_t)(c.b * p.n_kv + c.h) * p.t_max + j0) * ROW_BYTES;
      bytes = (uint32_t)rows * ROW_BYTES;
    } else {
      const int lp = j0 / p.page_size;
      if (c.b != pt_b || lp < pt_base || lp >= pt_base + 32) {
        pt_b = c.b;
        pt_base = lp;
        const int e = pt_base + lane;
        pt_val = e < p.max_pages ? p.page_table[(size_t)c.b * p.max_pages + e] : -1;
      }
      const int page = __shfl_sync(0xffffffffu, pt_val, lp - pt_base);
      if (page >= 0 && page < p.n_pages) {
        src = p.k + (((size_t)page * p.n_kv + c.h) * p.page_size + (j0 % p.page_size)) * ROW_BYTES;
        bytes = BLOCK_BYTES;
      } else if (lane == 0) {
        flag_status(ASP_DEV_BAD_PAGE);
      }
    }
    if (lane == 0) {
      fence_proxy_async_smem();
      mbar_arrive_expect_tx(&bars[slot], bytes);
      if (bytes) bulk_g2s_hint(wbuf + slot * BLOCK_BYTES, src, bytes, &bars[slot], policy);
    }
  };

  float2 q2[G][CPL / 2];
  auto load_q = [&](int b, int h) {
    const float* qp = p.qpred + (size_t)(b * p.n_q_heads + h * G) * D + (lane % LPR) * CPL;
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
      for (int c = 0; c < CPL / 2; ++c) {
        const float2 x = *reinterpret_cast<const float2*>(qp + g * D + 2 * c);
        q2[g][c] = make_float2(x.x * p.scale, x.y * p.scale);
      }
  };

  Cursor ic, cc;
  locate(i0, ic);
  cc = ic;
  int qb = cc.b, qh = cc.h;
  load_q(qb, qh);

  int issued = 0;
#pragma unroll 1
  for (int s = 0; s < STAGES && i0 + s < i1; ++s) {
    issue(s, ic);
    advance(ic);
    ++issued;
  }

  int consumed = 0;
  bool ok = true;
#pragma unroll 1
  for (int i = i0; i < i1; ++i) {
    const int k = i - i0;
    const int slot = k % STAGES;
    const uint32_t parity = (uint32_t)(k / STAGES) & 1u;
    if (cc.b != qb || cc.h != qh) {
      qb = cc.b;
      qh = cc.h;
      load_q(qb, qh);
    }
    ok = __all_sync(0xffffffffu, mbar_wait(&bars[slot], parity));
    if (!ok) break;
    ++consumed;

    const uint8_t* base = wbuf + slot * BLOCK_BYTES;
    const int j0 = cc.blk * kRows;
    float* srow = p.scores + (size_t)(cc.b * p.n_kv + cc.h) * p.t_max;
#pragma unroll
    for (int pass = 0; pass < NPASS; ++pass) {
      float vals[NV];
#pragma unroll
      for (int s = 0; s < SPP; ++s) {
        const int row = (pass * SPP + s) * RPS + lane / LPR;
        const uint4 v = *reinterpret_cast<const uint4*>(base + row * ROW_BYTES + (lane % LPR) * 16);
        float2 kf[CPL / 2];
        E::unpack(v, kf);
#pragma unroll
        for (int g = 0; g < G; ++g) {
          float2 acc = __fmul2_rn(kf[0], q2[g][0]);
#pragma unroll
          for (int c = 1; c < CPL / 2; ++c) acc = __ffma2_rn(kf[c], q2[g][c], acc);
          vals[s * G + g] = acc.x + acc.y;
        }
      }
      ReduceScatter<NV, LPR / 2>::run(vals, lane);
      constexpr int VPL = NV >= LPR ? NV / LPR : 1;   // values held per lane
      constexpr int LPS = G * LPR / NV;               // lanes holding one row's G values
      float m = vals[0];
#pragma unroll
      for (int t = 1; t < VPL; ++t) m = fmaxf(m, vals[t]);
#pragma unroll
      for (int o = 1; o < LPS; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      const int l = lane % LPR;
      bool has = false;
      if (l % LPS == 0) {
        const int row = (pass * SPP + l / LPS) * RPS + lane / LPR;
        const int j = j0 + row;
        if (j < cc.T) {
          srow[j] = m;
          has = true;
        }
      }
      if (p.hist) {   // first radix pass of the selection, fused: count the top key bits
        const uint32_t dig = order_key(m) >> kTopShift;
        const uint32_t hm = __ballot_sync(0xffffffffu, has);
        if (has) {
          const uint32_t peers = __match_any_sync(hm, dig);
          if (lane == __ffs(peers) - 1)
            atomicAdd(p.hist + (size_t)(cc.b * p.n_kv + cc.h) * kTopBins + dig, __popc(peers));
        }
      }
    }
    __syncwarp();
    if (issued < i1 - i0) {
      issue(slot, ic);
      advance(ic);
      ++issued;
    }
    advance(cc);
  }
  if (!ok) {
    // a wait ran out: give the copies still in flight a bounded chance to land
    for (int k = consumed + 1; k < issued; ++k) mbar_wait(&bars[k % STAGES], (uint32_t)(k / STAGES) & 1u);
  }
}

template <typename KT, int D, int G>
cudaError_t launch_score_t(const ScoreParams& p, cudaStream_t s) {
  constexpr int WARPS = 8;
  constexpr int BLOCK_BYTES = kRows * D * Elem<KT>::kBytes;
  constexpr int STAGES = (12288 / BLOCK_BYTES) > 2 ? (12288 / BLOCK_BYTES) : 2;
  auto kern = score_kernel<KT, D, G, WARPS, STAGES>;
  const size_t smem = (size_t)WARPS * STAGES * BLOCK_BYTES + WARPS * STAGES * 8 + (2 * (size_t)p.batch + 1) * 4;
  const int per_sm = prepare_kernel((const void*)kern, smem, WARPS * 32);
  if (per_sm < 1) return cudaErrorInvalidConfiguration;
  return launch_pdl(kern, dim3(sm_count() * per_sm), dim3(WARPS * 32), smem, s, p);
}

template <typename KT, int D>
cudaError_t dispatch_g(int G, const ScoreParams& p, cudaStream_t s) {
  switch (G) {
    case 1: return launch_score_t<KT, D, 1>(p, s);
    case 2: return launch_score_t<KT, D, 2>(p, s);
    case 4: return launch_score_t<KT, D, 4>(p, s);
    case 8: return launch_score_t<KT, D, 8>(p, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

cudaError_t launch_score(const float* qpred, int n_q_heads, const KvView& kv, float* scores, cudaStream_t s,
                         int32_t* hist, bool early) {
  if (score_tc_supported(kv, n_q_heads, qpred)) return launch_score_tc(qpred, n_q_heads, kv, scores, s, hist, early);
  return launch_score_cuda_cores(qpred, n_q_heads, kv, scores, s, hist);
}

cudaError_t launch_score_cuda_cores(const float* qpred, int n_q_heads, const KvView& kv, float* scores,
                                    cudaStream_t s, int32_t* hist) {
  ScoreParams p;
  p.qpred = qpred;
  p.n_q_heads = n_q_heads;
  p.k = static_cast<const uint8_t*>(kv.k);
  p.batch = kv.batch;
  p.n_kv = kv.n_kv;
  p.t_max = kv.t_max;
  p.page_size = kv.page_size;
  p.max_pages = kv.max_pages;
  p.n_pages = kv.n_pages;
  p.page_table = kv.page_table;
  p.seq_lens = kv.seq_lens;
  p.scores = scores;
  p.hist = hist;
  p.scale = 1.0f / sqrtf((float)kv.head_dim);
  const int G = n_q_heads / kv.n_kv;
  if (kv.kv_f32) {
    return kv.head_dim == 64 ? dispatch_g<float, 64>(G, p, s) : dispatch_g<float, 128>(G, p, s);
  }
  return kv.head_dim == 64 ? dispatch_g<__nv_bfloat16, 64>(G, p, s) : dispatch_g<__nv_bfloat16, 128>(G, p, s);
}

ASP_STATUS_READER(read_status_score)

}  // namespace asp
