// asp_quest.cu -- the page-level comparison path.
//
// meta[b, h, p, 0 / 1, :] = per-channel minimum / maximum of the keys of page p;
// u_p = max_g sum_c max(q_c kmin_c, q_c kmax_c) / sqrt(d)
//     = max_g (q+ . kmax + q- . kmin) / sqrt(d),   q+ = max(q, 0), q- = min(q, 0),
// which turns the per-channel max into two packed FMAs without a select.
#include <cfloat>

#include "asp_common.cuh"
#include "asp_internal.h"

namespace asp {
namespace {

constexpr int kWarps = 4;

__device__ __forceinline__ int seq_len(const KvView& kv, int b) {
  int t = kv.seq_lens ? kv.seq_lens[b] : kv.t_max;
  return t < 0 ? 0 : (t > kv.t_max ? kv.t_max : t);
}

// One warp per page: grid (ceil(n_meta_pages / kWarps), batch * n_kv).
template <typename KT, int D>
__global__ void __launch_bounds__(kWarps * 32) quest_meta_kernel(KvView kv, int P, int npm, KT* meta) {
  using E = Elem<KT>;
  constexpr int ROW_BYTES = D * E::kBytes;
  constexpr int LPR = ROW_BYTES / 16;
  constexpr int RPS = 32 / LPR;
  constexpr int CPL = E::kPerVec;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int unit = blockIdx.y;
  const int b = unit / kv.n_kv, h = unit - b * kv.n_kv;
  const int p = blockIdx.x * kWarps + warp;
  const int T = seq_len(kv, b);
  if (p >= npm || p * P >= T) return;
  const int nrows = min(P, T - p * P);
  const uint8_t* base;
  if (kv.page_size == 0) {
    base = static_cast<const uint8_t*>(kv.k) + ((size_t)unit * kv.t_max + (size_t)p * P) * ROW_BYTES;
  } else {
    const int page = kv.page_table[(size_t)b * kv.max_pages + p];
    if (page < 0 || page >= kv.n_pages) {
      if (lane == 0) flag_status(ASP_DEV_BAD_PAGE);
      return;
    }
    base = static_cast<const uint8_t*>(kv.k) + ((size_t)page * kv.n_kv + h) * P * ROW_BYTES;
  }
  float mn[CPL], mx[CPL];
#pragma unroll
  for (int c = 0; c < CPL; ++c) {
    mn[c] = INFINITY;
    mx[c] = -INFINITY;
  }
  for (int r = lane / LPR; r < nrows; r += RPS) {
    const uint4 v = *reinterpret_cast<const uint4*>(base + (size_t)r * ROW_BYTES + (lane % LPR) * 16);
    float2 f[CPL / 2];
    E::unpack(v, f);
#pragma unroll
    for (int c = 0; c < CPL / 2; ++c) {
      mn[2 * c] = fminf(mn[2 * c], f[c].x);
      mx[2 * c] = fmaxf(mx[2 * c], f[c].x);
      mn[2 * c + 1] = fminf(mn[2 * c + 1], f[c].y);
      mx[2 * c + 1] = fmaxf(mx[2 * c + 1], f[c].y);
    }
  }
#pragma unroll
  for (int o = LPR; o < 32; o <<= 1)
#pragma unroll
    for (int c = 0; c < CPL; ++c) {
      mn[c] = fminf(mn[c], __shfl_xor_sync(0xffffffffu, mn[c], o));
      mx[c] = fmaxf(mx[c], __shfl_xor_sync(0xffffffffu, mx[c], o));
    }
  KT* dst = meta + ((size_t)unit * npm + p) * 2 * D + (lane % LPR) * CPL;
  const int grp = lane / LPR;
  if (grp == 0) {
#pragma unroll
    for (int c = 0; c < CPL; ++c) dst[c] = E::from_float(mn[c]);
  }
  if (grp == (RPS > 1 ? 1 : 0)) {
#pragma unroll
    for (int c = 0; c < CPL; ++c) dst[D + c] = E::from_float(mx[c]);
  }
}

// Page scores: grid (ceil(npm / (kWarps * PPW)), batch * n_kv); a warp takes PPW pages.
template <typename KT, int D, int G>
__global__ void __launch_bounds__(kWarps * 32) quest_score_kernel(const void* q, int q_f32, int n_q_heads, KvView kv,
                                                                  int P, int npm, const KT* meta, float* scores,
                                                                  float scale) {
  using E = Elem<KT>;
  constexpr int ROW_BYTES = D * E::kBytes;
  constexpr int LPR = ROW_BYTES / 16;
  constexpr int RPS = 32 / LPR;
  constexpr int CPL = E::kPerVec;
  constexpr int PPW = 16;                       // pages per warp
  constexpr int NSTEP = PPW / RPS;
  constexpr int SPP = (NSTEP * G <= 32) ? NSTEP : (32 / G);
  constexpr int NPASS = NSTEP / SPP;
  constexpr int NV = SPP * G;
  static_assert(NV <= 32 && G * LPR >= NV, "layout");
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int unit = blockIdx.y;
  const int b = unit / kv.n_kv, h = unit - b * kv.n_kv;
  const int T = seq_len(kv, b);
  const int npages = (T + P - 1) / P;
  const int p0 = (blockIdx.x * kWarps + warp) * PPW;
  if (p0 >= npages) return;

  float2 qp[G][CPL / 2], qn[G][CPL / 2];
  const int c0 = (lane % LPR) * CPL;
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const size_t off = (size_t)(b * n_q_heads + h * G + g) * D + c0;
#pragma unroll
    for (int c = 0; c < CPL / 2; ++c) {
      float x0, x1;
      if (q_f32) {
        x0 = static_cast<const float*>(q)[off + 2 * c];
        x1 = static_cast<const float*>(q)[off + 2 * c + 1];
      } else {
        x0 = __bfloat162float(static_cast<const __nv_bfloat16*>(q)[off + 2 * c]);
        x1 = __bfloat162float(static_cast<const __nv_bfloat16*>(q)[off + 2 * c + 1]);
      }
      x0 *= scale;
      x1 *= scale;
      qp[g][c] = make_float2(fmaxf(x0, 0.f), fmaxf(x1, 0.f));
      qn[g][c] = make_float2(fminf(x0, 0.f), fminf(x1, 0.f));
    }
  }
  const uint8_t* mrow = reinterpret_cast<const uint8_t*>(meta) + (size_t)unit * npm * 2 * ROW_BYTES;
  float* srow = scores + (size_t)unit * npm;
#pragma unroll
  for (int pass = 0; pass < NPASS; ++pass) {
    float vals[NV];
#pragma unroll
    for (int s = 0; s < SPP; ++s) {
      const int pg = p0 + (pass * SPP + s) * RPS + lane / LPR;
      float2 lo[CPL / 2], hi[CPL / 2];
      if (pg < npages) {
        const uint8_t* m = mrow + (size_t)pg * 2 * ROW_BYTES + (lane % LPR) * 16;
        E::unpack(*reinterpret_cast<const uint4*>(m), lo);
        E::unpack(*reinterpret_cast<const uint4*>(m + ROW_BYTES), hi);
      } else {
#pragma unroll
        for (int c = 0; c < CPL / 2; ++c) lo[c] = hi[c] = make_float2(0.f, 0.f);
      }
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float2 acc = __fmul2_rn(hi[0], qp[g][0]);
        acc = __ffma2_rn(lo[0], qn[g][0], acc);
#pragma unroll
        for (int c = 1; c < CPL / 2; ++c) {
          acc = __ffma2_rn(hi[c], qp[g][c], acc);
          acc = __ffma2_rn(lo[c], qn[g][c], acc);
        }
        vals[s * G + g] = acc.x + acc.y;
      }
    }
    ReduceScatter<NV, LPR / 2>::run(vals, lane);
    constexpr int VPL = NV >= LPR ? NV / LPR : 1;
    constexpr int LPS = G * LPR / NV;
    float m = vals[0];
#pragma unroll
    for (int t = 1; t < VPL; ++t) m = fmaxf(m, vals[t]);
#pragma unroll
    for (int o = 1; o < LPS; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    const int l = lane % LPR;
    if (l % LPS == 0) {
      const int pg = p0 + (pass * SPP + l / LPS) * RPS + lane / LPR;
      if (pg < npages) srow[pg] = m;
    }
  }
}

template <typename KT, int D>
cudaError_t meta_t(const KvView& kv, int P, void* meta, cudaStream_t s) {
  const int npm = (kv.t_max + P - 1) / P;
  quest_meta_kernel<KT, D><<<dim3((npm + kWarps - 1) / kWarps, kv.batch * kv.n_kv), kWarps * 32, 0, s>>>(
      kv, P, npm, static_cast<KT*>(meta));
  return cudaGetLastError();
}

template <typename KT, int D, int G>
cudaError_t score_t(const void* q, int q_f32, int n_q_heads, const KvView& kv, const void* meta, int P,
                    float* scores, cudaStream_t s) {
  const int npm = (kv.t_max + P - 1) / P;
  const int per_cta = kWarps * 16;
  quest_score_kernel<KT, D, G><<<dim3((npm + per_cta - 1) / per_cta, kv.batch * kv.n_kv), kWarps * 32, 0, s>>>(
      q, q_f32, n_q_heads, kv, P, npm, static_cast<const KT*>(meta), scores, 1.0f / sqrtf((float)D));
  return cudaGetLastError();
}

template <typename KT, int D>
cudaError_t score_g(int G, const void* q, int q_f32, int n_q_heads, const KvView& kv, const void* meta, int P,
                    float* scores, cudaStream_t s) {
  switch (G) {
    case 1: return score_t<KT, D, 1>(q, q_f32, n_q_heads, kv, meta, P, scores, s);
    case 2: return score_t<KT, D, 2>(q, q_f32, n_q_heads, kv, meta, P, scores, s);
    case 4: return score_t<KT, D, 4>(q, q_f32, n_q_heads, kv, meta, P, scores, s);
    case 8: return score_t<KT, D, 8>(q, q_f32, n_q_heads, kv, meta, P, scores, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

cudaError_t launch_quest_meta(const KvView& kv, int quest_page, void* meta, cudaStream_t s) {
  if (kv.kv_f32) return kv.head_dim == 64 ? meta_t<float, 64>(kv, quest_page, meta, s) : meta_t<float, 128>(kv, quest_page, meta, s);
  return kv.head_dim == 64 ? meta_t<__nv_bfloat16, 64>(kv, quest_page, meta, s)
                           : meta_t<__nv_bfloat16, 128>(kv, quest_page, meta, s);
}

cudaError_t launch_quest_score(const void* q, int q_f32, int n_q_heads, const KvView& kv, const void* meta,
                               int quest_page, float* page_scores, cudaStream_t s) {
  if (quest_tc_supported(kv, n_q_heads, q))   // bf16 bounds: on the tensor cores
    return launch_quest_score_tc(q, q_f32, n_q_heads, kv, meta, quest_page, page_scores, s);
  const int G = n_q_heads / kv.n_kv;
  if (kv.kv_f32) {
    return kv.head_dim == 64 ? score_g<float, 64>(G, q, q_f32, n_q_heads, kv, meta, quest_page, page_scores, s)
                             : score_g<float, 128>(G, q, q_f32, n_q_heads, kv, meta, quest_page, page_scores, s);
  }
  return kv.head_dim == 64 ? score_g<__nv_bfloat16, 64>(G, q, q_f32, n_q_heads, kv, meta, quest_page, page_scores, s)
                           : score_g<__nv_bfloat16, 128>(G, q, q_f32, n_q_heads, kv, meta, quest_page, page_scores, s);
}

ASP_STATUS_READER(read_status_quest)

}  // namespace asp
