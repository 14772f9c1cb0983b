// asp_predict.cu -- step 1: predicted next query per query head.
//
// For each window w: ridge fit of q_t on the lags q_{t-w}..q_{t-1} (samples =
// channels), a = (X X^T + lambda I)^-1 X q_t; weights alpha = softmax(a) (or a);
// qhat^(w) = sum_i alpha_i q_{t-w+i}; qhat = mean over the windows.
//
// One warp per query head; the history is tiny (17 x 128 fp32 for W = 16), so
// the kernel is latency-bound and the work is arranged to keep the dependency
// chains short:
//  * the lags are ordered newest first (r = 0 is q_{t-1}), which makes every
//    window's system the *leading* w x w block of one matrix.  A Cholesky
//    factor's leading block is the factor of the leading block, and the forward
//    substitution of a leading block is the leading part of the full one, so a
//    single factorisation and forward solve serve all windows; only the back
//    substitution is per window;
//  * Gram and right-hand side in fp64 (products of fp32 values are exact in
//    fp64), chunked over 32 (i, j) pairs with a warp reduce-scatter;
//  * the Cholesky is warp-parallel (right-looking: lane i updates row i).
#include "asp_common.cuh"
#include "asp_internal.h"

namespace asp {
namespace {

constexpr int kWarps = 4;
constexpr int kLda = 33;   // row stride (doubles) of the lag Gram: column accesses hit distinct banks
constexpr size_t kSolveBytes = (32 * kLda + 3 * 32) * 8;   // A[32][33], rhs, 1/diag, spare (fp64)

template <int N, int OFF>
struct ReduceScatterD {
  __device__ __forceinline__ static void run(double* vals, int lane) {
    if constexpr (OFF >= 1) {
      if constexpr (N >= 2) {
        constexpr int H = N / 2;
        const bool upper = (lane & OFF) != 0;
#pragma unroll
        for (int i = 0; i < H; ++i) {
          const double send = upper ? vals[i] : vals[i + H];
          const double keep = upper ? vals[i + H] : vals[i];
          vals[i] = keep + __shfl_xor_sync(0xffffffffu, send, OFF);
        }
        ReduceScatterD<H, OFF / 2>::run(vals, lane);
      } else {
        vals[0] += __shfl_xor_sync(0xffffffffu, vals[0], OFF);
        ReduceScatterD<1, OFF / 2>::run(vals, lane);
      }
    }
  }
};

template <int D>
__global__ void __launch_bounds__(kWarps * 32) predict_kernel(PredictArgs a) {
  constexpr int CPL = D / 32;   // channels per lane
  extern __shared__ __align__(16) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int head = blockIdx.x * kWarps + warp;
  if (head >= a.n_heads) return;

  const int n = a.wmax + 1;            // vectors used: target + wmax lags
  const int nslot = a.W + 1;
  // per-warp shared memory: hv[n][D] fp32, A[wmax][wmax] fp64, rhs[wmax], y[wmax], coef[wmax]
  const size_t hv_bytes = (((size_t)(a.wmax + 1) * D * 4) + 15) / 16 * 16;
  uint8_t* base = smem + warp * (hv_bytes + kSolveBytes);
  float* hv = reinterpret_cast<float*>(base);
  double* A = reinterpret_cast<double*>(base + hv_bytes);
  double* rhs = A + 32 * kLda;
  double* invd = rhs + 32;

  float* hist = a.qhist + (size_t)head * nslot * D;
  // chronological position s (0 = oldest, W = newest) -> ring slot
  const int start = a.q_new ? a.ring_start + 1 : a.ring_start;
  // hv[0] = q_t (target), hv[1 + r] = q_{t-1-r} for r < wmax
  for (int v = 0; v < n; ++v) {
    const int s = a.W - v;   // chronological position of hv[v]
    const int slot = (start + s) % nslot;
    for (int c = lane; c < D; c += 32) {
      float x;
      if (a.q_new && v == 0) {
        const size_t off = (size_t)head * D + c;
        x = a.q_new_f32 ? static_cast<const float*>(a.q_new)[off]
                        : __bfloat162float(static_cast<const __nv_bfloat16*>(a.q_new)[off]);
        hist[(size_t)slot * D + c] = x;   // push into the ring (slot == ring_start)
      } else {
        x = hist[(size_t)slot * D + c];
      }
      hv[v * D + c] = x;
    }
  }
  __syncwarp();

  // Gram over the lags (newest first) and right-hand side, fp64, 32 pairs per round.
  // Pairs are enumerated as the lower triangle (i, j), j <= i < wmax, row by row,
  // followed by the wmax (lag i, target) pairs of the right-hand side.
  const int wm = a.wmax;
  const int n_lag_pairs = wm * (wm + 1) / 2;
  const int n_pairs = n_lag_pairs + wm;
  int ci = 0, cj = 0;   // pair cursor (uniform across the warp)
  for (int p0 = 0; p0 < n_pairs; p0 += 32) {
    double vals[32];
    int si = ci, sj = cj;   // first pair of this round
#pragma unroll
    for (int k = 0; k < 32; ++k) {
      const int pi = p0 + k;
      double acc = 0.0;
      if (pi < n_pairs) {
        const int u = (ci < wm) ? 1 + ci : 1 + cj;   // lag row
        const int v = (ci < wm) ? 1 + cj : 0;        // lag column, or the target
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
          const int ch = lane + 32 * c;
          acc = fma((double)hv[u * D + ch], (double)hv[v * D + ch], acc);
        }
        if (ci < wm) {
          if (++cj > ci) { ++ci; cj = 0; }
        } else {
          ++cj;
        }
      }
      vals[k] = acc;
    }
    ReduceScatterD<32, 16>::run(vals, lane);
    // lane holds pair p0 + lane: step the round's first pair forward by `lane`
    int ti = si, tj = sj;
    for (int k = 0; k < lane; ++k) {
      if (ti < wm) {
        if (++tj > ti) { ++ti; tj = 0; }
      } else {
        ++tj;
      }
    }
    if (p0 + lane < n_pairs) {
      if (ti < wm) A[ti * kLda + tj] = vals[0] + (ti == tj ? a.lam : 0.0);
      else rhs[tj] = vals[0];
    }
  }
  __syncwarp();

  // Cholesky A = L L^T in place (lower triangle), right-looking.  Every lane
  // computes the pivot; lane i owns row i; column k is broadcast by shuffles.
  for (int k = 0; k < wm; ++k) {
    const double dkk = sqrt(A[k * kLda + k]);
    const double inv = 1.0 / dkk;
    double lik = 0.0;
    if (lane > k && lane < wm) {
      lik = A[lane * kLda + k] * inv;
      A[lane * kLda + k] = lik;
    }
    if (lane == k) {
      A[k * kLda + k] = dkk;
      invd[k] = inv;
    }
    for (int j = k + 1; j < wm; ++j) {
      const double ljk = __shfl_sync(0xffffffffu, lik, j);
      if (lane >= j && lane < wm) A[lane * kLda + j] -= lik * ljk;
    }
    __syncwarp();
  }
  // forward substitution L z = rhs (shared by every window): lane i keeps z_i
  double z = lane < wm ? rhs[lane] : 0.0;
  for (int k = 0; k < wm; ++k) {
    const double zk = __shfl_sync(0xffffffffu, z, k) * invd[k];
    if (lane == k) z = zk;
    if (lane > k && lane < wm) z -= A[lane * kLda + k] * zk;
  }

  double acc[CPL];
#pragma unroll
  for (int c = 0; c < CPL; ++c) acc[c] = 0.0;
  for (int wi = 0; wi < a.n_win; ++wi) {
    const int w = a.windows[wi];
    // back substitution L_w^T a = z_w on the leading w x w block: lane i keeps a_i
    double av = lane < w ? z : 0.0;
    for (int k = w - 1; k >= 0; --k) {
      const double ak = __shfl_sync(0xffffffffu, av, k) * invd[k];
      if (lane == k) av = ak;
      if (lane < k) av -= A[k * kLda + lane] * ak;
    }
    // weights over the w lags
    double wgt = lane < w ? av : 0.0;
    if (!a.coef_raw) {
      double m = lane < w ? wgt : -INFINITY;
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) m = fmax(m, __shfl_xor_sync(0xffffffffu, m, o));
      const double e = lane < w ? exp(wgt - m) : 0.0;
      double zs = e;
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) zs += __shfl_xor_sync(0xffffffffu, zs, o);
      wgt = e / zs;
    }
    // lag r (q_{t-1-r}) weights the vector one step later, q_{t-r} = hv[r]
    for (int r = 0; r < w; ++r) {
      const double wr = __shfl_sync(0xffffffffu, wgt, r);
#pragma unroll
      for (int c = 0; c < CPL; ++c) acc[c] = fma(wr, (double)hv[r * D + lane + 32 * c], acc[c]);
    }
    __syncwarp();
  }
  float* out = a.qpred + (size_t)head * D;
#pragma unroll
  for (int c = 0; c < CPL; ++c) out[lane + 32 * c] = (float)(acc[c] / a.n_win);
}

}  // namespace

cudaError_t launch_predict(const PredictArgs& a, cudaStream_t s) {
  const int grid = (a.n_heads + kWarps - 1) / kWarps;
  const size_t hv_bytes = (((size_t)(a.wmax + 1) * a.head_dim * 4) + 15) / 16 * 16;
  const size_t smem = kWarps * (hv_bytes + kSolveBytes);
  auto kern = a.head_dim == 64 ? predict_kernel<64> : predict_kernel<128>;
  if (prepare_kernel((const void*)kern, smem, kWarps * 32) < 1) return cudaErrorInvalidConfiguration;
  kern<<<grid, kWarps * 32, smem, s>>>(a);
  return cudaGetLastError();
}

ASP_STATUS_READER(read_status_predict)

}  // namespace asp
