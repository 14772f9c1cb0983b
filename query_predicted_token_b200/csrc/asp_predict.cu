// asp_predict.cu -- step 1: predicted next query per query head.
//
// For each window w: ridge fit of q_t on the lags q_{t-w}..q_{t-1} (samples =
// channels), a = (X X^T + lambda I)^-1 X q_t; weights alpha = softmax(a) (or a);
// qhat^(w) = sum_i alpha_i q_{t-w+i}; qhat = mean over the windows.
//
// One warp per query head; the history is tiny (17 x 128 fp32 for W = 16), so
// the kernel is latency-bound and the work is arranged to keep the dependency
// chains short:
//  * every lane loads its 16-byte slice of every history vector up front (all
//    loads in flight at once) and keeps them in registers;
//  * the lags are ordered newest first (r = 0 is q_{t-1}), which makes every
//    window's system the *leading* w x w block of one matrix.  A Cholesky
//    factor's leading block is the factor of the leading block, and the forward
//    substitution of a leading block is the leading part of the full one, so a
//    single factorisation and forward solve serve all windows; only the back
//    substitution is per window;
//  * Gram and right-hand side in fp32 (the lane's partial dot products, summed
//    over the warp with a 32-wide reduce-scatter), the Cholesky and both
//    substitutions in fp64 (the lag Gram's condition number is ~1e3 on AR(1)
//    histories; fp64 keeps the coefficients' error far below the output bound);
//  * the Cholesky is warp-parallel (pivot computed by every lane, column
//    broadcast through shared memory, lane i updates row i).
#include "asp_common.cuh"
#include "asp_internal.h"

namespace asp {
namespace {

constexpr int kWarps = 4;
// Per-warp solve area for NV history vectors (NV - 1 lags): the lag Gram A with an
// odd row stride (column accesses hit distinct banks), then rhs/beta, 1/diag and a
// spare column of 32 doubles each (fp64).
template <int NV>
struct Solve {
  static constexpr int kRows = NV - 1;
  static constexpr int kLda = (NV - 1) | 1;
  static constexpr size_t kBytes = ((size_t)kRows * kLda + 3 * 32) * 8;
};

// 1/sqrt(x) for x > 0 in fp64: the fp32 hardware estimate refined by one
// Newton-Raphson step y <- y (3 - x y^2) / 2, which squares its relative error
// (about 1e-7 -> 1e-14); written as y + y (1/2 - (x/2) y^2), x/2 formed beside the
// estimate, so three dependent fp64 operations follow it.
__device__ __forceinline__ double rsqrt_f64(double x) {
  const double hx = 0.5 * x;
  const double y = (double)rsqrtf((float)x);
  return fma(y, fma(-hx * y, y, 0.5), y);
}

// Stores the reduced pair `q` (lane's pair of a round) into the solve arrays:
// pairs (i >= 1, j >= 1) are lag-Gram entries, pairs (i >= 1, 0) the right-hand side.
template <int LDA>
__device__ __forceinline__ void store_pair(int q, float val, int wmax, double lam, double* A, double* rhs) {
  int qi = (int)((sqrtf(8.f * q + 1.f) - 1.f) * 0.5f);
  while (qi * (qi + 1) / 2 > q) --qi;
  while ((qi + 1) * (qi + 2) / 2 <= q) ++qi;
  const int qj = q - qi * (qi + 1) / 2;
  if (qi >= 1 && qi <= wmax) {
    if (qj >= 1) A[(qi - 1) * LDA + (qj - 1)] = (double)val + (qi == qj ? lam : 0.0);
    else rhs[qi - 1] = (double)val;
  }
}

// Compile-time walk over the pairs (I, J), J <= I, P = I (I + 1) / 2 + J, so that
// every register of the history is addressed statically (rows outer, columns
// inner keeps the template recursion shallow).
template <int NV, int CPL, int I, int J>
struct GramCol {
  __device__ __forceinline__ static void run(const float (&h)[NV][CPL], float (&part)[32], int lane, int wmax,
                                             double lam, double* A, double* rhs) {
    constexpr int NPAIR = NV * (NV + 1) / 2;
    constexpr int P = I * (I + 1) / 2 + J;
    float acc = h[I][0] * h[J][0];
#pragma unroll
    for (int c = 1; c < CPL; ++c) acc = fmaf(h[I][c], h[J][c], acc);
    part[P % 32] = acc;
    if constexpr (P % 32 == 31 || P == NPAIR - 1) {
#pragma unroll
      for (int k = P % 32 + 1; k < 32; ++k) part[k] = 0.f;
      ReduceScatter<32, 16>::run(part, lane);
      const int q = (P / 32) * 32 + lane;
      if (q < NPAIR) store_pair<Solve<NV>::kLda>(q, part[0], wmax, lam, A, rhs);
    }
    if constexpr (J < I) GramCol<NV, CPL, I, J + 1>::run(h, part, lane, wmax, lam, A, rhs);
  }
};

template <int NV, int CPL, int I>
struct GramRows {
  __device__ __forceinline__ static void run(const float (&h)[NV][CPL], float (&part)[32], int lane, int wmax,
                                             double lam, double* A, double* rhs) {
    GramCol<NV, CPL, I, 0>::run(h, part, lane, wmax, lam, A, rhs);
    if constexpr (I + 1 < NV) GramRows<NV, CPL, I + 1>::run(h, part, lane, wmax, lam, A, rhs);
  }
};

// FAST: the windows are powers of two that fit one warp (PredictArgs::win_fast);
// the kernel for that case carries no code for the general one.  EXACT: the
// widest window has NV - 1 lags, so every bound on the lags is a constant.
// MODE (decode loop, FAST and EXACT only): the lag Gram of the next step holds
// only queries that are known one step ahead -- the next step's lags are this
// step's query and the W - 1 before it -- so its factorisation can run beside the
// current step instead of on the next step's critical path.
//   kPredFull:    factorise and predict (every other use);
//   kPredFactor:  only factorise the next step's lag Gram (the current query
//                 q_new becomes the newest lag) and store the factor;
//   kPredUsing:   predict with the factor the previous step stored: only the
//                 right-hand side (the lags' dot products with q_t) and the
//                 substitutions remain.
constexpr int kPredFull = 0, kPredFactor = 1, kPredUsing = 2;

template <int D, int NV, bool FAST, bool EXACT, int MODE = kPredFull>
__global__ void __launch_bounds__(kWarps * 32, NV <= 17 ? 4 : 1) predict_kernel(PredictArgs a) {
  constexpr int CPL = D / 32;   // contiguous channels per lane
  extern __shared__ __align__(16) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int head = blockIdx.x * kWarps + warp;
  static_assert(MODE == kPredFull || (FAST && EXACT), "the factor modes serve the decode loop's windows");
  pdl_trigger();   // the key scan may launch and run its prologue meanwhile
  if (MODE != kPredFactor && a.zero) {   // clear the next kernel's histogram (16-byte stores, spread over all warps)
    const size_t n4 = a.zero_words / 4;
    int4* z4 = reinterpret_cast<int4*>(a.zero);
    for (size_t i = (size_t)head * 32 + lane; i < n4; i += (size_t)gridDim.x * kWarps * 32) z4[i] = make_int4(0, 0, 0, 0);
    for (size_t i = n4 * 4 + (size_t)head * 32 + lane; i < a.zero_words; i += (size_t)gridDim.x * kWarps * 32) a.zero[i] = 0;
  }
  if (head >= a.n_heads) return;

  constexpr int kLda = Solve<NV>::kLda;
  double* A = reinterpret_cast<double*>(smem + warp * Solve<NV>::kBytes);   // [NV-1][kLda] lag Gram, then L
  double* rhs = A + Solve<NV>::kRows * kLda;
  double* invd = rhs + 32;

  const int wmax = EXACT ? NV - 1 : a.wmax;   // lags of the widest window
  const int n = wmax + 1;                      // vectors used: the target and wmax lags
  const int nslot = a.W + 1;
  float* hist = a.qhist + (size_t)head * nslot * D;
  const int start = a.q_new ? a.ring_start + 1 : a.ring_start;
  // h[v] = q_{t-v}: h[0] is the target q_t, h[1 + r] is lag r (q_{t-1-r})
  float h[NV][CPL];
#pragma unroll
  for (int v = 0; v < NV; ++v) {
#pragma unroll
    for (int c = 0; c < CPL; ++c) h[v][c] = 0.f;
    if (MODE == kPredFactor) {
      // the next step's vectors: h[0] (its target) unknown, h[1] = q_new, h[v >= 2] =
      // q_{t+1-v}, in slot ring_start + 1 - v (not the slot the current step's push
      // overwrites, so the two kernels may run at the same time)
      if (v >= 1 && v < n) {
        if (v == 1) {
          const size_t off = (size_t)head * D + lane * CPL;
#pragma unroll
          for (int c = 0; c < CPL; ++c)
            h[1][c] = a.q_new_f32 ? static_cast<const float*>(a.q_new)[off + c]
                                  : __bfloat162float(static_cast<const __nv_bfloat16*>(a.q_new)[off + c]);
        } else {
          int slot = a.ring_start + 1 - v;
          if (slot < 0) slot += nslot;
          const float* src = hist + (size_t)slot * D + lane * CPL;
#pragma unroll
          for (int c = 0; c < CPL; ++c) h[v][c] = src[c];
        }
      }
    } else if (v < n) {
      // start <= nslot and 0 <= W - v <= W < nslot: one subtraction wraps the slot
      int slot = start + a.W - v;
      if (slot >= nslot) slot -= nslot;
      float* src = hist + (size_t)slot * D + lane * CPL;
      if (v == 0 && a.q_new) {
        const size_t off = (size_t)head * D + lane * CPL;
#pragma unroll
        for (int c = 0; c < CPL; ++c)
          h[0][c] = a.q_new_f32 ? static_cast<const float*>(a.q_new)[off + c]
                                : __bfloat162float(static_cast<const __nv_bfloat16*>(a.q_new)[off + c]);
      } else if constexpr (CPL == 4) {
        const float4 x = *reinterpret_cast<const float4*>(src);
        h[v][0] = x.x; h[v][1] = x.y; h[v][2] = x.z; h[v][3] = x.w;
      } else {
        const float2 x = *reinterpret_cast<const float2*>(src);
        h[v][0] = x.x; h[v][1] = x.y;
      }
    }
  }
  constexpr int WMAX = NV - 1;   // lags the registers can hold
  // the stored factor of one head: rows of L scaled by 1 / L_ii ([WMAX][WMAX], j < i),
  // then the 1 / L_ii ([WMAX]); lane i's row is requested with the history, so
  // that both loads share one round trip
  constexpr int kFac = WMAX * WMAX + WMAX;
  double srow[MODE == kPredUsing ? WMAX : 1];
  double my_inv_f = 0.0;
  if constexpr (MODE == kPredUsing) {
    const double* fac = a.factor_in + (size_t)head * kFac;
#pragma unroll
    for (int j = 0; j < WMAX; ++j) srow[j] = (lane < WMAX && j < lane) ? fac[lane * WMAX + j] : 0.0;
    my_inv_f = lane < WMAX ? fac[WMAX * WMAX + lane] : 0.0;
  }
  if (MODE != kPredFactor && a.q_new) {   // push q_t into the ring: it replaces the oldest slot (ring_start)
    float* dst = hist + (size_t)a.ring_start * D + lane * CPL;
#pragma unroll
    for (int c = 0; c < CPL; ++c) dst[c] = h[0][c];
  }

  const int wm = wmax;
  if constexpr (MODE == kPredUsing) {
    // right-hand side only: the lags' dot products with the target, reduced over
    // the warp (lane r then holds rhs_r)
    float part[32];
#pragma unroll
    for (int r = 0; r < 32; ++r) {
      float acc = 0.f;
      if (r < WMAX) {
        acc = h[1 + r][0] * h[0][0];
#pragma unroll
        for (int c = 1; c < CPL; ++c) acc = fmaf(h[1 + r][c], h[0][c], acc);
      }
      part[r] = acc;
    }
    ReduceScatter<32, 16>::run(part, lane);
    // forward substitution L z = rhs with the stored factor: z_i = rhs_i / L_ii -
    // sum_{j<i} (L_ij / L_ii) z_j, one shuffle and one multiply-add per step
    const double my_inv = my_inv_f;
    double zacc = lane < WMAX ? (double)part[0] * my_inv : 0.0;
#pragma unroll
    for (int k = 0; k < WMAX; ++k) {
      const double zk = __shfl_sync(0xffffffffu, zacc, k);
      if (lane > k) zacc = fma(-srow[k], zk, zacc);
    }
    // the factor goes where the back substitutions read it
    if (lane < WMAX) {
      invd[lane] = my_inv;
#pragma unroll
      for (int j = 0; j < WMAX; ++j)
        if (j < lane) A[lane * kLda + j] = srow[j];
    }
    rhs[lane] = zacc;
    __syncwarp();
  } else {
    // Gram of the n vectors: pairs (i, j), j <= i < NV, enumerated row by row, 32
    // per round; after the reduce-scatter lane l holds pair (round base + l).
    float part[32];
    GramRows<NV, CPL, 0>::run(h, part, lane, wmax, a.lam, A, rhs);
    __syncwarp();
  }

  // Cholesky A = L L^T fused with the forward substitution L z = rhs.  Lane i
  // holds row i of A (then of L) and rhs_i (then z_i) in registers.  The chain
  // that bounds the loop is pivot -> 1/L_kk -> the next pivot: lane k+1 forms its
  // updated diagonal from its own entry L_{k+1,k} and sends it round by one
  // shuffle, ahead of the rest of the column update (whose entries L_jk go through
  // shared memory, one store per lane and one broadcast load per later column).
  double z = lane < wm ? rhs[lane] : 0.0;
  double* col = invd + 32;
  if constexpr (MODE != kPredUsing) {
    double arow[WMAX];
#pragma unroll
    for (int j = 0; j < WMAX; ++j) arow[j] = (j <= lane && lane < wm && j < wm) ? A[lane * kLda + j] : 0.0;
    double piv = __shfl_sync(0xffffffffu, arow[0], 0);
    double my_inv = 1.0;   // 1 / L_ii of this lane's row
#pragma unroll
    for (int k = 0; k < WMAX; ++k) {
      if (k < wm) {
        const double inv = rsqrt_f64(piv);   // 1 / L_kk
        const double lik = (lane > k && lane < wm) ? arow[k] * inv : 0.0;
        if (k + 1 < WMAX) {
          const double dn = fma(-lik, lik, arow[k + 1]);   // lane k+1: A_{k+1,k+1} - L_{k+1,k}^2
          piv = __shfl_sync(0xffffffffu, dn, k + 1);
        }
        const double zk = __shfl_sync(0xffffffffu, z, k) * inv;   // z_k
        if (lane == k) {
          my_inv = inv;
          invd[k] = inv;
          z = zk;
        } else if (lane > k) {
          arow[k] = lik;
          z = fma(-lik, zk, z);
        }
        col[lane] = lik;
        __syncwarp();
#pragma unroll
        for (int j = k + 1; j < WMAX; ++j) {
          const double ljk = col[j];
          if (j < wm && lane >= j && lane < wm) arow[j] = fma(-lik, ljk, arow[j]);
        }
        __syncwarp();   // the next column overwrites col
      }
    }
    // rows of L scaled by their own 1 / L_ii: the back substitutions then need one
    // multiply-add per step
    if (lane < wm) {
#pragma unroll
      for (int j = 0; j < WMAX; ++j)
        if (j < lane) A[lane * kLda + j] = arow[j] * my_inv;
    }
    if constexpr (MODE == kPredFactor) {
      double* fac = a.factor_out + (size_t)head * kFac;
      if (lane < WMAX) {
#pragma unroll
        for (int j = 0; j < WMAX; ++j)
          if (j < lane) fac[lane * WMAX + j] = arow[j] * my_inv;
        fac[WMAX * WMAX + lane] = my_inv;
      }
      return;
    }
  }
  __syncwarp();
  // Back substitutions L_w^T a = z_w for all windows at once: window wi owns the
  // lanes [base_wi, base_wi + w) (in rounds if the widths exceed 32).  With
  // y_k = z_k - sum_{j>k} L_jk a_j (complete once step k is reached) and
  // a_k = y_k / L_kk, lane i < k takes y_k from lane k and subtracts
  // (L_ki / L_kk) y_k.  The weights are folded into beta_r = sum_w alpha_{w,r},
  // so that qhat = (1/|windows|) sum_r beta_r q_{t-r}.
  double* beta = rhs;   // rhs is no longer needed: reuse it for beta
  if constexpr (!FAST) {
    beta[lane] = 0.0;
    __syncwarp();
  }
  int win[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) win[k] = a.windows[k];
  float bfast = 0.f;   // beta of lag `lane` on the fast path
  for (int first = 0; first < a.n_win;) {
    int last = first;   // windows [first, last) share this round
    int my_w = 0, my_base = 0, kmax = 0;
    if constexpr (FAST) {
      // one round holds every window; loops over a constant bound keep win[] in
      // registers
      last = a.n_win;
      int base = 0;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        if (k < last) {
          if (lane >= base && lane < base + win[k]) {
            my_w = win[k];
            my_base = base;
          }
          base += win[k];
          kmax = max(kmax, win[k]);
        }
      }
    } else {
      int used = 0;
      while (last < a.n_win && used + win[last] <= 32) used += win[last++];
      int base = 0;
      for (int k = first; k < last; ++k) {
        if (lane >= base && lane < base + win[k]) {
          my_w = win[k];
          my_base = base;
        }
        base += win[k];
        kmax = max(kmax, win[k]);
      }
    }
    const int li = lane - my_base;   // this lane's lag index in its window
    double av = (my_w > 0) ? __shfl_sync(0xffffffffu, z, li) : __shfl_sync(0xffffffffu, z, 0);
    if constexpr (WMAX <= 16) {
      // the lane's column of the scaled factor in registers, then a chain of
      // one shuffle and one multiply-add per step
      double lt[WMAX];
#pragma unroll
      for (int k = 0; k < WMAX; ++k) lt[k] = (li < k && k < my_w) ? A[k * kLda + li] : 0.0;
#pragma unroll
      for (int k = WMAX - 1; k >= 0; --k) {
        if (k < kmax) {
          const double yk = __shfl_sync(0xffffffffu, av, k < my_w ? my_base + k : lane);
          if (li < k && k < my_w) av = fma(-lt[k], yk, av);
        }
      }
    } else {
      for (int k = kmax - 1; k >= 0; --k) {
        const double yk = __shfl_sync(0xffffffffu, av, k < my_w ? my_base + k : lane);
        if (li < k && k < my_w) av = fma(-A[k * kLda + li], yk, av);
      }
    }
    if (my_w > 0) av *= invd[li];   // a_li
    if constexpr (FAST) {
      // Windows of 2^j lanes at multiples of their width: maxima and sums over a
      // window are xor butterflies, and lag r gathers its weights by shuffles.
      float w32 = my_w > 0 ? (float)av : 0.f;
      if (!a.coef_raw) {
        float m = my_w > 0 ? w32 : -INFINITY;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const float y = __shfl_xor_sync(0xffffffffu, m, o);
          if (o < my_w) m = fmaxf(m, y);
        }
        const float ex = my_w > 0 ? expf(w32 - m) : 0.f;
        float zs = ex;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const float y = __shfl_xor_sync(0xffffffffu, zs, o);
          if (o < my_w) zs += y;
        }
        w32 = my_w > 0 ? ex / zs : 0.f;
      }
      int bb = 0;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        if (k < last) {
          const float v = __shfl_sync(0xffffffffu, w32, bb + (lane < win[k] ? lane : 0));
          if (lane < win[k]) bfast += v;
          bb += win[k];
        }
      }
      first = last;
      continue;
    }
    // weights over each window's lags (softmax within the window unless raw)
    double wgt = av;
    if (!a.coef_raw) {   // one exp per lane; maxima and sums over the window through shared memory
      double* tmp = invd + 32;   // 32 spare doubles
      tmp[lane] = (my_w > 0) ? av : 0.0;
      __syncwarp();
      double m = -INFINITY;
      for (int r = 0; r < my_w; ++r) m = fmax(m, tmp[my_base + r]);
      const double e = (my_w > 0) ? (double)expf((float)(av - m)) : 0.0;
      __syncwarp();
      tmp[lane] = e;
      __syncwarp();
      double zs = 0.0;
      for (int r = 0; r < my_w; ++r) zs += tmp[my_base + r];
      wgt = (my_w > 0) ? e / zs : 0.0;
      __syncwarp();
    }
    // beta_r += weight of lag r in each window of the round
    double* tmp2 = invd + 32;
    tmp2[lane] = (my_w > 0) ? wgt : 0.0;
    __syncwarp();
    if (lane < WMAX) {
      double add = 0.0;
      int bb = 0;
      for (int k = first; k < last; ++k) {
        if (lane < win[k]) add += tmp2[bb + lane];
        bb += win[k];
      }
      beta[lane] += add;
    }
    __syncwarp();
    first = last;
  }
  float acc[CPL];
#pragma unroll
  for (int c = 0; c < CPL; ++c) acc[c] = 0.f;
  const float bl = lane < WMAX ? (FAST ? bfast : (float)beta[lane]) : 0.f;
#pragma unroll
  for (int r = 0; r < NV - 1; ++r) {   // lag r (q_{t-1-r}) weights q_{t-r} = h[r]
    const float br = __shfl_sync(0xffffffffu, bl, r);
#pragma unroll
    for (int c = 0; c < CPL; ++c) acc[c] = fmaf(br, h[r][c], acc[c]);
  }
  float* out = a.qpred + (size_t)head * D + lane * CPL;
  const float inv_nw = 1.f / (float)a.n_win;
#pragma unroll
  for (int c = 0; c < CPL; ++c) out[c] = acc[c] * inv_nw;
}


// ---- the recorded alternative reading of the pooling: regress on pooled features ----
//
// One warp per query head.  With h[v] = q_{t-v} (v = 0: the target q_t), window
// w's feature is the mean of its w most recent vectors, f_w(t) = mean(h[0..w-1]),
// and one step back f_w(t-1) = mean(h[1..w]).  The ridge fit of q_t on the
// features f_w(t-1) (samples = channels) is a k x k system (k windows, at most
// 8): the features are formed in fp64 in shared memory (each lane its own
// channels), the Gram and right-hand side reduced over the warp in fp64 and solved
// by lane 0 (Cholesky, fp64); the weights (softmax or raw) apply to f_w(t).
constexpr int kPoolMax = 8;

template <int D, int NV>
__global__ void __launch_bounds__(kWarps * 32) predict_pooled_kernel(PredictArgs a) {
  constexpr int CPL = D / 32;
  extern __shared__ __align__(16) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int head = blockIdx.x * kWarps + warp;
  pdl_trigger();
  if (a.zero) {   // clear the next kernel's histogram, as predict_kernel does
    const size_t n4 = a.zero_words / 4;
    int4* z4 = reinterpret_cast<int4*>(a.zero);
    for (size_t i = (size_t)head * 32 + lane; i < n4; i += (size_t)gridDim.x * kWarps * 32) z4[i] = make_int4(0, 0, 0, 0);
    for (size_t i = n4 * 4 + (size_t)head * 32 + lane; i < a.zero_words; i += (size_t)gridDim.x * kWarps * 32) a.zero[i] = 0;
  }
  if (head >= a.n_heads) return;
  // per warp: features [2][kPoolMax][D] (cur, prev), then the k x k Gram and rhs
  double* feat = reinterpret_cast<double*>(smem) + (size_t)warp * (2 * kPoolMax * D + kPoolMax * (kPoolMax + 1));
  double* G = feat + 2 * kPoolMax * D;
  double* rhs = G + kPoolMax * kPoolMax;
  const int k = a.n_win;
  const int n = a.wmax + 1;
  const int nslot = a.W + 1;
  float* hist = a.qhist + (size_t)head * nslot * D;
  const int start = a.q_new ? a.ring_start + 1 : a.ring_start;
  float h[NV][CPL];
#pragma unroll
  for (int v = 0; v < NV; ++v) {
#pragma unroll
    for (int c = 0; c < CPL; ++c) h[v][c] = 0.f;
    if (v < n) {
      int slot = start + a.W - v;
      if (slot >= nslot) slot -= nslot;
      if (v == 0 && a.q_new) {
        const size_t off = (size_t)head * D + lane * CPL;
#pragma unroll
        for (int c = 0; c < CPL; ++c)
          h[0][c] = a.q_new_f32 ? static_cast<const float*>(a.q_new)[off + c]
                                : __bfloat162float(static_cast<const __nv_bfloat16*>(a.q_new)[off + c]);
      } else {
#pragma unroll
        for (int c = 0; c < CPL; ++c) h[v][c] = hist[(size_t)slot * D + lane * CPL + c];
      }
    }
  }
  if (a.q_new) {   // push q_t into the ring: it replaces the oldest slot (ring_start)
#pragma unroll
    for (int c = 0; c < CPL; ++c) hist[(size_t)a.ring_start * D + lane * CPL + c] = h[0][c];
  }
  // features of this lane's channels
  for (int i = 0; i < k; ++i) {
    const int w = a.windows[i];
#pragma unroll
    for (int c = 0; c < CPL; ++c) {
      double cur = 0.0, prev = 0.0;
#pragma unroll
      for (int v = 0; v < NV; ++v) {
        if (v < w) cur += (double)h[v][c];
        if (v >= 1 && v <= w) prev += (double)h[v][c];
      }
      feat[(size_t)i * D + lane * CPL + c] = cur / w;
      feat[(size_t)(kPoolMax + i) * D + lane * CPL + c] = prev / w;
    }
  }
  __syncwarp();
  // Gram of the one-step-back features and the right-hand side, reduced over the warp
  for (int i = 0; i < k; ++i) {
    for (int j = 0; j <= i; ++j) {
      double part = 0.0;
#pragma unroll
      for (int c = 0; c < CPL; ++c)
        part += feat[(size_t)(kPoolMax + i) * D + lane * CPL + c] * feat[(size_t)(kPoolMax + j) * D + lane * CPL + c];
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
      if (lane == 0) G[i * kPoolMax + j] = part + (i == j ? a.lam : 0.0);
    }
    double part = 0.0;
#pragma unroll
    for (int c = 0; c < CPL; ++c) part += feat[(size_t)(kPoolMax + i) * D + lane * CPL + c] * (double)h[0][c];
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
    if (lane == 0) rhs[i] = part;
  }
  __syncwarp();
  if (lane == 0) {
    // Cholesky G = L L^T (lower triangle in place), then L z = rhs, L^T beta = z
    for (int j = 0; j < k; ++j) {
      double d = G[j * kPoolMax + j];
      for (int m = 0; m < j; ++m) d -= G[j * kPoolMax + m] * G[j * kPoolMax + m];
      const double ljj = sqrt(d);
      G[j * kPoolMax + j] = ljj;
      for (int i = j + 1; i < k; ++i) {
        double e = G[i * kPoolMax + j];
        for (int m = 0; m < j; ++m) e -= G[i * kPoolMax + m] * G[j * kPoolMax + m];
        G[i * kPoolMax + j] = e / ljj;
      }
    }
    for (int i = 0; i < k; ++i) {
      double e = rhs[i];
      for (int m = 0; m < i; ++m) e -= G[i * kPoolMax + m] * rhs[m];
      rhs[i] = e / G[i * kPoolMax + i];
    }
    for (int i = k - 1; i >= 0; --i) {
      double e = rhs[i];
      for (int m = i + 1; m < k; ++m) e -= G[m * kPoolMax + i] * rhs[m];
      rhs[i] = e / G[i * kPoolMax + i];
    }
    if (!a.coef_raw) {   // softmax over the k coefficients
      double mx = rhs[0];
      for (int i = 1; i < k; ++i) mx = fmax(mx, rhs[i]);
      double sum = 0.0;
      for (int i = 0; i < k; ++i) {
        rhs[i] = exp(rhs[i] - mx);
        sum += rhs[i];
      }
      for (int i = 0; i < k; ++i) rhs[i] /= sum;
    }
  }
  __syncwarp();
  float* out = a.qpred + (size_t)head * D + lane * CPL;
#pragma unroll
  for (int c = 0; c < CPL; ++c) {
    double acc = 0.0;
    for (int i = 0; i < k; ++i) acc += rhs[i] * feat[(size_t)i * D + lane * CPL + c];
    out[c] = (float)acc;
  }
}

template <int D, int NV>
cudaError_t launch_pooled_t(const PredictArgs& a, cudaStream_t s) {
  const int grid = (a.n_heads + kWarps - 1) / kWarps;
  const size_t smem = (size_t)kWarps * (2 * kPoolMax * D + kPoolMax * (kPoolMax + 1)) * sizeof(double);
  auto kern = predict_pooled_kernel<D, NV>;
  if (prepare_kernel((const void*)kern, smem, kWarps * 32) < 1) return cudaErrorInvalidConfiguration;
  return launch_prio(kern, dim3(grid), dim3(kWarps * 32), smem, s, a);
}

template <int D, int NV>
cudaError_t launch_t(const PredictArgs& a, cudaStream_t s) {
  if (a.pool_features) return launch_pooled_t<D, NV>(a, s);
  const int grid = (a.n_heads + kWarps - 1) / kWarps;
  const size_t smem = kWarps * Solve<NV>::kBytes;
  const bool exact = a.wmax == NV - 1;
  if (a.mode != kPredFull) {   // the decode loop's factor modes (see predict_factor_eligible)
    auto kern = a.mode == kPredFactor ? predict_kernel<D, NV, true, true, kPredFactor>
                                      : predict_kernel<D, NV, true, true, kPredUsing>;
    if (prepare_kernel((const void*)kern, smem, kWarps * 32) < 1) return cudaErrorInvalidConfiguration;
    return launch_prio(kern, dim3(grid), dim3(kWarps * 32), smem, s, a);
  }
  auto kern = a.win_fast ? (exact ? predict_kernel<D, NV, true, true> : predict_kernel<D, NV, true, false>)
                         : (exact ? predict_kernel<D, NV, false, true> : predict_kernel<D, NV, false, false>);
  if (prepare_kernel((const void*)kern, smem, kWarps * 32) < 1) return cudaErrorInvalidConfiguration;
  return launch_prio(kern, dim3(grid), dim3(kWarps * 32), smem, s, a);
}

template <int D>
cudaError_t launch_d(const PredictArgs& a, cudaStream_t s) {
  if (a.wmax + 1 <= 9) return launch_t<D, 9>(a, s);
  if (a.wmax + 1 <= 17) return launch_t<D, 17>(a, s);
  return launch_t<D, 33>(a, s);
}

}  // namespace

// Windows sorted widest first; whether they are powers of two filling at most one
// round of lanes.
static void sort_windows(PredictArgs& a) {
  for (int i = 1; i < a.n_win; ++i)
    for (int j = i; j > 0 && a.windows[j] > a.windows[j - 1]; --j) {
      const int t = a.windows[j];
      a.windows[j] = a.windows[j - 1];
      a.windows[j - 1] = t;
    }
  int sum = 0;
  bool pow2 = true;
  for (int i = 0; i < a.n_win; ++i) {
    sum += a.windows[i];
    pow2 = pow2 && a.windows[i] > 0 && (a.windows[i] & (a.windows[i] - 1)) == 0;
  }
  a.win_fast = (pow2 && sum <= 32) ? 1 : 0;
}

bool predict_factor_eligible(const PredictArgs& args) {
  PredictArgs a = args;
  sort_windows(a);
  const int nv = a.wmax + 1 <= 9 ? 9 : (a.wmax + 1 <= 17 ? 17 : 33);
  return !a.pool_features && a.win_fast && a.wmax == nv - 1;
}

size_t predict_factor_bytes(int n_heads, int wmax) {
  const int nv = wmax + 1 <= 9 ? 9 : (wmax + 1 <= 17 ? 17 : 33);
  return (size_t)n_heads * ((size_t)(nv - 1) * (nv - 1) + (nv - 1)) * sizeof(double);
}

cudaError_t launch_predict(const PredictArgs& args, cudaStream_t s) {
  // The mean over the windows does not depend on their order: sort them widest
  // first, so that windows whose widths are powers of two and add up to at most
  // 32 lanes each start at a multiple of their width.
  PredictArgs a = args;
  if (a.mode != kPredFull && !predict_factor_eligible(a)) {
    if (a.mode == kPredFactor) return cudaSuccess;   // nothing to precompute
    a.mode = kPredFull;
  }
  sort_windows(a);
  return a.head_dim == 64 ? launch_d<64>(a, s) : launch_d<128>(a, s);
}

ASP_STATUS_READER(read_status_predict)

}  // namespace asp
