// asp_attend.cu -- step 4: single-token attention over the selected K/V rows.
//
// out[b, hq] = sum_{j in S} softmax_j(q . k_j / sqrt(d)) v_j over S = selected u tail.
//
// HBM-bound gather (each selected K and V row read once, 256 B for bf16 d=128).
//  * work items (split, batch * n_kv): a CTA takes a contiguous slice of one KV
//    head's attended rows and computes all G query heads of the group, so a row
//    is read once for the whole group;
//  * a warp gathers 16 rows per tile (K and V) into its stage, counted on one
//    mbarrier, with STAGES tiles in flight per warp: the CUDA-core kernel (fp32)
//    by one 1-D bulk copy (TMA) per lane, the tensor-core kernel (bf16) by
//    16-byte cp.async copies, several rows per warp instruction;
//  * logits: 16-byte shared-memory vectors per lane, packed FMAs, warp
//    reduce-scatter over the row's lanes; online softmax in base 2 (log2 e folded
//    into the query scale); V accumulated in fp32 registers;
//  * warps of a CTA merge through shared memory; with several splits the partial
//    (max, sum, unnormalised output) go to the workspace and a small kernel does
//    the log-sum-exp merge.
#include <cfloat>
#include <mutex>

#include "asp_common.cuh"
#include "asp_internal.h"

namespace asp {
namespace {

constexpr int kTile = 16;
constexpr int kWarps = 4;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

struct AttParams {
  const void* q;
  int q_f32;
  int n_q_heads;
  const uint8_t* k;
  const uint8_t* v;
  int batch, n_kv, t_max, page_size, max_pages, n_pages;
  const int32_t* page_table;
  const int32_t* seq_lens;
  const int32_t* idx;
  const int32_t* count;
  int C;
  const int32_t* tail_begin;
  int max_tail;
  int splits, rows_per_split;
  int n_items;   // units * splits: the persistent kernel's work items
  int lean;      // launch the kernel form with fewer registers
  int ctas;      // its grid
  float* part_o;
  float* part_ml;
  void* out;
  float* lse;
  float qscale;   // log2(e) / sqrt(d)
};

template <typename KT, int D, int G, int STAGES>
__global__ void __launch_bounds__(kWarps * 32) attend_kernel(AttParams p) {
  using E = Elem<KT>;
  constexpr int ROW_BYTES = D * E::kBytes;
  constexpr int LPR = ROW_BYTES / 16;
  constexpr int RPS = 32 / LPR;
  constexpr int CPL = E::kPerVec;
  constexpr int NSTEP = kTile / RPS;
  constexpr int TILE_BYTES = 2 * kTile * ROW_BYTES;
  constexpr int SPP = (NSTEP * G <= 32) ? NSTEP : (32 / G);
  constexpr int NPASS = NSTEP / SPP;
  constexpr int NV = SPP * G;
  constexpr int LPG = 32 / G;                         // lanes per head in the softmax stage
  constexpr int RPL = (kTile + LPG - 1) / LPG;        // tile rows per lane in the softmax stage
  static_assert(LPR >= 2 && 32 % LPR == 0 && NV <= 32 && G * LPR >= NV, "layout");

  extern __shared__ __align__(128) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint8_t* wbuf = smem + (size_t)warp * STAGES * TILE_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (size_t)kWarps * STAGES * TILE_BYTES) + warp * STAGES;
  float* lg = reinterpret_cast<float*>(smem + (size_t)kWarps * STAGES * TILE_BYTES + kWarps * STAGES * 8) +
              warp * (kTile * G + G);
  float* cs = lg + kTile * G;

  const int unit = blockIdx.y, split = blockIdx.x;
  const int b = unit / p.n_kv, h = unit - b * p.n_kv;
  int T = p.seq_lens ? p.seq_lens[b] : p.t_max;
  T = T < 0 ? 0 : (T > p.t_max ? p.t_max : T);
  int n_sel = (p.C > 0 && p.count) ? p.count[unit] : 0;
  n_sel = n_sel < 0 ? 0 : (n_sel > p.C ? p.C : n_sel);
  int tb = T;
  if (p.tail_begin) {
    tb = p.tail_begin[b];
    tb = tb < 0 ? 0 : (tb > T ? T : tb);
  }
  int tail = T - tb;
  if (tail > p.max_tail) {
    if (threadIdx.x == 0 && split == 0) flag_status(ASP_DEV_TAIL_LIMIT);
    tail = p.max_tail;
  }
  const int n_rows = n_sel + tail;
  const int r0 = split * p.rows_per_split;
  const int r1 = min(n_rows, r0 + p.rows_per_split);
  const int n_tiles = r1 > r0 ? (r1 - r0 + kTile - 1) / kTile : 0;
  const int32_t* idx_row = n_sel ? p.idx + (size_t)unit * p.C : nullptr;

  if (lane == 0) {
    for (int s = 0; s < STAGES; ++s) mbar_init(&bars[s], 1);
    mbar_init_fence();
  }
  __syncwarp();

  // query of the G heads, scaled by log2(e)/sqrt(d)
  float2 q2[G][CPL / 2];
  {
    const int c0 = (lane % LPR) * CPL;
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const size_t off = (size_t)(b * p.n_q_heads + h * G + g) * D + c0;
#pragma unroll
      for (int c = 0; c < CPL / 2; ++c) {
        float x0, x1;
        if (p.q_f32) {
          const float2 x = *reinterpret_cast<const float2*>(static_cast<const float*>(p.q) + off + 2 * c);
          x0 = x.x;
          x1 = x.y;
        } else {
          const __nv_bfloat162 x = *reinterpret_cast<const __nv_bfloat162*>(static_cast<const __nv_bfloat16*>(p.q) + off + 2 * c);
          x0 = __low2float(x);
          x1 = __high2float(x);
        }
        q2[g][c] = make_float2(x0 * p.qscale, x1 * p.qscale);
      }
    }
  }

  // tile t of this warp covers rows r0 + (warp + t * kWarps) * kTile + [0, 16)
  const int my_tiles = n_tiles > warp ? (n_tiles - warp + kWarps - 1) / kWarps : 0;

  // Row source of this lane for tile t (lanes 0-15: K rows, 16-31: V rows).  The
  // index and page-table loads of the next tile are issued one tile ahead, so
  // their latency hides behind the current tile's compute.
  struct RowSrc {
    const uint8_t* src;
    bool valid;
  };
  auto resolve = [&](int t) -> RowSrc {
    const int rr = lane & 15;
    const bool isv = lane >= 16;
    const int r = r0 + (warp + t * kWarps) * kTile + rr;
    bool valid = r < r1;
    int j = 0;
    if (valid) {
      if (r < n_sel) {
        j = idx_row[r];
        if (j < 0 || j >= T) {
          valid = false;
          if (!isv) flag_status(ASP_DEV_BAD_INDEX);
        } else if (j >= tb) {
          valid = false;   // covered by the tail
        }
      } else {
        j = tb + (r - n_sel);
      }
    }
    const uint8_t* src = nullptr;
    if (valid) {
      const uint8_t* base = isv ? p.v : p.k;
      if (p.page_size == 0) {
        src = base + ((size_t)unit * p.t_max + j) * ROW_BYTES;
      } else {
        const int page = p.page_table[(size_t)b * p.max_pages + j / p.page_size];
        if (page < 0 || page >= p.n_pages) {
          valid = false;
          if (!isv) flag_status(ASP_DEV_BAD_PAGE);
        } else {
          src = base + (((size_t)page * p.n_kv + h) * p.page_size + (j % p.page_size)) * ROW_BYTES;
        }
      }
    }
    return RowSrc{src, valid};
  };
  // Gathers one tile into a stage: one bulk copy per valid row, rows with no
  // source zero-filled; returns the tile's valid-row mask.
  auto issue = [&](const RowSrc& rs, int slot) -> uint32_t {
    const int rr = lane & 15;
    const bool isv = lane >= 16;
    const uint32_t vm = __ballot_sync(0xffffffffu, rs.valid) & 0xffffu;
    uint8_t* dst = wbuf + slot * TILE_BYTES + (isv ? kTile * ROW_BYTES : 0) + rr * ROW_BYTES;
    if (!rs.valid) {
#pragma unroll
      for (int c = 0; c < ROW_BYTES / 16; ++c) reinterpret_cast<uint4*>(dst)[c] = make_uint4(0, 0, 0, 0);
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive_expect_tx(&bars[slot], (uint32_t)__popc(vm) * 2u * ROW_BYTES);
    __syncwarp();
    if (rs.valid) bulk_g2s(dst, rs.src, ROW_BYTES, &bars[slot]);
    return vm;
  };

  float2 o2[G][CPL / 2];
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int c = 0; c < CPL / 2; ++c) o2[g][c] = make_float2(0.f, 0.f);
  float m_run = -INFINITY;   // running max (base 2) of head lane % G
  float l_run = 0.f;         // this lane's share of the running sum of head lane % G

  uint32_t vmask[STAGES];
  int issued = 0;
#pragma unroll 1
  for (int s = 0; s < STAGES && s < my_tiles; ++s) {
    vmask[s] = issue(resolve(s), s);
    ++issued;
  }
  RowSrc next = issued < my_tiles ? resolve(issued) : RowSrc{nullptr, false};

  int consumed = 0;
  bool ok = true;
#pragma unroll 1
  for (int t = 0; t < my_tiles; ++t) {
    const int slot = t % STAGES;
    ok = __all_sync(0xffffffffu, mbar_wait(&bars[slot], (uint32_t)(t / STAGES) & 1u));
    if (!ok) break;
    ++consumed;
    const uint32_t vm = vmask[slot];
    const uint8_t* kb = wbuf + slot * TILE_BYTES;
    const uint8_t* vb = kb + kTile * ROW_BYTES;

    // 1. logits (base 2) of the 16 rows x G heads -> lg[row][g]
#pragma unroll
    for (int pass = 0; pass < NPASS; ++pass) {
      float vals[NV];
#pragma unroll
      for (int s = 0; s < SPP; ++s) {
        const int row = (pass * SPP + s) * RPS + lane / LPR;
        const uint4 v = *reinterpret_cast<const uint4*>(kb + row * ROW_BYTES + (lane % LPR) * 16);
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
      const int l = lane % LPR;
      if constexpr (NV >= LPR) {
        constexpr int VPL = NV / LPR;
#pragma unroll
        for (int i = 0; i < VPL; ++i) {
          const int pidx = VPL * l + i;
          const int row = (pass * SPP + pidx / G) * RPS + lane / LPR;
          lg[row * G + pidx % G] = vals[i];
        }
      } else {
        const int pidx = l / (LPR / NV);
        const int row = (pass * SPP + pidx / G) * RPS + lane / LPR;
        lg[row * G + pidx % G] = vals[0];
      }
    }
    __syncwarp();

    // 2. online softmax statistics; probabilities overwrite the logits
    {
      const int g = lane % G, rl = lane / G;
      float x[RPL];
      float mloc = -INFINITY;
#pragma unroll
      for (int k = 0; k < RPL; ++k) {
        const int row = rl + k * LPG;
        x[k] = (row < kTile && ((vm >> row) & 1u)) ? lg[row * G + g] : -INFINITY;
        mloc = fmaxf(mloc, x[k]);
      }
#pragma unroll
      for (int o = G; o < 32; o <<= 1) mloc = fmaxf(mloc, __shfl_xor_sync(0xffffffffu, mloc, o));
      const float m_new = fmaxf(m_run, mloc);
      const float corr = (m_new == -INFINITY) ? 1.f : ex2(m_run - m_new);
      float psum = 0.f;
#pragma unroll
      for (int k = 0; k < RPL; ++k) {
        const int row = rl + k * LPG;
        const float pr = (x[k] == -INFINITY) ? 0.f : ex2(x[k] - m_new);
        if (row < kTile) lg[row * G + g] = pr;
        psum += pr;
      }
      l_run = l_run * corr + psum;
      m_run = m_new;
      if (lane < G) cs[lane] = corr;
    }
    __syncwarp();

    // 3. rescale and accumulate V
    {
      bool any = false;
      float cr[G];
#pragma unroll
      for (int g = 0; g < G; ++g) {
        cr[g] = cs[g];
        any |= cr[g] != 1.f;
      }
      if (any) {
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
          for (int c = 0; c < CPL / 2; ++c) o2[g][c] = __fmul2_rn(o2[g][c], make_float2(cr[g], cr[g]));
      }
#pragma unroll
      for (int s = 0; s < NSTEP; ++s) {
        const int row = s * RPS + lane / LPR;
        const uint4 v = *reinterpret_cast<const uint4*>(vb + row * ROW_BYTES + (lane % LPR) * 16);
        float2 vf[CPL / 2];
        E::unpack(v, vf);
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float pr = lg[row * G + g];
          const float2 pp = make_float2(pr, pr);
#pragma unroll
          for (int c = 0; c < CPL / 2; ++c) o2[g][c] = __ffma2_rn(vf[c], pp, o2[g][c]);
        }
      }
    }
    __syncwarp();
    if (issued < my_tiles) {
      vmask[slot] = issue(next, slot);
      ++issued;
      if (issued < my_tiles) next = resolve(issued);
    }
  }
  if (!ok) {
    for (int k = consumed + 1; k < issued; ++k) mbar_wait(&bars[k % STAGES], (uint32_t)(k / STAGES) & 1u);
  }

  // combine within the warp: V partials over the row groups, sums over the lanes of a head
#pragma unroll
  for (int o = LPR; o < 32; o <<= 1)
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
      for (int c = 0; c < CPL / 2; ++c) {
        o2[g][c].x += __shfl_xor_sync(0xffffffffu, o2[g][c].x, o);
        o2[g][c].y += __shfl_xor_sync(0xffffffffu, o2[g][c].y, o);
      }
#pragma unroll
  for (int o = G; o < 32; o <<= 1) l_run += __shfl_xor_sync(0xffffffffu, l_run, o);

  // combine the warps (shared memory reused from the stages)
  __syncthreads();
  float* mo = reinterpret_cast<float*>(smem);   // [kWarps][G][D] outputs, then [kWarps][G][2] (m, l)
  float* mml = mo + kWarps * G * D;
  if (lane < LPR) {
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
      for (int c = 0; c < CPL / 2; ++c)
        *reinterpret_cast<float2*>(mo + (warp * G + g) * D + lane * CPL + 2 * c) = o2[g][c];
  }
  if (lane < G) {
    mml[(warp * G + lane) * 2 + 0] = m_run;
    mml[(warp * G + lane) * 2 + 1] = l_run;
  }
  __syncthreads();
  for (int e = threadIdx.x; e < G * D; e += kWarps * 32) {
    const int g = e / D, c = e - g * D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, mml[(w * G + g) * 2]);
    float L = 0.f, O = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        const float mw = mml[(w * G + g) * 2];
        if (mw == -INFINITY) continue;
        const float f = ex2(mw - M);
        L += mml[(w * G + g) * 2 + 1] * f;
        O += mo[(w * G + g) * D + c] * f;
      }
    }
    const int hq = h * G + g;
    const size_t bh = (size_t)b * p.n_q_heads + hq;
    if (p.splits == 1) {
      const float r = L > 0.f ? O / L : 0.f;
      static_cast<KT*>(p.out)[bh * D + c] = E::from_float(r);
      if (c == 0 && p.lse) p.lse[bh] = L > 0.f ? (M + __log2f(L)) * kLn2 : -INFINITY;
    } else {
      p.part_o[(bh * p.splits + split) * D + c] = O;
      if (c == 0) {
        p.part_ml[(bh * p.splits + split) * 2 + 0] = M;
        p.part_ml[(bh * p.splits + split) * 2 + 1] = L;
      }
    }
  }
}

// ---- bf16 cache with a bf16 query: both small contractions on tensor cores ----
//
// Per 16-row tile a warp computes S^T[head x row] = Q[head x d] . K^T with
// mma.m16n8k16 (M = query heads, G <= 8 of the 16 rows used; N = 8 rows per
// n-tile; K = 16 channels), takes the online softmax in fp32, splits the
// probabilities into bf16 hi and lo parts and accumulates O[head x d] +=
// P[head x row] . V with two more mmas (K = the 16 rows); the accumulator
// layout of the logits is the operand layout of P.  The query and the cache are
// bf16, so every product is exact and only fp32 summation order differs from a
// CUDA-core dot product.  K and V rows sit in shared memory at a 16-byte padded
// stride, so the eight rows an ldmatrix phase reads fall in distinct banks.

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

// d01 += A . B on the top 8 rows of a 16x8 tile; the A rows 8-15 are zero, so
// their accumulators are not kept.  a0: (row g, k 2t..2t+1), a2: (row g, k
// 8+2t..9+2t); b0: (k 2t..2t+1, col g), b1: (k 8+2t..9+2t, col g).
__device__ __forceinline__ void mma_top8(float& d0, float& d1, uint32_t a0, uint32_t a2, uint32_t b0, uint32_t b1) {
  float x2, x3;
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%10, %11, %12, %13};"
      : "=f"(d0), "=f"(d1), "=f"(x2), "=f"(x3)
      : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1), "f"(d0), "f"(d1), "f"(0.f), "f"(0.f));
}

// (x0, x1) -> hi = bf16 pair rn(x), lo = bf16 pair rn(x - hi); x0 in the low half.
__device__ __forceinline__ void split_bf16x2(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
  const float2 hf = __bfloat1622float2(h);
  const __nv_bfloat162 l = __floats2bfloat162_rn(x0 - hf.x, x1 - hf.y);
  hi = *reinterpret_cast<const uint32_t*>(&h);
  lo = *reinterpret_cast<const uint32_t*>(&l);
}

// LEAN: the row copies are issued from a partly unrolled loop, which keeps the
// registers at the level that lets one CTA share an SM with the key scan's and the
// predictor's (the decode step); the fully unrolled form keeps more copies in
// flight where three CTAs share an SM (stand-alone calls).
template <int D, int G, int STAGES, bool LEAN>
__global__ void __launch_bounds__(kWarps * 32) attend_mma_kernel(AttParams p) {
  constexpr int ROW_BYTES = D * 2;
  constexpr int STRIDE = ROW_BYTES + 16;          // padded row pitch in shared memory
  constexpr int HALF = kTile * STRIDE;            // the K (or V) rows of one stage
  constexpr int TILE_BYTES = 2 * HALF;
  constexpr int KS = D / 16;                      // k-steps of the logits
  constexpr int NT = D / 8;                       // n-tiles of the output
  static_assert(G >= 1 && G <= 8 && kTile == 16, "layout");

  extern __shared__ __align__(128) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;          // fragment row (query head) and column pair
  uint8_t* wbuf = smem + (size_t)warp * STAGES * TILE_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (size_t)kWarps * STAGES * TILE_BYTES) + warp * STAGES;
  if (lane == 0) {
    for (int s = 0; s < STAGES; ++s) mbar_init(&bars[s], 32);   // one arrival per lane's copies
    mbar_init_fence();
  }
  __syncwarp();

  // A persistent grid: each CTA takes work items (unit, split) in turn; the stage
  // barriers' phases run on over the items (tbase: this warp's tiles so far).
  uint32_t tbase = 0;
  for (int item = blockIdx.x; item < p.n_items; item += gridDim.x) {
  const int unit = item / p.splits, split = item - unit * p.splits;
  const int b = unit / p.n_kv, h = unit - b * p.n_kv;
  int T = p.seq_lens ? p.seq_lens[b] : p.t_max;
  T = T < 0 ? 0 : (T > p.t_max ? p.t_max : T);
  int n_sel = (p.C > 0 && p.count) ? p.count[unit] : 0;
  n_sel = n_sel < 0 ? 0 : (n_sel > p.C ? p.C : n_sel);
  int tb = T;
  if (p.tail_begin) {
    tb = p.tail_begin[b];
    tb = tb < 0 ? 0 : (tb > T ? T : tb);
  }
  int tail = T - tb;
  if (tail > p.max_tail) {
    if (threadIdx.x == 0 && split == 0) flag_status(ASP_DEV_TAIL_LIMIT);
    tail = p.max_tail;
  }
  const int n_rows = n_sel + tail;
  const int r0 = split * p.rows_per_split;
  const int r1 = min(n_rows, r0 + p.rows_per_split);
  const int n_tiles = r1 > r0 ? (r1 - r0 + kTile - 1) / kTile : 0;
  const int32_t* idx_row = n_sel ? p.idx + (size_t)unit * p.C : nullptr;

  // query fragments: head g (zero rows for g >= G), channels 16kk + 2t (+8)
  uint32_t qa[KS][2];
  {
    const __nv_bfloat16* qrow =
        static_cast<const __nv_bfloat16*>(p.q) + (size_t)(b * p.n_q_heads + h * G + (g < G ? g : 0)) * D;
#pragma unroll
    for (int kk = 0; kk < KS; ++kk) {
      qa[kk][0] = g < G ? *reinterpret_cast<const uint32_t*>(qrow + 16 * kk + 2 * t) : 0u;
      qa[kk][1] = g < G ? *reinterpret_cast<const uint32_t*>(qrow + 16 * kk + 8 + 2 * t) : 0u;
    }
  }

  const int my_tiles = n_tiles > warp ? (n_tiles - warp + kWarps - 1) / kWarps : 0;

  struct RowSrc {
    const uint8_t* src;
    bool valid;
  };
  // Row source of this lane for tile t (lanes 0-15: K rows, 16-31: V rows).
  auto resolve = [&](int tt) -> RowSrc {
    const int rr = lane & 15;
    const bool isv = lane >= 16;
    const int r = r0 + (warp + tt * kWarps) * kTile + rr;
    bool valid = r < r1;
    int j = 0;
    if (valid) {
      if (r < n_sel) {
        j = idx_row[r];
        if (j < 0 || j >= T) {
          valid = false;
          if (!isv) flag_status(ASP_DEV_BAD_INDEX);
        } else if (j >= tb) {
          valid = false;   // covered by the tail
        }
      } else {
        j = tb + (r - n_sel);
      }
    }
    const uint8_t* src = nullptr;
    if (valid) {
      const uint8_t* base = isv ? p.v : p.k;
      if (p.page_size == 0) {
        src = base + ((size_t)unit * p.t_max + j) * ROW_BYTES;
      } else {
        const int page = p.page_table[(size_t)b * p.max_pages + j / p.page_size];
        if (page < 0 || page >= p.n_pages) {
          valid = false;
          if (!isv) flag_status(ASP_DEV_BAD_PAGE);
        } else {
          src = base + (((size_t)page * p.n_kv + h) * p.page_size + (j % p.page_size)) * ROW_BYTES;
        }
      }
    }
    return RowSrc{src, valid};
  };
  // The tile's 32 rows go in as 16-byte copies, several rows per warp instruction
  // (chunk lane%CPR of row RPI*i + lane/CPR): a row-sized bulk copy per lane kept
  // too few bytes in flight per SM.  Rows that are not valid are zero-filled
  // (source size 0, nothing is read).  Each lane's copies arrive once on the
  // stage's barrier (count 32).
  auto issue = [&](const RowSrc& rs, int slot) -> uint32_t {
    constexpr int CPR = ROW_BYTES / 16;   // 16-byte chunks per row: 16 (d 128) or 8 (d 64)
    constexpr int RPI = 32 / CPR;          // rows per warp instruction
    const uint32_t vm = __ballot_sync(0xffffffffu, rs.valid) & 0xffffu;
    uint8_t* const tile = wbuf + slot * TILE_BYTES;
    const uint32_t c16 = (uint32_t)(lane % CPR) * 16u;
    auto copy_rows = [&](int i) {   // warp instruction i: rows RPI*i .. RPI*i + RPI - 1
      const int ri = RPI * i + lane / CPR;   // 0-15 K rows, 16-31 V rows (row ri is resolved by lane ri)
      const uint64_t src = __shfl_sync(0xffffffffu, reinterpret_cast<uint64_t>(rs.src), ri);
      const int valid = __shfl_sync(0xffffffffu, rs.valid ? 1 : 0, ri);
      const uint32_t dst = smem_u32(tile + (ri < 16 ? 0 : HALF) + (ri & 15) * STRIDE) + c16;
      const uint64_t from = valid ? src + c16 : reinterpret_cast<uint64_t>(p.k);
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(from), "r"(valid ? 16 : 0)
                   : "memory");
    };
    if constexpr (LEAN) {
#pragma unroll 2
      for (int i = 0; i < 32 / RPI; ++i) copy_rows(i);
    } else {
#pragma unroll
      for (int i = 0; i < 32 / RPI; ++i) copy_rows(i);
    }
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(&bars[slot])) : "memory");
    return vm;
  };

  float o[NT][2];
#pragma unroll
  for (int n = 0; n < NT; ++n) o[n][0] = o[n][1] = 0.f;
  float m_run = -INFINITY;   // running max (base 2) of head g
  float l_run = 0.f;         // this lane's share of head g's running sum

  // ldmatrix row addresses (byte offsets in a stage): lane l feeds row l & 7 of
  // matrix l >> 3
  const int mat = lane >> 3, mrow = lane & 7;
  const uint32_t k_off = (uint32_t)(((mat >> 1) * 8 + mrow) * STRIDE + (mat & 1) * 16);        // + 32 kk
  const uint32_t v_off = (uint32_t)(HALF + ((mat & 1) * 8 + mrow) * STRIDE + (mat >> 1) * 16);  // + 32 j

  uint32_t vmask[STAGES];
  int issued = 0;
#pragma unroll 1
  for (int s = 0; s < STAGES && s < my_tiles; ++s) {
    const int sl = (int)((tbase + s) % STAGES);
    vmask[sl] = issue(resolve(s), sl);
    ++issued;
  }
  RowSrc next = issued < my_tiles ? resolve(issued) : RowSrc{nullptr, false};

  int consumed = 0;
  bool ok = true;
#pragma unroll 1
  for (int tt = 0; tt < my_tiles; ++tt) {
    const int slot = (int)((tbase + tt) % STAGES);
    ok = __all_sync(0xffffffffu, mbar_wait(&bars[slot], (uint32_t)((tbase + tt) / STAGES) & 1u));
    if (!ok) break;
    ++consumed;
    const uint32_t vm = vmask[slot];
    const uint32_t base = smem_u32(wbuf + slot * TILE_BYTES);

    // 1. logits: n-tile 0 = rows 0-7, n-tile 1 = rows 8-15
    float s0[2] = {0.f, 0.f}, s1[2] = {0.f, 0.f};
#pragma unroll
    for (int kk = 0; kk < KS; ++kk) {
      uint32_t kb[4];
      ldsm_x4(kb, base + k_off + 32 * kk);
      mma_top8(s0[0], s0[1], qa[kk][0], qa[kk][1], kb[0], kb[1]);
      mma_top8(s1[0], s1[1], qa[kk][0], qa[kk][1], kb[2], kb[3]);
    }

    // 2. online softmax of head g over its 16 rows (4 per lane, 4 lanes per head)
    float x[4] = {s0[0] * p.qscale, s0[1] * p.qscale, s1[0] * p.qscale, s1[1] * p.qscale};
    const int rows[4] = {2 * t, 2 * t + 1, 8 + 2 * t, 9 + 2 * t};
    float mloc = -INFINITY;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if (!((vm >> rows[e]) & 1u)) x[e] = -INFINITY;
      mloc = fmaxf(mloc, x[e]);
    }
    mloc = fmaxf(mloc, __shfl_xor_sync(0xffffffffu, mloc, 1));
    mloc = fmaxf(mloc, __shfl_xor_sync(0xffffffffu, mloc, 2));
    const float m_new = fmaxf(m_run, mloc);
    const float corr = (m_new == -INFINITY) ? 1.f : ex2(m_run - m_new);
    float pr[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) pr[e] = (x[e] == -INFINITY) ? 0.f : ex2(x[e] - m_new);
    l_run = l_run * corr + ((pr[0] + pr[1]) + (pr[2] + pr[3]));
    m_run = m_new;
    // P as bf16 hi + lo parts: the products with bf16 V are exact in fp32, so
    // the weights keep ~16 significant bits
    uint32_t pa0, pa2, pl0, pl2;
    split_bf16x2(pr[0], pr[1], pa0, pl0);
    split_bf16x2(pr[2], pr[3], pa2, pl2);

    // 3. O = O * corr + P . V
    if (corr != 1.f) {
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        o[n][0] *= corr;
        o[n][1] *= corr;
      }
    }
#pragma unroll
    for (int j = 0; j < D / 16; ++j) {
      uint32_t vb[4];
      ldsm_x4_trans(vb, base + v_off + 32 * j);
      mma_top8(o[2 * j][0], o[2 * j][1], pa0, pa2, vb[0], vb[1]);
      mma_top8(o[2 * j + 1][0], o[2 * j + 1][1], pa0, pa2, vb[2], vb[3]);
      mma_top8(o[2 * j][0], o[2 * j][1], pl0, pl2, vb[0], vb[1]);
      mma_top8(o[2 * j + 1][0], o[2 * j + 1][1], pl0, pl2, vb[2], vb[3]);
    }
    __syncwarp();
    if (issued < my_tiles) {
      vmask[slot] = issue(next, slot);
      ++issued;
      if (issued < my_tiles) next = resolve(issued);
    }
  }
  if (!ok) {
    for (int k = consumed + 1; k < issued; ++k)
      mbar_wait(&bars[(tbase + k) % STAGES], (uint32_t)((tbase + k) / STAGES) & 1u);
  }
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 1);
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 2);

  // combine the warps (shared memory reused from the stages)
  __syncthreads();
  float* mo = reinterpret_cast<float*>(smem);   // [kWarps][G][D] outputs, then [kWarps][G][2] (m, l)
  float* mml = mo + kWarps * G * D;
  if (g < G) {
#pragma unroll
    for (int n = 0; n < NT; ++n)
      *reinterpret_cast<float2*>(mo + (warp * G + g) * D + n * 8 + 2 * t) = make_float2(o[n][0], o[n][1]);
    if (t == 0) {
      mml[(warp * G + g) * 2 + 0] = m_run;
      mml[(warp * G + g) * 2 + 1] = l_run;
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < G * D; e += kWarps * 32) {
    const int gg = e / D, c = e - gg * D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, mml[(w * G + gg) * 2]);
    float L = 0.f, O = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        const float mw = mml[(w * G + gg) * 2];
        if (mw == -INFINITY) continue;
        const float f = ex2(mw - M);
        L += mml[(w * G + gg) * 2 + 1] * f;
        O += mo[(w * G + gg) * D + c] * f;
      }
    }
    const size_t bh = (size_t)b * p.n_q_heads + h * G + gg;
    if (p.splits == 1) {
      const float r = L > 0.f ? O / L : 0.f;
      static_cast<__nv_bfloat16*>(p.out)[bh * D + c] = __float2bfloat16_rn(r);
      if (c == 0 && p.lse) p.lse[bh] = L > 0.f ? (M + __log2f(L)) * kLn2 : -INFINITY;
    } else {
      p.part_o[(bh * p.splits + split) * D + c] = O;
      if (c == 0) {
        p.part_ml[(bh * p.splits + split) * 2 + 0] = M;
        p.part_ml[(bh * p.splits + split) * 2 + 1] = L;
      }
    }
  }
  // the next item's copies overwrite the merge area: generic accesses first
  fence_proxy_async_smem();
  tbase += (uint32_t)my_tiles;
  if (__syncthreads_or(!ok)) break;   // a wait ran out: stop (the copies have drained)
  }
}

// Log-sum-exp merge of the split partials: one CTA of D threads per query head.
template <typename KT, int D>
__global__ void __launch_bounds__(D) attend_merge_kernel(const float* __restrict__ part_o,
                                                         const float* __restrict__ part_ml, int splits, void* out,
                                                         float* lse) {
  using E = Elem<KT>;
  const size_t bh = blockIdx.x;
  const int c = threadIdx.x;
  pdl_wait();   // the split partials come from the previous kernel
  const float* ml = part_ml + bh * splits * 2;
  float M = -INFINITY;
  for (int s = 0; s < splits; ++s) M = fmaxf(M, ml[2 * s]);
  float L = 0.f, O = 0.f;
  if (M != -INFINITY) {
    for (int s = 0; s < splits; ++s) {
      const float ms = ml[2 * s];
      if (ms == -INFINITY) continue;
      const float f = ex2(ms - M);
      L += ml[2 * s + 1] * f;
      O += part_o[(bh * splits + s) * D + c] * f;
    }
  }
  static_cast<KT*>(out)[bh * D + c] = E::from_float(L > 0.f ? O / L : 0.f);
  if (c == 0 && lse) lse[bh] = L > 0.f ? (M + __log2f(L)) * kLn2 : -INFINITY;
}

template <typename KT, int D, int G>
cudaError_t launch_t(const AttParams& p, cudaStream_t s) {
  constexpr int ROW_BYTES = D * Elem<KT>::kBytes;
  constexpr int TILE_BYTES = 2 * kTile * ROW_BYTES;
  constexpr int STAGES = 2;
  auto kern = attend_kernel<KT, D, G, STAGES>;
  size_t smem = (size_t)kWarps * STAGES * TILE_BYTES + kWarps * STAGES * 8 + (size_t)kWarps * (kTile * G + G) * 4;
  const size_t merge = (size_t)kWarps * G * (D + 2) * 4;
  if (smem < merge) smem = merge;
  if (prepare_kernel((const void*)kern, smem, kWarps * 32) < 1) return cudaErrorInvalidConfiguration;
  kern<<<dim3(p.splits, p.batch * p.n_kv), kWarps * 32, smem, s>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || p.splits == 1) return e;
  return launch_pdl(attend_merge_kernel<KT, D>, dim3(p.batch * p.n_q_heads), dim3(D), 0, s, (const float*)p.part_o,
                    (const float*)p.part_ml, p.splits, p.out, p.lse);
}

template <int D, int G>
cudaError_t launch_mma(const AttParams& p, cudaStream_t s) {
  constexpr int STAGES = 2;
  constexpr int TILE_BYTES = 2 * kTile * (D * 2 + 16);
  auto kern = p.lean ? attend_mma_kernel<D, G, STAGES, true> : attend_mma_kernel<D, G, STAGES, false>;
  size_t smem = (size_t)kWarps * STAGES * TILE_BYTES + kWarps * STAGES * 8;
  const size_t merge = (size_t)kWarps * G * (D + 2) * 4;
  if (smem < merge) smem = merge;
  if (prepare_kernel((const void*)kern, smem, kWarps * 32) < 1) return cudaErrorInvalidConfiguration;
  kern<<<dim3(p.ctas), kWarps * 32, smem, s>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || p.splits == 1) return e;
  return launch_pdl(attend_merge_kernel<__nv_bfloat16, D>, dim3(p.batch * p.n_q_heads), dim3(D), 0, s,
                    (const float*)p.part_o, (const float*)p.part_ml, p.splits, p.out, p.lse);
}

template <int D>
cudaError_t dispatch_mma(int G, const AttParams& p, cudaStream_t s) {
  switch (G) {
    case 1: return launch_mma<D, 1>(p, s);
    case 2: return launch_mma<D, 2>(p, s);
    case 4: return launch_mma<D, 4>(p, s);
    case 8: return launch_mma<D, 8>(p, s);
    default: return cudaErrorInvalidValue;
  }
}

template <typename KT, int D>
cudaError_t dispatch_g(int G, const AttParams& p, cudaStream_t s) {
  switch (G) {
    case 1: return launch_t<KT, D, 1>(p, s);
    case 2: return launch_t<KT, D, 2>(p, s);
    case 4: return launch_t<KT, D, 4>(p, s);
    case 8: return launch_t<KT, D, 8>(p, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

// Split plan: as many splits per KV head as fit in one wave of resident CTAs on
// a 148-SM B200 (by default 3 CTAs per SM for G <= 4, 2 for G = 8, set by the
// registers), each split a multiple of 64 rows (one 16-row tile per warp).  A
// pure function of the sizes, so the workspace size is known without a device.
AttendPlan attend_plan(int batch, int n_q_heads, int n_kv_heads, int head_dim, int C, int max_tail,
                       int ctas_per_sm) {
  AttendPlan pl{1, 64, 0, 1, ctas_per_sm > 0 ? 1 : 0};
  const long rows = (long)C + (max_tail > 0 ? max_tail : 0);
  const long units = (long)batch * n_kv_heads;
  if (rows <= 0 || units <= 0 || n_kv_heads <= 0) return pl;
  const int G = n_q_heads / n_kv_heads;
  const long target = 148L * (ctas_per_sm > 0 ? ctas_per_sm : (G >= 8 ? 2 : 3));
  const int quantum = kTile * kWarps;
  long splits = target / units;
  if (splits < 1) splits = 1;
  long per = (rows + splits - 1) / splits;
  per = ((per + quantum - 1) / quantum) * quantum;
  pl.rows_per_split = (int)per;
  pl.splits = (int)((rows + per - 1) / per);
  // The decode step's plan (ctas_per_sm given) runs its items, all of about C rows,
  // as a persistent grid of at most one wave.  Otherwise one CTA per item: the
  // rows of a tail can be as ragged as the sequences, and the hardware's CTA
  // scheduling balances those better than a fixed stride over the items.
  const long items = units * pl.splits;
  pl.ctas = (int)(ctas_per_sm > 0 && items > target ? target : items);
  if (pl.splits > 1) {
    const size_t o = (size_t)batch * n_q_heads * pl.splits * head_dim * 4;
    const size_t ml = (size_t)batch * n_q_heads * pl.splits * 2 * 4;
    pl.workspace_bytes = ((o + 255) / 256) * 256 + ((ml + 255) / 256) * 256;
  }
  return pl;
}

cudaError_t launch_attend(const void* q, int q_f32, int n_q_heads, const KvView& kv, const int32_t* idx,
                          const int32_t* count, int C, const int32_t* tail_begin, int max_tail, void* out,
                          float* lse, void* workspace, const AttendPlan& plan, cudaStream_t s) {
  AttParams p;
  p.q = q;
  p.q_f32 = q_f32;
  p.n_q_heads = n_q_heads;
  p.k = static_cast<const uint8_t*>(kv.k);
  p.v = static_cast<const uint8_t*>(kv.v);
  p.batch = kv.batch;
  p.n_kv = kv.n_kv;
  p.t_max = kv.t_max;
  p.page_size = kv.page_size;
  p.max_pages = kv.max_pages;
  p.n_pages = kv.n_pages;
  p.page_table = kv.page_table;
  p.seq_lens = kv.seq_lens;
  p.idx = idx;
  p.count = count;
  p.C = C;
  p.tail_begin = tail_begin;
  p.max_tail = tail_begin ? max_tail : 0;
  p.splits = plan.splits;
  p.n_items = plan.splits * kv.batch * kv.n_kv;
  p.ctas = plan.ctas > 0 ? plan.ctas : 1;
  p.lean = plan.lean;
  p.rows_per_split = plan.rows_per_split;
  if (plan.splits > 1) {
    const size_t o = (size_t)kv.batch * n_q_heads * plan.splits * kv.head_dim * 4;
    p.part_o = static_cast<float*>(workspace);
    p.part_ml = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + ((o + 255) / 256) * 256);
  } else {
    p.part_o = nullptr;
    p.part_ml = nullptr;
  }
  p.out = out;
  p.lse = lse;
  p.qscale = kLog2e / sqrtf((float)kv.head_dim);
  const int G = n_q_heads / kv.n_kv;
  if (kv.kv_f32) return kv.head_dim == 64 ? dispatch_g<float, 64>(G, p, s) : dispatch_g<float, 128>(G, p, s);
  if (!q_f32) return kv.head_dim == 64 ? dispatch_mma<64>(G, p, s) : dispatch_mma<128>(G, p, s);
  return kv.head_dim == 64 ? dispatch_g<__nv_bfloat16, 64>(G, p, s) : dispatch_g<__nv_bfloat16, 128>(G, p, s);
}

// Scratch of asp_sparse_attend_noalloc: the split-K partials of one call, for
// callers that cannot allocate.  File scope, so every device that loads the
// library holds it for the life of the process.
static __device__ __align__(256) unsigned char g_noalloc_scratch[ASP_NOALLOC_SCRATCH_BYTES];

// Device address of g_noalloc_scratch on the current device.  In host code the
// array's name is only a host-side stand-in, so the address is looked up once per
// device (with that device current) and cached.
static cudaError_t noalloc_scratch_address(void** ptr) {
  static std::mutex mu;
  static void* addr[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    addr[dev] = p;
  }
  *ptr = addr[dev];
  return cudaSuccess;
}

cudaError_t launch_attend_noalloc(const void* q, int q_f32, int n_q_heads, const KvView& kv, const int32_t* idx,
                                  const int32_t* count, int C, const int32_t* tail_begin, int max_tail, void* out,
                                  float* lse, const AttendPlan& plan, cudaStream_t s) {
  if (plan.workspace_bytes > ASP_NOALLOC_SCRATCH_BYTES) return cudaErrorInvalidValue;
  void* scratch = nullptr;
  cudaError_t e = noalloc_scratch_address(&scratch);
  if (e != cudaSuccess) return e;
  return launch_attend(q, q_f32, n_q_heads, kv, idx, count, C, tail_begin, max_tail, out, lse, scratch, plan, s);
}

ASP_STATUS_READER(read_status_attend)

}  // namespace asp
