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
  int tiles_per_unit;      // gather kernel: 16-row tiles planned per unit
  long long total_tiles;   // gather kernel: units * tiles_per_unit
  int stages;              // gather kernel: stages per producer / consumer pair
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
  [[maybe_unused]] float x2, x3;   // rows 8-15: zero, discarded
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

// Cluster helpers: a barrier over the CTAs of the cluster (release / acquire, so
// that shared-memory stores before it are seen after it), and a store of one
// float into the shared memory of CTA `rank` of the cluster at the offset of `p`.
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void st_cluster_f32(const float* p, uint32_t rank, float v) {
  uint32_t a;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(a) : "r"(smem_u32(p)), "r"(rank));
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(a), "f"(v) : "memory");
}
// Four floats at a 16-byte aligned `p` into the shared memory of CTA `rank`.
__device__ __forceinline__ void st_cluster_f32x4(const float* p, uint32_t rank, float4 v) {
  uint32_t a;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(a) : "r"(smem_u32(p)), "r"(rank));
  asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(a), "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w)
               : "memory");
}

// LEAN: the row copies are issued from a partly unrolled loop, which keeps the
// registers at the level that lets one CTA share an SM with the key scan's and the
// predictor's (the decode step); the fully unrolled form keeps more copies in
// flight where three CTAs share an SM (stand-alone calls).
// CLUSTER: one work item per CTA and the splits of a unit form one thread-block
// cluster (rank = split): the splits' partials meet in the shared memory of the
// cluster's first CTA, which merges them and writes the output -- no partials in
// global memory and no merge kernel.  Every CTA reaches both cluster barriers:
// the only waits before them are the bounded stage waits, and no CTA leaves the
// item loop early in this mode.
template <int D, int G, int STAGES, bool LEAN, bool CLUSTER = false>
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
  // launched with programmatic stream serialisation: everything above overlaps the
  // previous kernel; every global access comes after its completion
  pdl_wait();

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
  // The raw index of this lane's row in tile t, loaded without waiting for the
  // unit's count (any r < C lies inside the index array): the index loads of a
  // tile go out a tile ahead of its copies, and those of the first tiles together
  // with the count.
  auto load_raw = [&](int tt) -> int {
    const int r = r0 + (warp + tt * kWarps) * kTile + (lane & 15);
    return (p.idx && r < p.C) ? __ldg(p.idx + (size_t)unit * p.C + r) : 0;
  };
  // Row source of this lane for tile t (lanes 0-15: K rows, 16-31: V rows), given
  // its raw index.
  auto resolve = [&](int tt, int jraw) -> RowSrc {
    const int rr = lane & 15;
    const bool isv = lane >= 16;
    const int r = r0 + (warp + tt * kWarps) * kTile + rr;
    bool valid = r < r1;
    int j = 0;
    if (valid) {
      if (r < n_sel) {
        j = jraw;
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
  int raw[STAGES];
#pragma unroll
  for (int s = 0; s < STAGES; ++s) raw[s] = load_raw(s);
  int issued = 0;
#pragma unroll
  for (int s = 0; s < STAGES; ++s) {
    if (s < my_tiles) {
      const int sl = (int)((tbase + s) % STAGES);
      vmask[sl] = issue(resolve(s, raw[s]), sl);
      ++issued;
    }
  }
  int raw_next = issued < my_tiles ? load_raw(issued) : 0;

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
      vmask[slot] = issue(resolve(issued, raw_next), slot);
      ++issued;
      if (issued < my_tiles) raw_next = load_raw(issued);
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
  if constexpr (CLUSTER) {
    // Every CTA of the cluster is past its stages, so the first CTA's shared memory
    // beyond its warp-merge area is free for the partials: [splits][G][D] outputs,
    // then [splits][G][2] (max, sum).  Four channels per thread and store.
    cluster_sync_all();
    float* slot_o = mml + kWarps * G * 2;   // 16-byte aligned: kWarps * G * (D + 2) floats in
    float* slot_ml = slot_o + p.splits * G * D;
    for (int e4 = threadIdx.x; e4 < G * D / 4; e4 += kWarps * 32) {
      const int gg = (4 * e4) / D, c = 4 * e4 - gg * D;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) M = fmaxf(M, mml[(w * G + gg) * 2]);
      float L = 0.f;
      float4 O = make_float4(0.f, 0.f, 0.f, 0.f);
      if (M != -INFINITY) {
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
          const float mw = mml[(w * G + gg) * 2];
          if (mw == -INFINITY) continue;
          const float f = ex2(mw - M);
          L += mml[(w * G + gg) * 2 + 1] * f;
          const float4 x = *reinterpret_cast<const float4*>(mo + (w * G + gg) * D + c);
          O.x += x.x * f;
          O.y += x.y * f;
          O.z += x.z * f;
          O.w += x.w * f;
        }
      }
      st_cluster_f32x4(slot_o + (split * G + gg) * D + c, 0, O);
      if (c == 0) {
        st_cluster_f32(slot_ml + (split * G + gg) * 2 + 0, 0, M);
        st_cluster_f32(slot_ml + (split * G + gg) * 2 + 1, 0, L);
      }
    }
    cluster_sync_all();   // the partials are in the first CTA's shared memory
    if (split == 0) {
      for (int e4 = threadIdx.x; e4 < G * D / 4; e4 += kWarps * 32) {
        const int gg = (4 * e4) / D, c = 4 * e4 - gg * D;
        float M = -INFINITY;
        for (int sp = 0; sp < p.splits; ++sp) M = fmaxf(M, slot_ml[(sp * G + gg) * 2]);
        float L = 0.f;
        float4 O = make_float4(0.f, 0.f, 0.f, 0.f);
        if (M != -INFINITY) {
          for (int sp = 0; sp < p.splits; ++sp) {
            const float ms = slot_ml[(sp * G + gg) * 2];
            if (ms == -INFINITY) continue;
            const float f = ex2(ms - M);
            L += slot_ml[(sp * G + gg) * 2 + 1] * f;
            const float4 x = *reinterpret_cast<const float4*>(slot_o + (sp * G + gg) * D + c);
            O.x += x.x * f;
            O.y += x.y * f;
            O.z += x.z * f;
            O.w += x.w * f;
          }
        }
        const float r = L > 0.f ? 1.f / L : 0.f;
        const size_t bh = (size_t)b * p.n_q_heads + h * G + gg;
        const __nv_bfloat162 lo2 = __floats2bfloat162_rn(O.x * r, O.y * r);
        const __nv_bfloat162 hi2 = __floats2bfloat162_rn(O.z * r, O.w * r);
        __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(p.out) + bh * D + c;
        if ((reinterpret_cast<uintptr_t>(p.out) & 7) == 0) {   // D * 2 and c * 2 keep the 8-byte alignment
          uint2 packed;
          packed.x = *reinterpret_cast<const uint32_t*>(&lo2);
          packed.y = *reinterpret_cast<const uint32_t*>(&hi2);
          *reinterpret_cast<uint2*>(dst) = packed;
        } else {
          dst[0] = lo2.x;
          dst[1] = lo2.y;
          dst[2] = hi2.x;
          dst[3] = hi2.y;
        }
        if (c == 0 && p.lse) p.lse[bh] = L > 0.f ? (M + __log2f(L)) * kLn2 : -INFINITY;
      }
    }
    break;   // one item per CTA
  } else {
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
  }
  // the next item's copies overwrite the merge area: generic accesses first
  fence_proxy_async_smem();
  tbase += (uint32_t)my_tiles;
  if (__syncthreads_or(!ok)) break;   // a wait ran out: stop (the copies have drained)
  }
}

// ---- bf16 cache and query: persistent gather, producer / consumer warp pairs --
//
// Every (sequence, KV head) unit is planned for C + max_tail rows, cut into
// 16-row tiles; the flattened tiles of all units are split into equal
// contiguous ranges, one per CTA (at most one CTA per SM), so every CTA gathers
// the same number of rows whatever the split of units.  Within a CTA, tile k of
// its range belongs to warp pair k % NP: producer warp NP + w issues the pair's
// tiles into the pair's ring of SP stages (16 K + 16 V rows each, 16-byte padded
// pitch for conflict-free ldmatrix) and consumer warp w consumes them in the same
// order -- one in-order ring per pair, so no barrier phase can be waited on
// before its predecessor completed.
//   producer: walks its tiles with the unit and tile position kept incrementally
//     (no division per tile), the unit's lengths cached; two tiles per round
//     (lanes 0-15 and 16-31 resolve one row each); index loads two rounds ahead
//     of the copies, page lookups one round ahead; the 32 rows of a tile go in
//     as 16-byte cp.async (several rows per warp instruction, rows that are not
//     read zero-filled), each lane's copies arriving on the stage's "full"
//     barrier when they land, lane 0 adding the tile's row mask;
//   consumer: the tensor-core logits, online softmax and P.V of
//     attend_mma_kernel, then releases the stage on its "empty" barrier.
// The rows a CTA holds of one unit form a segment: at a segment's end the
// consumers merge through shared memory; a unit held by one CTA is written out
// directly, otherwise the CTA writes a partial (max, sum, unnormalised output)
// and attend_gather_merge_kernel combines them.  The producers run on into the
// next segment meanwhile.  Every barrier wait is bounded (ASP_DEV_WAIT_LIMIT).
constexpr int kGatherPairs = 6;
constexpr int kGatherThreads = 2 * kGatherPairs * 32;

// Tiles [t0, t1) of CTA c out of I over N CTAs; owner of tile i.
__device__ __forceinline__ long long tile_start(long long c, long long I, long long N) { return c * I / N; }
__device__ __forceinline__ long long tile_owner(long long i, long long I, long long N) { return ((i + 1) * N - 1) / I; }

// Bounded wait that also gives up once another warp of the CTA has given up.
__device__ __forceinline__ bool gather_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  for (uint32_t i = 0; i < kWaitTries; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
  }
  flag_status(ASP_DEV_WAIT_LIMIT);
  *abort_flag = 1;
  return false;
}

__device__ __forceinline__ void consumers_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(kGatherPairs * 32) : "memory");
}

__device__ __forceinline__ void mbar_arrive_plain(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

template <int D, int G>
__global__ void __launch_bounds__(kGatherThreads, 1) attend_gather_kernel(AttParams p) {
  constexpr int NP = kGatherPairs;
  constexpr int ROW_BYTES = D * 2;
  constexpr int STRIDE = ROW_BYTES + 16;
  constexpr int HALF = kTile * STRIDE;
  constexpr int STAGE = 2 * HALF;
  constexpr int KS = D / 16;
  constexpr int NT = D / 8;
  constexpr int CPR = ROW_BYTES / 16;   // 16-byte chunks per row
  constexpr int RPI = 32 / CPR;         // rows per warp instruction
  constexpr uint32_t kNone = 0xffffffffu;
  static_assert(G >= 1 && G <= 8 && kTile == 16 && (32 % CPR) == 0, "layout");

  extern __shared__ __align__(128) uint8_t smem[];
  const int SP = p.stages;   // stages per pair
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint8_t* const ring = smem;                                                 // [NP][SP] stages
  float* const mo = reinterpret_cast<float*>(ring + (size_t)NP * SP * STAGE);   // [NP][G][D]
  float* const mml = mo + NP * G * D;                                         // [NP][G][2]
  uint64_t* const full = reinterpret_cast<uint64_t*>(mml + NP * G * 2);       // [NP][SP]
  uint64_t* const empty = full + NP * SP;                                     // [NP][SP]
  uint32_t* const masks = reinterpret_cast<uint32_t*>(empty + NP * SP);       // [NP][SP]
  volatile int* const abort_flag = reinterpret_cast<volatile int*>(masks + NP * SP);

  if (threadIdx.x == 0) {
    for (int s = 0; s < NP * SP; ++s) {
      mbar_init(&full[s], 1);    // lane 0 of the producer; the copies add their own arrivals
      mbar_init(&empty[s], 1);
    }
    *abort_flag = 0;
    mbar_init_fence();
  }
  __syncthreads();

  const long long I = p.total_tiles, N = gridDim.x, c = blockIdx.x;
  const long long t0 = tile_start(c, I, N), t1 = tile_start(c + 1, I, N);
  if (t0 >= t1) return;
  const int TPU = p.tiles_per_unit;
  const int u_first = (int)(t0 / TPU);
  const int nseg = (int)((t1 - 1) / TPU) - u_first + 1;
  const int ntl = (int)(t1 - t0);
  const int pair = warp % NP;
  const int my_n = ntl > pair ? (ntl - pair + NP - 1) / NP : 0;   // the pair's tiles
  uint8_t* const pring = ring + (size_t)pair * SP * STAGE;

  if (warp >= NP) {
    // ------------------------------------------------------------ producer
    const int half = lane >> 4, rr = lane & 15;
    // position of the pair's first tile; advanced by NP tiles per tile, by 2 NP per round
    const long long gfirst = t0 + pair;
    int unit0 = (int)(gfirst / TPU);
    int tl0 = (int)(gfirst - (long long)unit0 * TPU);
    // this lane's tile in round i is the pair's tile 2i + half
    struct Pos {
      int unit, tl;
    };
    auto step = [&](Pos q, int tiles) -> Pos {   // q moved on by tiles * NP CTA tiles
      q.tl += tiles * NP;
      while (q.tl >= TPU) {
        q.tl -= TPU;
        ++q.unit;
      }
      return q;
    };
    // the unit's lengths, reloaded only when the unit changes
    int cu = -1, cT = 0, cn_sel = 0, ctb = 0, cn_rows = 0, cb = 0, ch = 0;
    auto unit_params = [&](int unit) {
      if (unit == cu) return;
      cu = unit;
      cb = unit / p.n_kv;
      ch = unit - cb * p.n_kv;
      int T = p.seq_lens ? __ldg(p.seq_lens + cb) : p.t_max;
      cT = T < 0 ? 0 : (T > p.t_max ? p.t_max : T);
      int n_sel = (p.C > 0 && p.count) ? __ldg(p.count + unit) : 0;
      cn_sel = n_sel < 0 ? 0 : (n_sel > p.C ? p.C : n_sel);
      int tb = cT;
      if (p.tail_begin) {
        tb = __ldg(p.tail_begin + cb);
        tb = tb < 0 ? 0 : (tb > cT ? cT : tb);
      }
      ctb = tb;
      int tail = cT - tb;
      if (tail > p.max_tail) {
        if (lane == 0 && pair == 0) flag_status(ASP_DEV_TAIL_LIMIT);
        tail = p.max_tail;
      }
      cn_rows = cn_sel + tail;
    };
    // stage A: the raw index of this lane's row (loads issued, not waited for)
    struct RowA {
      int unit, r, raw;
    };
    auto stage_a = [&](Pos q, int j) -> RowA {
      RowA a{-1, 0, 0};
      if (j >= my_n) return a;
      a.unit = q.unit;
      a.r = q.tl * kTile + rr;
      if (a.r < p.C) a.raw = __ldg(p.idx + (size_t)q.unit * p.C + a.r);
      return a;
    };
    // stage B: the token (-1: not read) and, for a paged cache, its page (load issued)
    struct RowB {
      int unit, tok, page;
    };
    auto stage_b = [&](const RowA& a) -> RowB {
      RowB bq{a.unit, -1, 0};
      if (a.unit < 0) return bq;
      unit_params(a.unit);
      if (a.r >= cn_rows) return bq;
      int tok;
      if (a.r < cn_sel) {
        tok = a.raw;
        if (tok < 0 || tok >= cT) {
          flag_status(ASP_DEV_BAD_INDEX);
          return bq;
        }
        if (tok >= ctb) return bq;   // covered by the tail
      } else {
        tok = ctb + (a.r - cn_sel);
      }
      bq.tok = tok;
      if (p.page_size) bq.page = __ldg(p.page_table + (size_t)cb * p.max_pages + tok / p.page_size);
      return bq;
    };
    // stage C: the source row in the k / v arrays (32 bits: the cache fits in device memory)
    auto stage_c = [&](const RowB& bq) -> uint32_t {
      if (bq.tok < 0) return kNone;
      if (p.page_size == 0) return (uint32_t)((size_t)bq.unit * p.t_max + bq.tok);
      if (bq.page < 0 || bq.page >= p.n_pages) {
        flag_status(ASP_DEV_BAD_PAGE);
        return kNone;
      }
      const int h = bq.unit % p.n_kv;
      return (uint32_t)(((size_t)bq.page * p.n_kv + h) * p.page_size + (bq.tok % p.page_size));
    };

    bool ok = true;
    unit_params(unit0);               // its loads go out with the first index loads
    Pos qA{unit0, tl0};               // position of this lane's tile in round 0
    if (half) qA = step(qA, 1);
    Pos qB = step(qA, 2), qC = step(qB, 2);
    RowA aA = stage_a(qA, half), aB = stage_a(qB, 2 + half);
    RowB bA = stage_b(aA);
    const int rounds = (my_n + 1) / 2;
#pragma unroll 1
    for (int i = 0; i < rounds && ok; ++i) {
      const RowA aC = stage_a(qC, 2 * (i + 2) + half);
      const RowB bB = stage_b(aB);
      const uint32_t row = stage_c(bA);
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const int j = 2 * i + hf;   // the pair's tile
        if (j >= my_n) break;
        const int slot = j % SP;
        if (j >= SP) {
          ok = __all_sync(0xffffffffu, gather_wait(&empty[pair * SP + slot], (uint32_t)(j / SP - 1) & 1u, abort_flag));
          if (!ok) break;
        }
        const uint32_t vm = (__ballot_sync(0xffffffffu, row != kNone) >> (16 * hf)) & 0xffffu;
        if (vm) {
          const uint32_t st = smem_u32(pring + (size_t)slot * STAGE);
          const uint32_t c16 = (uint32_t)(lane % CPR) * 16u;
#pragma unroll
          for (int ins = 0; ins < 32 / RPI; ++ins) {
            const int ri = RPI * ins + lane / CPR;   // 0-15 K rows, 16-31 V rows
            const uint32_t src = __shfl_sync(0xffffffffu, row, 16 * hf + (ri & 15));
            const bool valid = src != kNone;
            const uint8_t* from = (ri < 16 ? p.k : p.v) + (valid ? (size_t)src * ROW_BYTES + c16 : 0);
            const uint32_t dst = st + (uint32_t)((ri < 16 ? 0 : HALF) + (ri & 15) * STRIDE) + c16;
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(from),
                         "r"(valid ? 16 : 0)
                         : "memory");
          }
          asm volatile("cp.async.mbarrier.arrive.shared::cta.b64 [%0];" ::"r"(smem_u32(&full[pair * SP + slot]))
                       : "memory");
        }
        __syncwarp();
        if (lane == 0) {
          masks[pair * SP + slot] = vm;
          mbar_arrive_plain(&full[pair * SP + slot]);
        }
      }
      qC = step(qC, 2);
      aB = aC;
      bA = bB;
    }
    if (!ok) asm volatile("cp.async.wait_all;" ::: "memory");   // let this producer's copies land
    return;
  }

  // -------------------------------------------------------------- consumers
  const int g = lane >> 2, t = lane & 3;
  auto load_q = [&](int unit, uint32_t (&qa)[KS][2]) {
    const int b = unit / p.n_kv, h = unit - b * p.n_kv;
    const __nv_bfloat16* qrow =
        static_cast<const __nv_bfloat16*>(p.q) + ((size_t)b * p.n_q_heads + h * G + (g < G ? g : 0)) * D;
#pragma unroll
    for (int kk = 0; kk < KS; ++kk) {
      qa[kk][0] = g < G ? __ldg(reinterpret_cast<const uint32_t*>(qrow + 16 * kk + 2 * t)) : 0u;
      qa[kk][1] = g < G ? __ldg(reinterpret_cast<const uint32_t*>(qrow + 16 * kk + 8 + 2 * t)) : 0u;
    }
  };
  uint32_t qa[KS][2];
  load_q(u_first, qa);
  const int mat = lane >> 3, mrow = lane & 7;
  const uint32_t k_off = (uint32_t)(((mat >> 1) * 8 + mrow) * STRIDE + (mat & 1) * 16);
  const uint32_t v_off = (uint32_t)(HALF + ((mat & 1) * 8 + mrow) * STRIDE + (mat >> 1) * 16);
  bool ok = true;
  int j = 0;   // the pair's next tile
  for (int sg = 0; sg < nseg; ++sg) {
    const int u = u_first + sg;
    const long long ua = (long long)u * TPU;
    const long long hi = ua + TPU < t1 ? ua + TPU : t1;
    // the pair's tiles before hi: CTA-local k = pair + NP * j < hi - t0
    const long long khi = hi - t0 - pair;
    const int jhi = khi > 0 ? (int)((khi + NP - 1) / NP) : 0;
    float o[NT][2];
#pragma unroll
    for (int n = 0; n < NT; ++n) o[n][0] = o[n][1] = 0.f;
    float m_run = -INFINITY, l_run = 0.f;
#pragma unroll 1
    for (; j < jhi && ok; ++j) {
      const int slot = j % SP;
      if (!__all_sync(0xffffffffu, gather_wait(&full[pair * SP + slot], (uint32_t)(j / SP) & 1u, abort_flag))) {
        ok = false;
        break;
      }
      const uint32_t vm = masks[pair * SP + slot];
      if (vm) {
        const uint32_t base = smem_u32(pring + (size_t)slot * STAGE);
        float s0[2] = {0.f, 0.f}, s1[2] = {0.f, 0.f};
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
          uint32_t kb[4];
          ldsm_x4(kb, base + k_off + 32 * ks);
          mma_top8(s0[0], s0[1], qa[ks][0], qa[ks][1], kb[0], kb[1]);
          mma_top8(s1[0], s1[1], qa[ks][0], qa[ks][1], kb[2], kb[3]);
        }
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
        uint32_t pa0, pa2, pl0, pl2;
        split_bf16x2(pr[0], pr[1], pa0, pl0);
        split_bf16x2(pr[2], pr[3], pa2, pl2);
        if (corr != 1.f) {
#pragma unroll
          for (int n = 0; n < NT; ++n) {
            o[n][0] *= corr;
            o[n][1] *= corr;
          }
        }
#pragma unroll
        for (int jj = 0; jj < D / 16; ++jj) {
          uint32_t vb[4];
          ldsm_x4_trans(vb, base + v_off + 32 * jj);
          mma_top8(o[2 * jj][0], o[2 * jj][1], pa0, pa2, vb[0], vb[1]);
          mma_top8(o[2 * jj + 1][0], o[2 * jj + 1][1], pa0, pa2, vb[2], vb[3]);
          mma_top8(o[2 * jj][0], o[2 * jj][1], pl0, pl2, vb[0], vb[1]);
          mma_top8(o[2 * jj + 1][0], o[2 * jj + 1][1], pl0, pl2, vb[2], vb[3]);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive_plain(&empty[pair * SP + slot]);
    }
    l_run += __shfl_xor_sync(0xffffffffu, l_run, 1);
    l_run += __shfl_xor_sync(0xffffffffu, l_run, 2);

    // merge the consumers; a unit held by this CTA alone is written out
    if (g < G) {
#pragma unroll
      for (int n = 0; n < NT; ++n)
        *reinterpret_cast<float2*>(mo + (warp * G + g) * D + n * 8 + 2 * t) = make_float2(o[n][0], o[n][1]);
      if (t == 0) {
        mml[(warp * G + g) * 2 + 0] = m_run;
        mml[(warp * G + g) * 2 + 1] = l_run;
      }
    }
    consumers_sync();
    // the next segment's query loads while the partials are combined
    if (sg + 1 < nseg) load_q(u + 1, qa);
    const bool whole = tile_owner(ua, I, N) == tile_owner(ua + TPU - 1, I, N);
    const int pslot = 2 * (int)c + (sg == 0 ? 0 : 1);
    const int b = u / p.n_kv, h = u - b * p.n_kv;
    for (int e = threadIdx.x; e < G * D; e += NP * 32) {
      const int gg = e / D, cc = e - gg * D;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < NP; ++w) M = fmaxf(M, mml[(w * G + gg) * 2]);
      float L = 0.f, O = 0.f;
      if (M != -INFINITY) {
#pragma unroll
        for (int w = 0; w < NP; ++w) {
          const float mw = mml[(w * G + gg) * 2];
          if (mw == -INFINITY) continue;
          const float f = ex2(mw - M);
          L += mml[(w * G + gg) * 2 + 1] * f;
          O += mo[(w * G + gg) * D + cc] * f;
        }
      }
      if (whole) {
        const size_t bh = (size_t)b * p.n_q_heads + h * G + gg;
        static_cast<__nv_bfloat16*>(p.out)[bh * D + cc] = __float2bfloat16_rn(L > 0.f ? O / L : 0.f);
        if (cc == 0 && p.lse) p.lse[bh] = L > 0.f ? (M + __log2f(L)) * kLn2 : -INFINITY;
      } else {
        p.part_o[((size_t)pslot * G + gg) * D + cc] = O;
        if (cc == 0) {
          p.part_ml[((size_t)pslot * G + gg) * 2 + 0] = M;
          p.part_ml[((size_t)pslot * G + gg) * 2 + 1] = L;
        }
      }
    }
    consumers_sync();
  }
}

// Log-sum-exp merge of the units that several CTAs of attend_gather_kernel share:
// block (c, g) merges head g of the unit whose first tile lies in CTA c's range
// and whose last tile lies past it (at most one per CTA).  The partials are read
// eight CTAs at a time with independent loads.
template <int D, int G>
__global__ void __launch_bounds__(D) attend_gather_merge_kernel(AttParams p, int n_ctas) {
  const long long I = p.total_tiles, N = n_ctas, c = blockIdx.x;
  const int gg = blockIdx.y, cc = threadIdx.x;
  const int TPU = p.tiles_per_unit;
  const long long t0 = tile_start(c, I, N), t1 = tile_start(c + 1, I, N);
  if (t0 >= t1) return;
  const int u = (int)((t1 - 1) / TPU);
  const long long ua = (long long)u * TPU;
  if (ua < t0 || ua + TPU <= t1) return;
  pdl_wait();   // the partials come from the previous kernel
  const long long c1 = tile_owner(ua + TPU - 1, I, N);
  const int first_slot = (int)(2 * c + (u == (int)(t0 / TPU) ? 0 : 1));
  float M = -INFINITY, L = 0.f, O = 0.f;
  for (long long base = c; base <= c1; base += 8) {
    float mv[8], lv[8], ov[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const long long cx = base + i;
      // CTAs with an empty range (more CTAs than tiles) hold no partial
      const bool in = cx <= c1 && tile_start(cx, I, N) < tile_start(cx + 1, I, N);
      const int s = cx == c ? first_slot : (int)(2 * cx);
      mv[i] = in ? p.part_ml[((size_t)s * G + gg) * 2] : -INFINITY;
      lv[i] = in ? p.part_ml[((size_t)s * G + gg) * 2 + 1] : 0.f;
      ov[i] = in ? p.part_o[((size_t)s * G + gg) * D + cc] : 0.f;
    }
    float Mn = M;
#pragma unroll
    for (int i = 0; i < 8; ++i) Mn = fmaxf(Mn, mv[i]);
    if (Mn == -INFINITY) continue;
    if (M != -INFINITY) {
      const float f = ex2(M - Mn);
      L *= f;
      O *= f;
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (mv[i] == -INFINITY) continue;
      const float f = ex2(mv[i] - Mn);
      L += lv[i] * f;
      O += ov[i] * f;
    }
    M = Mn;
  }
  const int b = u / p.n_kv, h = u - b * p.n_kv;
  const size_t bh = (size_t)b * p.n_q_heads + h * G + gg;
  static_cast<__nv_bfloat16*>(p.out)[bh * D + cc] = __float2bfloat16_rn(L > 0.f ? O / L : 0.f);
  if (cc == 0 && p.lse) p.lse[bh] = L > 0.f ? (M + __log2f(L)) * kLn2 : -INFINITY;
}

// Log-sum-exp merge of the split partials: one CTA of D threads per query head.
template <typename KT, int D>
__global__ void __launch_bounds__(D) attend_merge_kernel(const float* __restrict__ part_o,
                                                         const float* __restrict__ part_ml, int splits, void* out,
                                                         float* lse) {
  using E = Elem<KT>;
  const size_t bh = blockIdx.x;
  const int c = threadIdx.x;
  pdl_trigger();   // the next call's attention may start its prologue
  pdl_wait();      // the split partials come from the previous kernel
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
  size_t smem = (size_t)kWarps * STAGES * TILE_BYTES + kWarps * STAGES * 8;
  const size_t merge = (size_t)kWarps * G * (D + 2) * 4;
  if (smem < merge) smem = merge;
  // One item per CTA and 4 to 8 splits (a portable cluster), whose partials fit
  // beside the warp-merge area: the splits merge inside their cluster.  Measured
  // alone (back to back over copies of the cache): 6 splits (Qwen3-8B shapes)
  // 19.8 against 22.3 us with the merge kernel; 3 splits (Qwen3-32B shapes) 34.8
  // against 33.5 us, so fewer splits keep the merge kernel.  Letting the next
  // kernel launch early from the cluster kernel cost 9 us at 3 splits.
  if (!p.lean && p.splits >= 4 && p.splits <= 8 && p.ctas == p.n_items &&
      merge + (size_t)p.splits * G * (D + 2) * 4 <= smem) {
    auto kc = attend_mma_kernel<D, G, STAGES, false, true>;
    if (prepare_kernel((const void*)kc, smem, kWarps * 32) < 1) return cudaErrorInvalidConfiguration;
    return launch_pdl_cluster(kc, dim3(p.ctas), dim3(kWarps * 32), smem, s, p.splits, p);
  }
  auto kern = p.lean ? attend_mma_kernel<D, G, STAGES, true> : attend_mma_kernel<D, G, STAGES, false>;
  if (prepare_kernel((const void*)kern, smem, kWarps * 32) < 1) return cudaErrorInvalidConfiguration;
  cudaError_t e = launch_pdl(kern, dim3(p.ctas), dim3(kWarps * 32), smem, s, p);
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

// Split plan of the per-item kernels: as many splits per KV head as fit in one
// wave of resident CTAs on a 148-SM B200 (by default 3 CTAs per SM: 166 registers
// x 128 threads; 2 per SM at G = 8 measured 41 against 36.5 us on the Qwen3-32B
// shapes), each split a multiple of 64 rows (one 16-row tile per warp).  The gather kernel's plan (stand-alone calls; the decode step
// keeps the per-item kernel, whose CTA fits beside the key scan's): every unit
// planned for C + max_tail rows, its tiles spread evenly over at most one CTA per
// SM (and at least 8 tiles per CTA), partials in 2 slots per CTA when a unit is
// shared.  A pure function of the sizes, so the workspace size (the larger of the
// two kernels' needs: which one runs depends on the data types) is known without
// a device.
constexpr int kGatherCtasMax = 148;
constexpr int kGatherMaxTail = 4096;   // longer tails (dense attention) keep one CTA per item
// The gather kernel pays a fixed cost per launch (filling 24 stages per SM before
// the first tile, the partials' merge) that the per-item kernel, three CTAs per SM
// streaming from the first row, does not: it is chosen from this many 16-row tiles
// per SM on (measured on the Qwen3 shapes: 55 tiles per SM slower, 110 even, 446 a
// third faster).
constexpr int kGatherMinTilesPerCta = 200;

// Whether any unit of the gather partition (total tiles over n CTAs, tpu tiles per
// unit) is shared by several CTAs: at most one unit starts in a CTA's range and
// runs past it.
static bool gather_has_shared(long long total, int tpu, int n) {
  for (long long c = 0; c < n; ++c) {
    const long long t0 = c * total / n, t1 = (c + 1) * total / n;
    if (t0 >= t1) continue;
    const long long ua = ((t1 - 1) / tpu) * tpu;
    if (ua >= t0 && ua + tpu > t1) return true;
  }
  return false;
}

AttendPlan attend_plan(int batch, int n_q_heads, int n_kv_heads, int head_dim, int C, int max_tail,
                       int ctas_per_sm) {
  AttendPlan pl{1, 64, 0, 1, ctas_per_sm > 0 ? 1 : 0, 0, 0, 0};
  const long rows = (long)C + (max_tail > 0 ? max_tail : 0);
  const long units = (long)batch * n_kv_heads;
  if (rows <= 0 || units <= 0 || n_kv_heads <= 0) return pl;
  const int G = n_q_heads / n_kv_heads;
  const long target = 148L * (ctas_per_sm > 0 ? ctas_per_sm : 3);
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
  const int mt = max_tail > 0 ? max_tail : 0;
  if (ctas_per_sm == 0 && mt <= (C > kGatherMaxTail ? C : kGatherMaxTail)) {
    pl.tiles_per_unit = (int)((rows + kTile - 1) / kTile);
    const long long total = (long long)units * pl.tiles_per_unit;
    const long long n = (total + 7) / 8;
    pl.gather_ctas = (int)(n < kGatherCtasMax ? n : kGatherCtasMax);
    pl.gather = total >= (long long)kGatherMinTilesPerCta * kGatherCtasMax ? 1 : 0;
    if (pl.gather && gather_has_shared(total, pl.tiles_per_unit, pl.gather_ctas)) {
      const size_t slots = 2 * (size_t)pl.gather_ctas * G;
      const size_t ws = ((slots * head_dim * 4 + 255) / 256) * 256 + ((slots * 2 * 4 + 255) / 256) * 256;
      if (ws > pl.workspace_bytes) pl.workspace_bytes = ws;
    }
  }
  return pl;
}

namespace {

int max_smem_optin() {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 232448;
  if (cache[dev] <= 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) == cudaSuccess && n > 0)
      cache[dev] = n;
  }
  return cache[dev] > 0 ? cache[dev] : 232448;
}

// Shared memory of the gather kernel: SP stages of 16 K + 16 V rows (16-byte
// padded pitch) per producer / consumer pair, the consumers' merge area, the
// stage barriers, masks and the abort flag.
template <int D, int G>
constexpr size_t gather_smem(int SP) {
  return (size_t)kGatherPairs * SP * 2 * kTile * (D * 2 + 16) + (size_t)kGatherPairs * G * (D + 2) * 4 +
         (size_t)kGatherPairs * SP * (8 + 8 + 4) + 16;
}

template <int D, int G>
cudaError_t launch_gather(AttParams p, cudaStream_t s) {
  // as many stages per pair as fit (at most 6, at least 2)
  const size_t budget = (size_t)max_smem_optin();
  int SP = 6;
  while (SP > 2 && gather_smem<D, G>(SP) > budget) --SP;
  if (gather_smem<D, G>(SP) > budget) return cudaErrorInvalidConfiguration;
  p.stages = SP;
  const size_t smem = gather_smem<D, G>(SP);
  auto kern = attend_gather_kernel<D, G>;
  if (prepare_kernel((const void*)kern, smem, kGatherThreads) < 1) return cudaErrorInvalidConfiguration;
  int n = p.ctas;
  if (n > sm_count()) n = sm_count();
  cudaError_t e = launch_prio(kern, dim3(n), dim3(kGatherThreads), smem, s, p);
  if (e != cudaSuccess) return e;
  if (!gather_has_shared(p.total_tiles, p.tiles_per_unit, n)) return cudaSuccess;
  return launch_pdl(attend_gather_merge_kernel<D, G>, dim3(n, G), dim3(D), 0, s, p, n);
}

template <int D>
cudaError_t dispatch_gather(int G, const AttParams& p, cudaStream_t s) {
  switch (G) {
    case 1: return launch_gather<D, 1>(p, s);
    case 2: return launch_gather<D, 2>(p, s);
    case 4: return launch_gather<D, 4>(p, s);
    case 8: return launch_gather<D, 8>(p, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

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
  p.tiles_per_unit = plan.tiles_per_unit;
  p.total_tiles = (long long)kv.batch * kv.n_kv * plan.tiles_per_unit;
  p.stages = 0;
  const bool gather = plan.gather && !kv.kv_f32 && !q_f32 && (reinterpret_cast<uintptr_t>(q) & 15) == 0;
  if (gather) {
    p.ctas = plan.gather_ctas > 0 ? plan.gather_ctas : 1;
    const size_t slots = 2 * (size_t)p.ctas * (n_q_heads / kv.n_kv);
    p.part_o = static_cast<float*>(workspace);
    p.part_ml = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) +
                                         ((slots * kv.head_dim * 4 + 255) / 256) * 256);
  } else if (plan.splits > 1) {
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
  if (gather) return kv.head_dim == 64 ? dispatch_gather<64>(G, p, s) : dispatch_gather<128>(G, p, s);
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
