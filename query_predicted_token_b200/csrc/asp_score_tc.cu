// asp_score_tc.cu -- step 2 on the 5th-generation tensor cores (bf16 keys).
//
// scores[b, h, j] = max_g (qpred[b, h*G+g] . k[b, h, j]) / sqrt(d) as the
// contraction S = K Q^T with K a 128-token x d tile (MMA M = 128) and Q the
// group's G predicted queries.  q_hat is fp32: each scaled query is split into
// bf16 hi = rn(q) and lo = rn(q - hi) (residual below 2^-17 |q|), both become
// rows of the B operand (N = 2G padded to 16), and the epilogue adds the two
// columns of each head -- bf16 x bf16 products are exact in the fp32
// accumulator, so the split keeps fp32-class accuracy at tensor-core rate.
//
// One persistent CTA per SM, warp-specialised:
//   warp 0     producer: 2-D TMA loads (128-byte swizzle) of each 128-token key
//              tile into a 4-stage ring, plus the tile's Q rows written in the
//              same swizzled K-major layout;
//   warp 1     allocates 32 TMEM columns and issues tcgen05.mma (M128 N16 K16,
//              fp32 accumulate) into one of two TMEM accumulators, committing to
//              the stage's "empty" and the accumulator's "full" barriers;
//   warps 2-5  epilogue: tcgen05.ld of their 32 TMEM lanes (one token each),
//              hi + lo per head, max over the group, coalesced store, and the
//              selection's first-digit histogram.
// Every barrier wait is bounded (ASP_DEV_WAIT_LIMIT).  The contiguous cache is
// one 2-D tensor [B*Hkv*t_max, d]; the paged cache [n_pages*Hkv*16, d] with one
// 16-row box per page.
#include <cuda.h>

#include "asp_common.cuh"
#include "asp_internal.h"

namespace asp {
namespace {

constexpr int kTileT = 128;    // tokens per tile = MMA M
constexpr int kN = 16;         // MMA N: rows (hi, lo) of the group's queries, padded
constexpr int kStages = 4;
// stages of the token-tile ring: three for 256-channel rows (64 KB tiles), and three
// for groups of 8 query heads, whose predictor runs as 2 CTAs per SM: a 3-stage scan
// CTA then fits beside them and the step's attention CTA, and starts its key
// prefetch during the prediction (32B shapes 237 -> 231 us); four otherwise (8B
// shapes: 136.5 us with four, 138.9 with three)
__host__ __device__ constexpr int stages_for(int D, int G) { return (D >= 256 || G >= 8) ? 3 : kStages; }
constexpr int kThreadsTC = 192;
constexpr uint32_t kTmemCols = 32;   // two 16-column fp32 accumulators
// instruction descriptor, kind::f16: D fp32, A and B bf16, both K-major, N, M
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kN >> 3) << 17) |
                            ((uint32_t)(kTileT >> 4) << 24);

struct TcParams {
  const float* qpred;
  // page-bound mode: each "key" row is a page's [kmin, kmax] (2d channels) and
  // each query row is [min(q, 0), max(q, 0)], so the dot product is the bound
  const void* qraw;   // the current query (bf16 or fp32) in page-bound mode, else null
  int qraw_f32;
  int len_div;        // units per length: 1 for tokens, the page size for page bounds
  int len_cap;        // cap of seq_lens (tokens)
  int early;          // stream the first tiles' keys before the previous kernel ends
  int n_q_heads, G;   // G is also the kernel's template argument
  int batch, n_kv, t_max, page_size, max_pages, n_pages;
  const int32_t* page_table;
  const int32_t* seq_lens;
  float* scores;
  int32_t* hist;
  float scale;
};

struct TileCursor {
  int b, h, tile, ntile, T;
};

// shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups 1024 B apart
__device__ __forceinline__ uint64_t sw128_desc(uint32_t addr) {
  return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint64_t* bar,
                                            uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void umma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(kIdesc), "r"(accumulate));
}

__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// Raises the barrier's expected transaction bytes without arriving.
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.expect_tx.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}

template <uint32_t IDESC>
__device__ __forceinline__ void umma_bf16_i(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(IDESC), "r"(accumulate));
}

// W consecutive accumulator columns of this warp's 32 TMEM lanes (W = 4, 8, 16, 32).
template <int W>
__device__ __forceinline__ void tmem_ld_w(uint32_t taddr, float (&v)[W]) {
  uint32_t r[W];
  if constexpr (W == 4) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(taddr));
  } else if constexpr (W == 8) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
  } else if constexpr (W == 16) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
  } else {
    static_assert(W == 32, "width");
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
  }
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < W; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ uint32_t bf16x2_bits(float lo_elem, float hi_elem) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo_elem, hi_elem);
  return *reinterpret_cast<const uint32_t*>(&v);
}

template <int D, int G>
__global__ void __launch_bounds__(kThreadsTC, 1) score_tc_kernel(const __grid_constant__ CUtensorMap kmap,
                                                                 TcParams p) {
  constexpr int HALVES = D / 64;                      // 64-channel (128-byte) swizzle columns
  constexpr int KBYTES = kTileT * D * 2;              // one key tile
  constexpr int QBYTES = HALVES * kN * 128;           // the tile's B operand
  constexpr int STAGE = KBYTES + QBYTES;              // multiple of 1024
  constexpr int KSTEPS = D / 16;
  constexpr int QCH = HALVES * kN * 8 / 32;           // 16-byte Q chunks per producer lane
  constexpr int kStages = stages_for(D, G);
  static_assert(STAGE % 1024 == 0, "stage alignment");

  extern __shared__ uint8_t smem_raw[];
  __shared__ uint32_t s_tmem;
  __shared__ int scratch[33];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  const uint32_t sbase = smem_u32(smem);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages * STAGE);
  uint64_t* empty = full + kStages;
  uint64_t* tfull = empty + kStages;
  uint64_t* tempty = tfull + 2;
  int* pre = reinterpret_cast<int*>(tempty + 2);
  int* lens = pre + p.batch + 1;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 4);
    }
    mbar_init_fence();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&s_tmem)),
                 "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  // Everything above touches no global memory, so it overlaps the previous
  // kernel; the predicted queries, the cleared histogram and the cache
  // description are read only after it has finished.  In early mode that kernel
  // writes nothing else, so the cache description is read at once and the
  // producer streams its first tiles' keys before it waits.
  const bool early = p.early && p.page_size == 0;
  if (!early) pdl_wait();
  for (int b = threadIdx.x; b < p.batch; b += blockDim.x) {
    int t = p.seq_lens ? p.seq_lens[b] : p.len_cap;
    t = t < 0 ? 0 : (t > p.len_cap ? p.len_cap : t);
    lens[b] = (t + p.len_div - 1) / p.len_div;   // rows of this sequence
  }
  __syncthreads();
  cta_prefix_sum(p.batch, pre, [&](int b) { return ((lens[b] + kTileT - 1) / kTileT) * p.n_kv; }, scratch);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  if (early && warp != 0) pdl_wait();
  pdl_trigger();   // the selection may launch while the scan runs

  const int total = pre[p.batch];
  const int chunk = (total + gridDim.x - 1) / gridDim.x;
  const int t0 = min(total, (int)blockIdx.x * chunk);
  const int t1 = min(total, t0 + chunk);
  const int n_my = t1 - t0;

  auto locate = [&](int i, TileCursor& c) {
    int lo = 0, hi = p.batch;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (pre[mid] <= i) lo = mid; else hi = mid;
    }
    c.b = lo;
    c.T = lens[lo];
    c.ntile = (pre[lo + 1] - pre[lo]) / p.n_kv;
    const int r = i - pre[lo];
    c.h = r / c.ntile;
    c.tile = r - c.h * c.ntile;
  };
  auto advance = [&](TileCursor& c) {
    if (++c.tile == c.ntile) {
      c.tile = 0;
      if (++c.h == p.n_kv) {
        c.h = 0;
        do { ++c.b; } while (c.b < p.batch && pre[c.b + 1] == pre[c.b]);
        if (c.b < p.batch) {
          c.T = lens[c.b];
          c.ntile = (pre[c.b + 1] - pre[c.b]) / p.n_kv;
        }
      }
    }
  };

  if (n_my > 0 && warp == 0) {
    // ------------------------------------------------------------ producer
    const uint64_t policy = l2_evict_first_policy();
    TileCursor c;
    locate(t0, c);
    int qb = -1, qh = -1;
    uint4 qreg[QCH];
    int pt_b = -1, pt_base = 0, pt_val = -1, pt_next = -1;
    int issued = 0, done_ok = 1;
    int pre_k = 0;   // tiles whose keys were requested before the wait
    if (early) {
      TileCursor pc;
      locate(t0, pc);
      pre_k = min(kStages, n_my);
      for (int k = 0; k < pre_k; ++k) {
        if (lane == 0) mbar_expect_tx(&full[k], KBYTES);
        __syncwarp();
        if (lane < HALVES) {
          const int y = (pc.b * p.n_kv + pc.h) * p.t_max + pc.tile * kTileT;
          tma_load_2d(sbase + k * STAGE + lane * (kTileT * 128), &kmap, lane * 64, y, &full[k], policy);
        }
        advance(pc);
      }
      pdl_wait();
    }
    for (int k = 0; k < n_my; ++k) {
      const int s = k % kStages;
      const uint32_t ph = (uint32_t)(k / kStages) & 1u;
      if (!__all_sync(0xffffffffu, mbar_wait(&empty[s], ph ^ 1u))) {
        done_ok = 0;
        break;
      }
      if (c.b != qb || c.h != qh) {   // the group's queries as bf16 hi / lo rows
        qb = c.b;
        qh = c.h;
#pragma unroll
        for (int m = 0; m < QCH; ++m) {
          const int cid = lane + 32 * m;   // chunk: half, row, 8-channel column
          const int half = cid / (kN * 8), r = (cid / 8) % kN, col = cid % 8;
          float x[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) x[e] = 0.f;
          const int g = r < G ? r : r - G;
          if (r < 2 * G) {
            float v[8];
            if (p.qraw) {   // page bounds: [min(q, 0), max(q, 0)] of the current query
              constexpr int DQ = D / 2;
              const int ch = half * 64 + col * 8;
              const size_t off = (size_t)(c.b * p.n_q_heads + c.h * G + g) * DQ + (ch < DQ ? ch : ch - DQ);
              if (p.qraw_f32) {
                const float4 a0 = *reinterpret_cast<const float4*>(static_cast<const float*>(p.qraw) + off);
                const float4 a1 = *reinterpret_cast<const float4*>(static_cast<const float*>(p.qraw) + off + 4);
                v[0] = a0.x; v[1] = a0.y; v[2] = a0.z; v[3] = a0.w;
                v[4] = a1.x; v[5] = a1.y; v[6] = a1.z; v[7] = a1.w;
              } else {
                const uint4 u = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.qraw) + off);
                float2 f[4];
                Elem<__nv_bfloat16>::unpack(u, f);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  v[2 * e] = f[e].x;
                  v[2 * e + 1] = f[e].y;
                }
              }
#pragma unroll
              for (int e = 0; e < 8; ++e) v[e] = ch < DQ ? fminf(v[e], 0.f) : fmaxf(v[e], 0.f);
            } else {
              const float* src = p.qpred + ((size_t)(c.b * p.n_q_heads + c.h * G + g)) * D + half * 64 + col * 8;
              const float4 a0 = *reinterpret_cast<const float4*>(src);
              const float4 a1 = *reinterpret_cast<const float4*>(src + 4);
              v[0] = a0.x; v[1] = a0.y; v[2] = a0.z; v[3] = a0.w;
              v[4] = a1.x; v[5] = a1.y; v[6] = a1.z; v[7] = a1.w;
            }
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const float q = v[e] * p.scale;
              const float hi = __bfloat162float(__float2bfloat16_rn(q));
              x[e] = r < G ? hi : q - hi;
            }
          }
          qreg[m] = make_uint4(bf16x2_bits(x[0], x[1]), bf16x2_bits(x[2], x[3]), bf16x2_bits(x[4], x[5]),
                               bf16x2_bits(x[6], x[7]));
        }
      }
      uint8_t* st = smem + s * STAGE;
#pragma unroll
      for (int m = 0; m < QCH; ++m) {
        const int cid = lane + 32 * m;
        const int half = cid / (kN * 8), r = (cid / 8) % kN, col = cid % 8;
        *reinterpret_cast<uint4*>(st + KBYTES + half * (kN * 128) + r * 128 + ((col ^ (r & 7)) << 4)) = qreg[m];
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (k < pre_k) {   // the keys are on their way: only the queries were missing
        if (lane == 0) mbar_arrive(&full[s]);
        ++issued;
        advance(c);
        continue;
      }
      if (lane == 0) mbar_arrive_expect_tx(&full[s], KBYTES);
      __syncwarp();
      const uint32_t sdst = sbase + s * STAGE;
      if (p.page_size == 0) {
        if (lane < HALVES) {
          const int y = (c.b * p.n_kv + c.h) * p.t_max + c.tile * kTileT;
          tma_load_2d(sdst + lane * (kTileT * 128), &kmap, lane * 64, y, &full[s], policy);
        }
      } else {   // 16-token pages: one 16-row box per page and half
        // page-table window: lane l holds entry pt_base + l of row pt_b; the next
        // window is loaded one window ahead, so table lookups stay off the
        // critical path
        const int lp0 = c.tile * 8;
        if (c.b != pt_b || lp0 < pt_base || lp0 + 8 > pt_base + 32) {
          if (c.b == pt_b && lp0 == pt_base + 32) {
            pt_val = pt_next;
          } else {
            const int e = lp0 + lane;
            pt_val = e < p.max_pages ? p.page_table[(size_t)c.b * p.max_pages + e] : -1;
          }
          pt_b = c.b;
          pt_base = lp0;
          const int e = lp0 + 32 + lane;
          pt_next = e < p.max_pages ? p.page_table[(size_t)c.b * p.max_pages + e] : -1;
        }
        const int pg = lane & 7, half = lane >> 3;
        int page = __shfl_sync(0xffffffffu, pt_val, lp0 - pt_base + pg);
        if (lane < 8 * HALVES) {
          if ((lp0 + pg) * 16 >= c.T) {
            page = 0;   // past the sequence: any valid page keeps the byte count
          } else if (page < 0 || page >= p.n_pages) {
            flag_status(ASP_DEV_BAD_PAGE);
            page = 0;   // keeps the byte count; the rows' scores are not meaningful
          }
          tma_load_2d(sdst + half * (kTileT * 128) + pg * (16 * 128), &kmap, half * 64,
                      (page * p.n_kv + c.h) * 16, &full[s], policy);
        }
      }
      ++issued;
      advance(c);
    }
    if (!done_ok) {   // a wait ran out: give the copies in flight a bounded chance to land
      for (int k = issued; k < pre_k; ++k)   // requested early, never completed by an arrival
        if (lane == 0) mbar_arrive(&full[k % kStages]);
      const int hi = max(issued, pre_k);
      for (int k = max(0, hi - kStages); k < hi; ++k) mbar_wait(&full[k % kStages], (uint32_t)(k / kStages) & 1u);
    }
  } else if (n_my > 0 && warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    for (int k = 0; k < n_my; ++k) {
      const int s = k % kStages;
      const uint32_t ph = (uint32_t)(k / kStages) & 1u;
      const int a = k & 1;
      const uint32_t aph = (uint32_t)(k >> 1) & 1u;
      if (!__all_sync(0xffffffffu, mbar_wait(&tempty[a], aph ^ 1u))) break;
      if (!__all_sync(0xffffffffu, mbar_wait(&full[s], ph))) break;
      tc_fence_after();
      if (lane == 0) {
        const uint32_t st = sbase + s * STAGE;
#pragma unroll
        for (int kk = 0; kk < KSTEPS; ++kk) {
          const int half = kk / 4, k4 = kk % 4;
          const uint64_t adesc = sw128_desc(st + half * (kTileT * 128) + k4 * 32);
          const uint64_t bdesc = sw128_desc(st + KBYTES + half * (kN * 128) + k4 * 32);
          umma_bf16(tmem + a * 16, adesc, bdesc, kk > 0 ? 1u : 0u);
        }
        umma_commit(&empty[s]);
        umma_commit(&tfull[a]);
      }
      __syncwarp();
    }
  } else if (n_my > 0 && warp >= 2) {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;   // TMEM lanes 32*quarter .. +31 belong to this warp
    TileCursor c;
    locate(t0, c);
    for (int k = 0; k < n_my; ++k) {
      const int a = k & 1;
      const uint32_t aph = (uint32_t)(k >> 1) & 1u;
      if (!__all_sync(0xffffffffu, mbar_wait(&tfull[a], aph))) break;
      tc_fence_after();
      float v[16];
      tmem_ld16(tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(a * 16), v);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[a]);
      float m = v[0] + v[G];
#pragma unroll
      for (int g = 1; g < G; ++g) m = fmaxf(m, v[g] + v[G + g]);
      const int j = c.tile * kTileT + quarter * 32 + lane;
      const bool has = j < c.T;
      if (has) p.scores[(size_t)(c.b * p.n_kv + c.h) * p.t_max + j] = m;
      if (p.hist) {   // first radix pass of the selection, fused
        const uint32_t dig = order_key(m) >> kTopShift;
        const uint32_t hm = __ballot_sync(0xffffffffu, has);
        if (has) {
          const uint32_t peers = __match_any_sync(hm, dig);
          if (lane == __ffs(peers) - 1)
            atomicAdd(p.hist + (size_t)(c.b * p.n_kv + c.h) * kTopBins + dig, __popc(peers));
        }
      }
      advance(c);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
  }
}

// ---- paged caches of 8 KV heads in 16-token pages: one whole page per tile ----
//
// A page holds the 16 tokens of all 8 KV heads in 128 contiguous rows (32 KB for
// d = 128), so here a tile is one page, fetched by one 2-D TMA box per 64-channel
// half: the DRAM stream runs in whole pages, where tiles of one head would read
// a 4 KB slice of each of 8 scattered pages.  The MMA's N covers every query
// head of the sequence (hi and lo rows, N = 2 Hq); row r (head r / 16) keeps only
// its group's 2G columns.  The B operand changes only with the sequence, so it
// lives in two buffers outside the stages: the producer rewrites a buffer at a
// sequence change once the MMAs that read its previous contents are complete.
constexpr int kPageStages = 3;   // with two B buffers: fits beside a step-attention CTA
constexpr int kPageHkv = 8;

__host__ __device__ constexpr uint32_t tmem_alloc_cols(int cols) {
  return cols <= 32 ? 32u : cols <= 64 ? 64u : cols <= 128 ? 128u : cols <= 256 ? 256u : 512u;
}

template <int D, int G>
__global__ void __launch_bounds__(kThreadsTC, 1) score_tc_page_kernel(const __grid_constant__ CUtensorMap kmap,
                                                                      TcParams p) {
  constexpr int HQ = G * kPageHkv;
  constexpr int N = 2 * HQ;                           // MMA N: hi and lo rows of every query head
  constexpr int HALVES = D / 64;
  constexpr int KBYTES = kTileT * D * 2;              // one page of every head
  constexpr int BBYTES = HALVES * N * 128;            // one B buffer
  constexpr int KSTEPS = D / 16;
  constexpr int S = kPageStages;
  constexpr int W = 4 * G;                            // accumulator columns of one epilogue warp
  constexpr uint32_t TCOLS = tmem_alloc_cols(2 * N);
  constexpr uint32_t IDESC = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) |
                             ((uint32_t)(kTileT >> 4) << 24);
  constexpr int QCHUNKS = HALVES * N * 8;             // 16-byte chunks of a B buffer
  static_assert(KBYTES % 1024 == 0 && BBYTES % 1024 == 0 && N <= 256, "layout");

  extern __shared__ uint8_t smem_raw[];
  __shared__ uint32_t s_tmem;
  __shared__ int scratch[33];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  const uint32_t sbase = smem_u32(smem);
  uint8_t* bbuf = smem + S * KBYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(bbuf + 2 * BBYTES);
  uint64_t* empty = full + S;
  uint64_t* tfull = empty + S;
  uint64_t* tempty = tfull + 2;
  int* bsel = reinterpret_cast<int*>(tempty + 2);     // B buffer of each stage's tile
  int* pre = bsel + S;
  int* lens = pre + p.batch + 1;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 4);
    }
    mbar_init_fence();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&s_tmem)),
                 "r"(TCOLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  pdl_wait();
  pdl_trigger();
  for (int b = threadIdx.x; b < p.batch; b += blockDim.x) {
    int t = p.seq_lens ? p.seq_lens[b] : p.t_max;
    lens[b] = t < 0 ? 0 : (t > p.t_max ? p.t_max : t);
  }
  __syncthreads();
  cta_prefix_sum(p.batch, pre, [&](int b) { return (lens[b] + 15) / 16; }, scratch);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;

  const int total = pre[p.batch];
  const int chunk = (total + gridDim.x - 1) / gridDim.x;
  const int t0 = min(total, (int)blockIdx.x * chunk);
  const int t1 = min(total, t0 + chunk);
  const int n_my = t1 - t0;

  struct PageCursor {
    int b, lp, np, T;
  };
  auto locate = [&](int i, PageCursor& c) {
    int lo = 0, hi = p.batch;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (pre[mid] <= i) lo = mid; else hi = mid;
    }
    c.b = lo;
    c.T = lens[lo];
    c.np = pre[lo + 1] - pre[lo];
    c.lp = i - pre[lo];
  };
  auto advance = [&](PageCursor& c) {
    if (++c.lp == c.np) {
      c.lp = 0;
      do { ++c.b; } while (c.b < p.batch && pre[c.b + 1] == pre[c.b]);
      if (c.b < p.batch) {
        c.T = lens[c.b];
        c.np = pre[c.b + 1] - pre[c.b];
      }
    }
  };

  if (n_my > 0 && warp == 0) {
    // ------------------------------------------------------------ producer
    const uint64_t policy = l2_evict_first_policy();
    PageCursor c;
    locate(t0, c);
    int seg_b = -1, seg = -1;
    int last_k[2] = {-1, -1};   // last tile that read each B buffer
    int pt_b = -1, pt_base = 0, pt_val = -1, pt_next = -1;
    int issued = 0, done_ok = 1;
    for (int k = 0; k < n_my; ++k) {
      const int s = k % S;
      const uint32_t ph = (uint32_t)(k / S) & 1u;
      if (!__all_sync(0xffffffffu, mbar_wait(&empty[s], ph ^ 1u))) {
        done_ok = 0;
        break;
      }
      // the page: lane l holds table entry pt_base + l of row pt_b; the next 32
      // entries are loaded one window ahead
      if (c.b != pt_b || c.lp < pt_base || c.lp >= pt_base + 32) {
        if (c.b == pt_b && c.lp == pt_base + 32) {
          pt_val = pt_next;
        } else {
          const int e = c.lp + lane;
          pt_val = e < p.max_pages ? p.page_table[(size_t)c.b * p.max_pages + e] : -1;
        }
        pt_b = c.b;
        pt_base = c.lp;
        const int e = c.lp + 32 + lane;
        pt_next = e < p.max_pages ? p.page_table[(size_t)c.b * p.max_pages + e] : -1;
      }
      int page = __shfl_sync(0xffffffffu, pt_val, c.lp - pt_base);
      if (page < 0 || page >= p.n_pages) {
        if (lane == 0) flag_status(ASP_DEV_BAD_PAGE);
        page = 0;   // keeps the byte count; the page's scores are not meaningful
      }
      // the keys first (expected bytes without arriving), the queries after
      if (lane == 0) mbar_expect_tx(&full[s], KBYTES);
      __syncwarp();
      if (lane < HALVES)
        tma_load_2d(sbase + s * KBYTES + lane * (kTileT * 128), &kmap, lane * 64, page * kTileT, &full[s], policy);
      if (c.b != seg_b) {   // a new sequence: its queries into the other B buffer
        seg_b = c.b;
        ++seg;
        const int x = seg & 1;
        const int j = last_k[x];
        if (j >= 0 && k - j < S &&
            !__all_sync(0xffffffffu, mbar_wait(&empty[j % S], (uint32_t)(j / S) & 1u))) {
          if (lane == 0) mbar_arrive(&full[s]);   // lets the copy just issued complete the stage
          done_ok = 0;
          ++issued;
          break;
        }
        uint8_t* bx = bbuf + x * BBYTES;
        const float* qb = p.qpred + (size_t)c.b * HQ * D;
        constexpr int PER = QCHUNKS / 32;             // chunks per lane
        constexpr int BATCH = PER < 8 ? PER : 8;      // loads in flight per lane
#pragma unroll 1
        for (int m0 = 0; m0 < PER; m0 += BATCH) {
          float4 lo4[BATCH], hi4[BATCH];
#pragma unroll
          for (int u = 0; u < BATCH; ++u) {
            const int cid = lane + 32 * (m0 + u);   // chunk: half, row, 8-channel column
            const int half = cid / (N * 8), r = (cid / 8) % N, col = cid % 8;
            const int hq = (r / (2 * G)) * G + (r % (2 * G)) % G;
            const float* src = qb + (size_t)hq * D + half * 64 + col * 8;
            lo4[u] = *reinterpret_cast<const float4*>(src);
            hi4[u] = *reinterpret_cast<const float4*>(src + 4);
          }
#pragma unroll
          for (int u = 0; u < BATCH; ++u) {
            const int cid = lane + 32 * (m0 + u);
            const int half = cid / (N * 8), r = (cid / 8) % N, col = cid % 8;
            const bool is_lo = (r % (2 * G)) >= G;
            const float v[8] = {lo4[u].x, lo4[u].y, lo4[u].z, lo4[u].w, hi4[u].x, hi4[u].y, hi4[u].z, hi4[u].w};
            float x8[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const float q = v[e] * p.scale;
              const float h = __bfloat162float(__float2bfloat16_rn(q));
              x8[e] = is_lo ? q - h : h;
            }
            *reinterpret_cast<uint4*>(bx + half * (N * 128) + r * 128 + ((col ^ (r & 7)) << 4)) =
                make_uint4(bf16x2_bits(x8[0], x8[1]), bf16x2_bits(x8[2], x8[3]), bf16x2_bits(x8[4], x8[5]),
                           bf16x2_bits(x8[6], x8[7]));
          }
        }
      }
      const int x = seg & 1;
      last_k[x] = k;
      if (lane == 0) bsel[s] = x;
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&full[s]);
      ++issued;
      advance(c);
    }
    if (!done_ok) {   // a wait ran out: give the copies in flight a bounded chance to land
      for (int k = max(0, issued - S); k < issued; ++k) mbar_wait(&full[k % S], (uint32_t)(k / S) & 1u);
    }
  } else if (n_my > 0 && warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    for (int k = 0; k < n_my; ++k) {
      const int s = k % S;
      const uint32_t ph = (uint32_t)(k / S) & 1u;
      const int a = k & 1;
      const uint32_t aph = (uint32_t)(k >> 1) & 1u;
      if (!__all_sync(0xffffffffu, mbar_wait(&tempty[a], aph ^ 1u))) break;
      if (!__all_sync(0xffffffffu, mbar_wait(&full[s], ph))) break;
      tc_fence_after();
      if (lane == 0) {
        const uint32_t st = sbase + s * KBYTES;
        const uint32_t bq = sbase + S * KBYTES + bsel[s] * BBYTES;
#pragma unroll
        for (int kk = 0; kk < KSTEPS; ++kk) {
          const int half = kk / 4, k4 = kk % 4;
          const uint64_t adesc = sw128_desc(st + half * (kTileT * 128) + k4 * 32);
          const uint64_t bdesc = sw128_desc(bq + half * (N * 128) + k4 * 32);
          umma_bf16_i<IDESC>(tmem + a * N, adesc, bdesc, kk > 0 ? 1u : 0u);
        }
        umma_commit(&empty[s]);
        umma_commit(&tfull[a]);
      }
      __syncwarp();
    }
  } else if (n_my > 0 && warp >= 2) {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;   // TMEM lanes (tile rows) 32*quarter .. +31: heads 2q, 2q+1
    const int h = 2 * quarter + (lane >> 4);
    const int tok = lane & 15;
    PageCursor c;
    locate(t0, c);
    for (int k = 0; k < n_my; ++k) {
      const int a = k & 1;
      const uint32_t aph = (uint32_t)(k >> 1) & 1u;
      if (!__all_sync(0xffffffffu, mbar_wait(&tfull[a], aph))) break;
      tc_fence_after();
      float v[W];
      tmem_ld_w<W>(tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(a * N + quarter * W), v);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[a]);
      // this lane's head: columns [0, 2G) for lanes 0-15, [2G, 4G) for lanes 16-31
      const bool upper = lane >= 16;
      float m = -INFINITY;
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float hi = upper ? v[2 * G + g] : v[g];
        const float lo = upper ? v[3 * G + g] : v[G + g];
        m = fmaxf(m, hi + lo);
      }
      const int j = c.lp * 16 + tok;
      const bool has = j < c.T;
      const size_t row = (size_t)c.b * kPageHkv + h;
      if (has) p.scores[row * p.t_max + j] = m;
      if (p.hist) {   // first radix pass of the selection, fused
        const uint32_t dig = order_key(m) >> kTopShift;
        const uint32_t hm = __ballot_sync(0xffffffffu, has);
        if (has) {
          const uint32_t peers = __match_any_sync(hm, dig | (upper ? 0x10000u : 0u));
          if (lane == __ffs(peers) - 1) atomicAdd(p.hist + row * kTopBins + dig, __popc(peers));
        }
      }
      advance(c);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TCOLS));
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  }
  return fn;
}

template <int D, int G>
cudaError_t launch_tc_t(const KvView& kv, const TcParams& p, cudaStream_t s) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return cudaErrorNotSupported;
  CUtensorMap map;
  const cuuint64_t rows = kv.page_size ? (cuuint64_t)kv.n_pages * kv.n_kv * 16
                                       : (cuuint64_t)kv.batch * kv.n_kv * kv.t_max;
  const cuuint64_t dims[2] = {(cuuint64_t)D, rows};
  const cuuint64_t strides[1] = {(cuuint64_t)D * 2};
  const cuuint32_t box[2] = {64, kv.page_size ? 16u : (cuuint32_t)kTileT};
  const cuuint32_t estride[2] = {1, 1};
  if (enc(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(kv.k), dims, strides, box, estride,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  constexpr int STAGE = kTileT * D * 2 + (D / 64) * kN * 128;
  constexpr int S = stages_for(D, G);
  const size_t smem = 1024 + (size_t)S * STAGE + (2 * S + 4) * 8 + (2 * (size_t)p.batch + 1) * 4;
  auto kern = score_tc_kernel<D, G>;
  if (prepare_kernel((const void*)kern, smem, kThreadsTC) < 1) return cudaErrorInvalidConfiguration;
  return launch_pdl(kern, dim3(sm_count()), dim3(kThreadsTC), smem, s, map, p);
}

template <int D, int G>
cudaError_t launch_tc_page_t(const KvView& kv, const TcParams& p, cudaStream_t s) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return cudaErrorNotSupported;
  CUtensorMap map;
  const cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)kv.n_pages * kPageHkv * 16};
  const cuuint64_t strides[1] = {(cuuint64_t)D * 2};
  const cuuint32_t box[2] = {64, (cuuint32_t)kTileT};
  const cuuint32_t estride[2] = {1, 1};
  if (enc(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(kv.k), dims, strides, box, estride,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  constexpr int N = 2 * G * kPageHkv;
  constexpr int S = kPageStages;
  const size_t smem = 1024 + (size_t)S * kTileT * D * 2 + 2 * (size_t)(D / 64) * N * 128 + (2 * S + 4) * 8 +
                      (size_t)S * 4 + (2 * (size_t)p.batch + 1) * 4;
  auto kern = score_tc_page_kernel<D, G>;
  if (prepare_kernel((const void*)kern, smem, kThreadsTC) < 1) return cudaErrorInvalidConfiguration;
  return launch_pdl(kern, dim3(sm_count()), dim3(kThreadsTC), smem, s, map, p);
}

}  // namespace

bool score_tc_supported(const KvView& kv, int n_q_heads, const float* qpred) {
  const int G = n_q_heads / kv.n_kv;
  return !kv.kv_f32 && (kv.head_dim == 64 || kv.head_dim == 128) && (kv.page_size == 0 || kv.page_size == 16) &&
         (G == 1 || G == 2 || G == 4 || G == 8) && kv.batch <= 8192 &&
         (reinterpret_cast<uintptr_t>(qpred) & 15) == 0;
}

cudaError_t launch_score_tc(const float* qpred, int n_q_heads, const KvView& kv, float* scores, cudaStream_t s,
                            int32_t* hist, bool early) {
  TcParams p;
  p.qpred = qpred;
  p.qraw = nullptr;
  p.qraw_f32 = 0;
  p.len_div = 1;
  p.len_cap = kv.t_max;
  p.early = early ? 1 : 0;
  p.n_q_heads = n_q_heads;
  p.G = n_q_heads / kv.n_kv;
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
  if (kv.page_size == 16 && kv.n_kv == kPageHkv) {   // whole pages per tile
    switch (p.G * (kv.head_dim == 64 ? 1 : -1)) {
      case 1: return launch_tc_page_t<64, 1>(kv, p, s);
      case 2: return launch_tc_page_t<64, 2>(kv, p, s);
      case 4: return launch_tc_page_t<64, 4>(kv, p, s);
      case 8: return launch_tc_page_t<64, 8>(kv, p, s);
      case -1: return launch_tc_page_t<128, 1>(kv, p, s);
      case -2: return launch_tc_page_t<128, 2>(kv, p, s);
      case -4: return launch_tc_page_t<128, 4>(kv, p, s);
      case -8: return launch_tc_page_t<128, 8>(kv, p, s);
      default: return cudaErrorInvalidValue;
    }
  }
  switch (p.G * (kv.head_dim == 64 ? 1 : -1)) {
    case 1: return launch_tc_t<64, 1>(kv, p, s);
    case 2: return launch_tc_t<64, 2>(kv, p, s);
    case 4: return launch_tc_t<64, 4>(kv, p, s);
    case 8: return launch_tc_t<64, 8>(kv, p, s);
    case -1: return launch_tc_t<128, 1>(kv, p, s);
    case -2: return launch_tc_t<128, 2>(kv, p, s);
    case -4: return launch_tc_t<128, 4>(kv, p, s);
    case -8: return launch_tc_t<128, 8>(kv, p, s);
    default: return cudaErrorInvalidValue;
  }
}

// Page bounds on the tensor cores: meta [batch, n_kv, npm, 2, d] read as a
// contiguous cache of 2d-channel rows, one row per page.
bool quest_tc_supported(const KvView& kv, int n_q_heads, const void* q) {
  const int G = n_q_heads / kv.n_kv;
  return !kv.kv_f32 && (kv.head_dim == 64 || kv.head_dim == 128) && (G == 1 || G == 2 || G == 4 || G == 8) &&
         kv.batch <= 1024 && (reinterpret_cast<uintptr_t>(q) & 15) == 0;
}

cudaError_t launch_quest_score_tc(const void* q, int q_f32, int n_q_heads, const KvView& kv, const void* meta,
                                  int quest_page, float* page_scores, cudaStream_t s) {
  const int npm = (kv.t_max + quest_page - 1) / quest_page;
  TcParams p;
  p.qpred = nullptr;
  p.qraw = q;
  p.qraw_f32 = q_f32;
  p.len_div = quest_page;
  p.len_cap = kv.t_max;
  p.early = 0;
  p.n_q_heads = n_q_heads;
  p.G = n_q_heads / kv.n_kv;
  p.batch = kv.batch;
  p.n_kv = kv.n_kv;
  p.t_max = npm;   // rows per (sequence, head) in meta, and the page scores' row stride
  p.page_size = 0;
  p.max_pages = 0;
  p.n_pages = 0;
  p.page_table = nullptr;
  p.seq_lens = kv.seq_lens;
  p.scores = page_scores;
  p.hist = nullptr;
  p.scale = 1.0f / sqrtf((float)kv.head_dim);
  KvView mv = kv;   // the tensor map's view: rows of meta
  mv.k = meta;
  mv.page_size = 0;
  mv.t_max = npm;
  switch (p.G * (kv.head_dim == 64 ? 1 : -1)) {
    case 1: return launch_tc_t<128, 1>(mv, p, s);
    case 2: return launch_tc_t<128, 2>(mv, p, s);
    case 4: return launch_tc_t<128, 4>(mv, p, s);
    case 8: return launch_tc_t<128, 8>(mv, p, s);
    case -1: return launch_tc_t<256, 1>(mv, p, s);
    case -2: return launch_tc_t<256, 2>(mv, p, s);
    case -4: return launch_tc_t<256, 4>(mv, p, s);
    case -8: return launch_tc_t<256, 8>(mv, p, s);
    default: return cudaErrorInvalidValue;
  }
}

ASP_STATUS_READER(read_status_score_tc)

}  // namespace asp
