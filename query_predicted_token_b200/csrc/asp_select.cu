// asp_select.cu -- step 3: top-C selection per (sequence, KV head).
//
// The C largest scores of scores[0:T_b] (IEEE order, -0.0 == +0.0), ties at the
// threshold to the lowest index, written ascending.
//
// Two kernels, one 1024-thread CTA per row in both.  select_regs_kernel (the
// decode step's rows of up to 32K tokens, the first digit's histogram given by
// the key scan) is described at its definition below.  select_kernel serves
// longer rows and stand-alone calls: the row's 32-bit order keys live in shared
// memory (up to 48K keys; longer rows are re-read from L2 in every sweep), so
// no step needs another CTA.  When the first digit's histogram is given, the
// threshold digit is found while the row's scores are still loading, and every
// unit is classified and packed straight from registers: the row is read once
// and no key array is built, so rows longer than the shared memory take this
// path too (unless the survivors of the first digit overflow their slots).  Radix select from the most significant end with
// digits of 11, 11 and 10 bits: the first digit's histogram comes with the
// scores (the key scan counts it with global atomics while it streams the
// cache) or is built while the keys are loaded; later passes count only keys
// that still match the threshold prefix (warp-aggregated with ballot/match, one
// shared atomic per distinct digit); the search stops once the threshold bin
// holds exactly the number of tokens still needed (for continuous scores: after
// the second digit).  The ascending write-out is a stable compaction: each warp
// owns a contiguous run of keys, counts (and, when the keys are in shared
// memory, packs in place) the tokens above and at the threshold with ballots,
// one scan over the warps gives the offsets, and the indices are written with
// the lowest-index rule for ties.
#include "asp_common.cuh"
#include "asp_internal.h"

namespace asp {
namespace {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;
constexpr int kSmemKeys = 48 * 1024;   // 192 KB of keys
constexpr int kBins = kTopBins;        // widest digit: 11 bits
constexpr int kBpt = kBins / kThreads;
constexpr uint32_t kGtTag = 0x80000000u;

// The float whose order key is k (see order_key), for a bin edge k: a NaN
// pattern below the key of -inf gives -inf, one above the key of +inf gives NaN
// (so that no score compares >= it).
__device__ __forceinline__ float key_edge(uint32_t k) {
  const uint32_t u = (k & 0x80000000u) ? (k & 0x7fffffffu) : ~k;
  if ((u & 0x7fffffffu) > 0x7f800000u) return (k & 0x80000000u) ? __uint_as_float(0x7fc00000u) : -INFINITY;
  return __uint_as_float(u);
}

// A 16-byte load the compiler keeps in program order before later barriers, so
// that every load of a thread is in flight before it waits at one.
__device__ __forceinline__ float4 ld_issue(const float4* p) {
  float4 v;
  asm volatile("ld.global.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "l"(p));
  return v;
}

// FUSED: the first digit's histogram is given and the scores load as 16-byte
// vectors (the decode step's case); that kernel carries no code for the others.
template <bool FUSED>
__global__ void __launch_bounds__(kThreads, 1) select_kernel(SelectArgs a) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int row = blockIdx.x;
  const int b = row / a.rows_per_seq;
  pdl_wait();   // the scores (and their histogram) come from the previous kernel

  extern __shared__ __align__(16) uint32_t keys[];
  __shared__ int hist[2][kBins];
  __shared__ int wsum[kWarps];
  __shared__ int wg[kWarps], we[kWarps];
  __shared__ int s_digit, s_above, s_bincnt, s_last_sel, s_overflow;

  int T = a.seq_lens ? a.seq_lens[b] : a.t_max;
  T = T < 0 ? 0 : (T > a.t_max ? a.t_max : T);
  const int E = a.expand;
  const int n = (T + E - 1) / E;   // candidate units of this row
  const int out_stride = a.c_units * E;
  int32_t* out = a.idx + (size_t)row * out_stride;

  auto write_unit = [&](int u, int pos) {
    for (int e = 0; e < E; ++e) {
      const int tok = u * E + e;
      out[pos * E + e] = tok < T ? tok : -1;
    }
  };

  if (n <= a.c_units) {   // every unit chosen
    for (int u = tid; u < n; u += kThreads) write_unit(u, u);
    for (int i = n * E + tid; i < out_stride; i += kThreads) out[i] = -1;
    if (tid == 0) a.count[row] = T;
    return;
  }

  const bool cached = n <= a.key_cap;   // the whole row fits the shared-memory slots
  const float* srow = a.scores + (size_t)row * a.row_stride;

  // ---- load the keys (cached rows) and, without a given first histogram, count the top digit
  const bool own_h0 = a.hist0 == nullptr;
  int* h0 = hist[0];
  if (own_h0) {
    for (int i = tid; i < kBins; i += kThreads) h0[i] = 0;
    __syncthreads();
  }
  auto count_digit = [&](int* h, bool act, uint32_t dig) {
    const uint32_t am = __ballot_sync(0xffffffffu, act);
    if (act) {
      const uint32_t peers = __match_any_sync(am, dig);
      if (lane == __ffs(peers) - 1) atomicAdd(&h[dig], __popc(peers));
    }
  };
  // 16-byte rows: a row's last vector stays inside the row (row_stride is a multiple of 4)
  const bool vec = (a.row_stride & 3) == 0 && (reinterpret_cast<uintptr_t>(a.scores) & 15) == 0;
  // With the first histogram given, the threshold digit is found while the row's
  // scores load, and the units are classified and packed straight from registers.
  const bool fused = FUSED;
  bool nan_seen = false;   // a NaN score (invalid input) in the part of the row this thread read
  if (FUSED && !(!own_h0 && vec && a.key_cap >= kWarps * 4)) {   // the launch rule was not met
    if (tid == 0) flag_status(ASP_DEV_SELECT);
    return;
  }
  const bool keys_in_smem = cached && !fused;   // the key array is built (else keys are re-read from L2)
  auto key_at = [&](int i) -> uint32_t { return keys_in_smem ? keys[i] : order_key(srow[i]); };
  if (!fused && cached && vec) {
    const int n4 = (n + 3) >> 2;
    constexpr int U = 4;           // vectors per thread in flight
    for (int base = 0; base < n4; base += U * kThreads) {
      float4 f[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int i4 = base + u * kThreads + tid;
        f[u] = i4 < n4 ? reinterpret_cast<const float4*>(srow)[i4] : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int i4 = base + u * kThreads + tid;
        const uint32_t k4[4] = {order_key(f[u].x), order_key(f[u].y), order_key(f[u].z), order_key(f[u].w)};
        nan_seen |= i4 < n4 && (isnan(f[u].x) || isnan(f[u].y) || isnan(f[u].z) || isnan(f[u].w));
        if (i4 < n4) *reinterpret_cast<uint4*>(&keys[4 * i4]) = make_uint4(k4[0], k4[1], k4[2], k4[3]);
        if (own_h0) {
#pragma unroll
          for (int c = 0; c < 4; ++c) count_digit(h0, 4 * i4 + c < n, k4[c] >> kTopShift);
        }
      }
    }
  } else if (!fused && (cached || own_h0)) {
    for (int base = 0; base < n; base += kThreads) {
      const int i = base + tid;
      uint32_t key = 0u;
      if (i < n) {
        const float sv = srow[i];
        nan_seen |= isnan(sv);
        key = order_key(sv);
        if (cached) keys[i] = key;
      }
      if (own_h0) count_digit(h0, i < n, key >> kTopShift);
    }
  }
  if (!fused && __syncthreads_or(nan_seen) && tid == 0) flag_status(ASP_DEV_NAN_SCORE);

  // Finds the digit (of width nb) that holds the krem-th largest of the counted
  // keys, given this CTA's histogram h (or the row's global one).
  uint32_t prefix = 0u, mask = 0u;
  int krem = a.c_units;
  // This thread's bins of a histogram, highest digit first.
  auto bins_of = [&](const int* h, int nb, int (&v)[kBpt]) {
    const int bpt = nb / kThreads;
#pragma unroll
    for (int j = 0; j < kBpt; ++j) v[j] = j < bpt ? h[nb - 1 - (tid * bpt + j)] : 0;
  };
  auto find_digit_in = [&](const int (&v)[kBpt], int nb, int shift) -> bool {
    const int bpt = nb / kThreads;
    int local = 0;
#pragma unroll
    for (int j = 0; j < kBpt; ++j) local += v[j];
    // exclusive prefix of `local` over the CTA with one barrier: warp totals go to
    // wsum, then every warp scans the 32 totals itself
    int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    int wincl = wsum[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, wincl, o);
      if (lane >= o) wincl += y;
    }
    const int wbase = __shfl_sync(0xffffffffu, wincl - wsum[lane], warp);   // sum over the earlier warps
    const int excl = wbase + incl - local;
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
    // s_digit, s_above, s_bincnt and wsum are written again only after the next
    // search's first barrier, which every thread reaches after these reads
    const int digit = s_digit;
    krem -= s_above;
    prefix |= (uint32_t)digit << shift;
    mask |= ((uint32_t)nb - 1u) << shift;
    return s_bincnt == krem;
  };
  auto find_digit = [&](const int* h, int nb, int shift) -> bool {
    int v[kBpt];
    bins_of(h, nb, v);
    return find_digit_in(v, nb, shift);
  };

  // Warp w owns the contiguous units [w0, w1) (in 128-unit chunks when fused).
  const int R = fused ? ((((n + kWarps - 1) / kWarps) + 127) & ~127) : ((((n + kWarps - 1) / kWarps) + 31) & ~31);
  const int w0 = min(n, warp * R), w1 = min(n, w0 + R);
  const uint32_t lt_mask = (1u << lane) - 1u;
  // Warp w's packed list lives in the slots [pb, pe): its own range when the row
  // fits, else an equal share of the slots (a longer list overflows it, and the
  // row falls back to re-reading its scores in every pass).
  const int share = (a.key_cap / kWarps) & ~3;
  const int pb = (fused && !cached) ? warp * share : w0;
  const int pe = (fused && !cached) ? pb + share : w1;
  int* h1 = hist[1];
  int n_packed = 0;
  bool done;
  bool packed = cached;   // the packed lists hold every surviving unit
  uint32_t prefix0, mask0;
  // Packed lists that fill at most half of their slots keep the candidates' keys
  // at the slots' end (entry k at pe - 1 - k), so later passes need not re-read
  // the scores.
  bool kcache = false;
  if (fused) {
    // Lane l of a chunk holds units c0 + 4l .. c0 + 4l + 3 (one 16-byte load);
    // four ballots give every surviving unit its packed position, in order.
    constexpr int U = 8;   // chunks per warp in flight
    const float4* s4 = reinterpret_cast<const float4*>(srow);
    float4 f[U];
    auto load_chunks = [&](int c0) {
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int i = c0 + u * 128 + 4 * lane;
        f[u] = i < w1 ? ld_issue(s4 + (i >> 2)) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    };
    // the histogram's bins are requested ahead of the scores, so that they do not
    // queue behind the row's loads
    static_assert(kBpt == 2, "two bins of the first digit per thread");
    int hv[kBpt];
    {   // bins 2047 - 2 tid and 2046 - 2 tid: one 8-byte load, kept ahead of the row's loads
      const int* hp = a.hist0 + (size_t)row * kBins + (kBins - 2 - 2 * tid);
      asm volatile("ld.global.v2.s32 {%0, %1}, [%2];" : "=r"(hv[1]), "=r"(hv[0]) : "l"(hp));
    }
    load_chunks(w0);
    for (int i = tid; i < kBins; i += kThreads) h1[i] = 0;   // ordered by find_digit's barriers
    if (tid == 0) s_overflow = 0;
    done = find_digit_in(hv, 2048, kTopShift);
    prefix0 = prefix;
    mask0 = mask;
    // The bin's edges as floats: a unit survives (is above the bin or in it) iff
    // score >= lo_f and is above it iff score >= hi_f.  An edge whose key is a NaN
    // pattern lies beyond an infinity: below -inf every score passes, above +inf
    // none does.  IEEE comparison already treats -0.0 as +0.0.
    const uint32_t digit0 = prefix0 >> kTopShift;
    const float lo_f = key_edge(prefix0);
    const float hi_f = digit0 + 1u < (uint32_t)kBins ? key_edge((digit0 + 1u) << kTopShift) : __uint_as_float(0x7fc00000u);
    const uint32_t lt = (1u << lane) - 1u;
    for (int c0 = w0; c0 < w1; c0 += U * 128) {
      if (c0 != w0) load_chunks(c0);
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int i = c0 + u * 128 + 4 * lane;
        const float fv[4] = {f[u].x, f[u].y, f[u].z, f[u].w};
        bool sv[4], gt[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          sv[c] = i + c < w1 && fv[c] >= lo_f;
          gt[c] = fv[c] >= hi_f;
          nan_seen |= i + c < w1 && isnan(fv[c]);
        }
        // rank of unit (lane, c) among the chunk's survivors: all of the lower
        // lanes' survivors, then this lane's earlier ones
        uint32_t bs[4];
        int before = 0, total = 0;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          bs[c] = __ballot_sync(0xffffffffu, sv[c]);
          before += __popc(bs[c] & lt);
          total += __popc(bs[c]);
        }
        if (n_packed + total <= pe - pb) {
          int pos = pb + n_packed + before;
#pragma unroll
          for (int c = 0; c < 4; ++c)
            if (sv[c]) keys[pos++] = (uint32_t)(i + c) | (gt[c] ? kGtTag : 0u);
        } else if (lane == 0) {
          s_overflow = 1;
        }
        n_packed += total;
      }
    }
    if (__syncthreads_or(nan_seen) && tid == 0) flag_status(ASP_DEV_NAN_SCORE);
    packed = s_overflow == 0;
    kcache = packed && 2 * n_packed <= pe - pb;
    if (!done && packed) {   // the candidates' second digit, from the packed lists
      constexpr int V = 4;   // entries per lane whose scores are in flight together
      for (int k0 = 0; k0 < n_packed; k0 += 32 * V) {
        uint32_t e[V];
        float sc[V];
#pragma unroll
        for (int v = 0; v < V; ++v) {
          const int k = k0 + v * 32 + lane;
          e[v] = k < n_packed ? keys[pb + k] : kGtTag;
          sc[v] = (e[v] & kGtTag) ? 0.f : srow[e[v]];
        }
#pragma unroll
        for (int v = 0; v < V; ++v) {
          const int k = k0 + v * 32 + lane;
          const bool cand = !(e[v] & kGtTag);
          const uint32_t key = order_key(sc[v]);
          if (kcache && cand) keys[pe - 1 - k] = key;
          count_digit(h1, cand, (key >> 10) & 2047u);
        }
      }
      __syncthreads();
    }
    if (!done && !packed) {   // overflow: count the candidates from the scores
      for (int base = 0; base < n; base += kThreads) {
        const int i = base + tid;
        const uint32_t key = i < n ? order_key(srow[i]) : 0u;
        count_digit(h1, i < n && (key & mask0) == prefix0, (key >> 10) & 2047u);
      }
      __syncthreads();
    }
  } else {
  // ---- first digit (11 bits)
  done = find_digit(own_h0 ? h0 : a.hist0 + (size_t)row * kBins, 2048, kTopShift);
  prefix0 = prefix;
  mask0 = mask;
  if (cached) {
    // One sweep packs, in order and in place, every unit above the first-digit
    // threshold (tagged kGtTag) or inside its bin (a candidate), and counts the
    // candidates' second digit.
    if (!done) {
      for (int i = tid; i < kBins; i += kThreads) h1[i] = 0;
      __syncthreads();
    }
    for (int i0 = w0; i0 < w1; i0 += 32) {
      const int i = i0 + lane;
      const uint32_t key = i < w1 ? keys[i] : 0u;
      const uint32_t mk = key & mask0;
      const bool gt = i < w1 && mk > prefix0;
      const bool cand = i < w1 && mk == prefix0;
      const uint32_t bs = __ballot_sync(0xffffffffu, gt || cand);
      if (gt || cand) keys[w0 + n_packed + __popc(bs & lt_mask)] = (uint32_t)i | (gt ? kGtTag : 0u);
      n_packed += __popc(bs);
      if (!done) count_digit(h1, cand, (key >> 10) & 2047u);
    }
    __syncthreads();
  } else if (!done) {
    for (int i = tid; i < kBins; i += kThreads) h1[i] = 0;
    __syncthreads();
    for (int base = 0; base < n; base += kThreads) {
      const int i = base + tid;
      const uint32_t key = i < n ? key_at(i) : 0u;
      count_digit(h1, i < n && (key & mask0) == prefix0, (key >> 10) & 2047u);
    }
    __syncthreads();
  }
  }
  // In the packed lists the tag bit marks units above the first-digit threshold;
  // candidates' keys come from the cache or are re-read from the scores (they
  // are few).
  auto packed_key = [&](uint32_t e, int k) -> uint32_t {
    if (e & kGtTag) return 0xffffffffu;
    return kcache ? keys[pe - 1 - k] : order_key(srow[e]);
  };

  // ---- second (11 bits) and third (10 bits) digits
  if (!done) {
    done = find_digit(h1, 2048, 10);
    if (!done) {
      int* h2 = hist[0];
      for (int i = tid; i < 1024; i += kThreads) h2[i] = 0;
      __syncthreads();
      if (packed) {
        for (int k0 = 0; k0 < n_packed; k0 += 32) {
          const int k = k0 + lane;
          const uint32_t e = k < n_packed ? keys[pb + k] : kGtTag;
          const uint32_t key = (e & kGtTag) ? 0u : packed_key(e, k);
          count_digit(h2, !(e & kGtTag) && (key & mask) == prefix, key & 1023u);
        }
      } else {
        for (int base = 0; base < n; base += kThreads) {
          const int i = base + tid;
          const uint32_t key = i < n ? key_at(i) : 0u;
          count_digit(h2, i < n && (key & mask) == prefix, key & 1023u);
        }
      }
      __syncthreads();
      find_digit(h2, 1024, 0);
    }
  }

  // ---- stable compaction: per-warp counts of units above and at the threshold,
  // a scan over the warps, then the ascending writes (lowest index first at ties)
  auto classify = [&](int i, uint32_t e, bool valid, bool& gt, bool& eq) {
    gt = eq = false;
    if (!valid) return;
    if (packed) {
      if (e & kGtTag) { gt = true; return; }
      const uint32_t mk = (mask == mask0) ? prefix0 : (packed_key(e, i - w0) & mask);   // first digit alone: whole bin
      gt = mk > prefix;
      eq = mk == prefix;
    } else {
      const uint32_t mk = key_at(i) & mask;
      gt = mk > prefix;
      eq = mk == prefix;
    }
  };
  const int span = packed ? n_packed : (w1 - w0);
  int c_gt = 0, c_eq = 0;
  for (int k0 = 0; k0 < span; k0 += 32) {
    const int k = k0 + lane;
    const bool valid = k < span;
    const uint32_t e = (packed && valid) ? keys[pb + k] : 0u;
    bool gt, eq;
    classify(w0 + k, e, valid, gt, eq);
    c_gt += __popc(__ballot_sync(0xffffffffu, gt));
    c_eq += __popc(__ballot_sync(0xffffffffu, eq));
  }
  if (lane == 0) {
    wg[warp] = c_gt;
    we[warp] = c_eq;
  }
  __syncthreads();
  if (warp == 0) {
    const int g = wg[lane], e = we[lane];
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
    wg[lane] = gi - g;   // exclusive offsets of the warps
    we[lane] = ei - e;
    if (lane == 0) s_last_sel = 0;
  }
  __syncthreads();
  int run_gt = wg[warp], run_eq = we[warp];
  for (int k0 = 0; k0 < span; k0 += 32) {
    const int k = k0 + lane;
    const bool valid = k < span;
    const uint32_t e = (packed && valid) ? keys[pb + k] : 0u;
    bool gt, eq;
    classify(w0 + k, e, valid, gt, eq);
    const uint32_t bg = __ballot_sync(0xffffffffu, gt);
    const uint32_t be = __ballot_sync(0xffffffffu, eq);
    const int Gj = run_gt + __popc(bg & lt_mask);
    const int Ej = run_eq + __popc(be & lt_mask);
    if (gt || (eq && Ej < krem)) {
      const int u = packed ? (int)(e & ~kGtTag) : w0 + k;
      const int pos = Gj + min(Ej, krem);
      if (pos < a.c_units) {
        write_unit(u, pos);
      } else {   // only reachable with a histogram that does not match the scores
        flag_status(ASP_DEV_SELECT);
      }
      if (u == n - 1) s_last_sel = 1;
    }
    run_gt += __popc(bg);
    run_eq += __popc(be);
  }
  __syncthreads();
  if (tid == 0) a.count[row] = out_stride - (s_last_sel ? (n * E - T) : 0);
}


// ---- rows of up to 32K scores with the first digit's histogram given ---------
//
// The decode step's rows at contexts up to 32K.  Warp 0 stages the row in shared
// memory with bulk copies while the CTA finds the threshold digit from the given
// histogram.  Then every lane classifies 32 consecutive scores (lane l of warp w:
// units 1024 w + 32 l .. + 31, its eight 16-byte vectors read in an order rotated
// by the lane, so that a warp's reads spread over all banks) against the float
// edges of the threshold bin, in one pass: two 32-bit masks per lane, in index
// order, of the units above the bin and of the candidates inside it.  The work is
// bound by instruction issue (32K scores on one SM), so that pass is the only one
// over every score; the candidates, a few percent of the row, are re-read from
// shared memory for their later digits (one shared atomic each) and their final
// class.  The output positions come from population counts, one scan over the
// lanes and one over the warps, and the writes walk the masks' set bits.
constexpr int kRegSpan = 1024;                             // units per warp
constexpr int kRegMaxUnits = kWarps * kRegSpan;            // 32768
constexpr uint32_t kRowPiece = 16384;                      // bytes per bulk copy

// The float at or above which a score's key reaches k + 2^shift (the upper edge of
// the bin of width 2^shift starting at k); NaN (no score) past the top key.
__device__ __forceinline__ float edge_above(uint32_t k, int shift) {
  const uint32_t e = k + (1u << shift);
  return e < k ? __uint_as_float(0x7fc00000u) : key_edge(e);
}

// max that propagates NaN (one operand NaN gives NaN)
__device__ __forceinline__ float max_nan(float a, float b) {
  float r;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
  return r;
}

// The digit (of width nb, bins taken two (or one) per thread, highest first) that
// holds the krem-th largest counted key; on return krem is the count still needed
// from that bin, and the result says whether the bin holds exactly that many.
__device__ __forceinline__ bool regs_find_digit(const int (&v)[2], int nb, int shift, int& krem, uint32_t& prefix,
                                                uint32_t& mask, int* wsum, int* s_res) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int bpt = nb / kThreads;
  const int local = v[0] + (bpt > 1 ? v[1] : 0);
  int incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  int wincl = wsum[lane];
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, wincl, o);
    if (lane >= o) wincl += y;
  }
  const int wbase = __shfl_sync(0xffffffffu, wincl - wsum[lane], warp);
  const int excl = wbase + incl - local;
  if (excl < krem && krem <= excl + local) {
    const int j = (bpt > 1 && excl + v[0] < krem) ? 1 : 0;
    s_res[0] = nb - 1 - (tid * bpt + j);   // the digit
    s_res[1] = j ? excl + v[0] : excl;     // counted keys above its bin
    s_res[2] = v[j];                       // keys in its bin
  }
  __syncthreads();
  // s_res and wsum are written again only after the next search's first barrier
  krem -= s_res[1];
  prefix |= (uint32_t)s_res[0] << shift;
  mask |= ((uint32_t)nb - 1u) << shift;
  return s_res[2] == krem;
}

__global__ void __launch_bounds__(kThreads, 1) select_regs_kernel(SelectArgs a) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int row = blockIdx.x;
  const int b = row / a.rows_per_seq;
  pdl_wait();   // the scores and their histogram come from the previous kernel

  extern __shared__ __align__(16) float srow_s[];   // the row, rounded up to 4 scores
  __shared__ int h1[kBins];    // second digit (11 bits)
  __shared__ int h2[1024];     // third digit (10 bits)
  __shared__ int wsum[kWarps];
  __shared__ int wg[kWarps], we[kWarps];
  __shared__ int s_res[3];
  __shared__ uint64_t s_bar;

  int T = a.seq_lens ? a.seq_lens[b] : a.t_max;
  T = T < 0 ? 0 : (T > a.t_max ? a.t_max : T);
  const int n = T;   // units are tokens (expand == 1)
  const int C = a.c_units;
  int32_t* out = a.idx + (size_t)row * C;
  if (n <= C) {   // every token chosen
    for (int u = tid; u < C; u += kThreads) out[u] = u < n ? u : -1;
    if (tid == 0) a.count[row] = n;
    return;
  }

  const float* srow = a.scores + (size_t)row * a.row_stride;
  const uint32_t row_bytes = (uint32_t)((n + 3) & ~3) * 4u;   // inside the row: row_stride is a multiple of 4
  if (warp == 0) {
    if (lane == 0) {
      mbar_init(&s_bar, 1);
      mbar_init_fence();
      mbar_arrive_expect_tx(&s_bar, row_bytes);
    }
    __syncwarp();
    for (uint32_t off = (uint32_t)lane * kRowPiece; off < row_bytes; off += 32u * kRowPiece)
      bulk_g2s(reinterpret_cast<uint8_t*>(srow_s) + off, reinterpret_cast<const uint8_t*>(srow) + off,
               min(kRowPiece, row_bytes - off), &s_bar);
  }
  // bins 2047 - 2 tid and 2046 - 2 tid of the first digit: one 8-byte load
  int hv[2];
  {
    const int* hp = a.hist0 + (size_t)row * kBins + (kBins - 2 - 2 * tid);
    asm volatile("ld.global.v2.s32 {%0, %1}, [%2];" : "=r"(hv[1]), "=r"(hv[0]) : "l"(hp));
  }
  for (int i = tid; i < kBins; i += kThreads) h1[i] = 0;   // ordered by the digit search's barriers
  for (int i = tid; i < 1024; i += kThreads) h2[i] = 0;
  uint32_t prefix = 0u, mask = 0u;
  int krem = C;
  bool done = regs_find_digit(hv, kBins, kTopShift, krem, prefix, mask, wsum, s_res);
  const float lo0 = key_edge(prefix), hi0 = edge_above(prefix, kTopShift);

  const bool landed = mbar_wait(&s_bar, 0);
  if (!__syncthreads_and(landed)) {   // ASP_DEV_WAIT_LIMIT recorded
    mbar_wait(&s_bar, 0);   // give the row's copies one more bounded wait before leaving
    return;
  }

  // ---- the one pass over the row: bit 4k + c of gk / ck is the unit of vector
  // (k + lane) mod 8, element c; a rotation by 4 (lane mod 8) puts the bits in index
  // order (bit j: unit base + j)
  const int base = warp * kRegSpan + lane * 32;
  uint32_t gmask = 0u, cmask = 0u;   // above the threshold bin / inside it
  bool nan_seen = false;
  if (base + 32 <= n) {
    const float4* r4 = reinterpret_cast<const float4*>(srow_s + base);
    float nacc = 0.f;
    uint32_t gk = 0u, ck = 0u;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const float4 x = r4[(k + lane) & 7];
      const float xv[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        nacc = max_nan(nacc, xv[c]);
        if (xv[c] >= hi0) gk |= 1u << (4 * k + c);
        if (xv[c] >= lo0) ck |= 1u << (4 * k + c);
      }
    }
    const int rot = 4 * (lane & 7);
    gmask = __funnelshift_l(gk, gk, rot);
    cmask = __funnelshift_l(ck, ck, rot) & ~gmask;
    nan_seen = isnan(nacc);
  } else if (base < n) {   // the lane that holds the end of the row
    for (int j = 0; j < n - base; ++j) {
      const float x = srow_s[base + j];
      nan_seen |= isnan(x);
      if (x >= hi0) gmask |= 1u << j;
      else if (x >= lo0) cmask |= 1u << j;
    }
  }
  // the candidates' later digits, from their scores in shared memory
  auto key_of = [&](int j) -> uint32_t { return order_key(srow_s[base + j]); };
  if (!done) {
    for (uint32_t m = cmask; m; m &= m - 1u) atomicAdd(&h1[(key_of(__ffs(m) - 1) >> 10) & 2047u], 1);
  }
  if (__syncthreads_or(nan_seen) && tid == 0) flag_status(ASP_DEV_NAN_SCORE);
  if (!done) {
    const int hb[2] = {h1[kBins - 1 - 2 * tid], h1[kBins - 2 - 2 * tid]};
    done = regs_find_digit(hb, kBins, 10, krem, prefix, mask, wsum, s_res);
    if (!done) {   // the third digit (10 bits): the rest of the key
      const uint32_t p1 = prefix, m1 = mask;
      for (uint32_t m = cmask; m; m &= m - 1u) {
        const uint32_t key = key_of(__ffs(m) - 1);
        if ((key & m1) == p1) atomicAdd(&h2[key & 1023u], 1);
      }
      __syncthreads();
      const int hb2[2] = {h2[1023 - tid], 0};
      regs_find_digit(hb2, 1024, 0, krem, prefix, mask, wsum, s_res);
    }
  }

  // ---- output: the units above the threshold, and the first krem of those at it
  // (all of them when the bin holds exactly krem), lowest index first, ascending
  uint32_t emask = cmask;   // at the threshold
  if (mask != (((uint32_t)kBins - 1u) << kTopShift)) {   // later digits: sort the candidates
    emask = 0u;
    for (uint32_t m = cmask; m; m &= m - 1u) {
      const int j = __ffs(m) - 1;
      const uint32_t mk = key_of(j) & mask;
      if (mk > prefix) gmask |= 1u << j;
      else if (mk == prefix) emask |= 1u << j;
    }
  }
  const int cg = __popc(gmask), ce = __popc(emask);
  int ig = cg, ie = ce;   // inclusive scans over the lanes
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int yg = __shfl_up_sync(0xffffffffu, ig, o);
    const int ye = __shfl_up_sync(0xffffffffu, ie, o);
    if (lane >= o) {
      ig += yg;
      ie += ye;
    }
  }
  if (lane == 31) {
    wg[warp] = ig;
    we[warp] = ie;
  }
  __syncthreads();
  if (warp == 0) {
    const int g = wg[lane], e = we[lane];
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
    wg[lane] = gi - g;   // exclusive offsets of the warps
    we[lane] = ei - e;
  }
  __syncthreads();
  int G = wg[warp] + ig - cg, E = we[warp] + ie - ce;   // units of each kind before this lane's
  uint32_t m = gmask | (E < krem ? emask : 0u);
  while (m) {
    const int j = __ffs(m) - 1;
    m &= m - 1u;
    const bool g = (gmask >> j) & 1u;
    const int pos = G + min(E, krem);
    if (pos < C) {
      out[pos] = base + j;
    } else {   // only reachable with a histogram that does not match the scores
      flag_status(ASP_DEV_SELECT);
    }
    if (g) ++G; else ++E;
    if (E >= krem) m &= gmask;   // the quota of ties is filled
  }
  if (tid == 0) a.count[row] = C;
}

}  // namespace

bool select_supported(int t_max, int expand) { return t_max >= 1 && expand >= 1; }

cudaError_t launch_select(const SelectArgs& a, cudaStream_t s) {
  const int len_max = (a.t_max + a.expand - 1) / a.expand;
  SelectArgs args = a;
  // shared-memory slots for keys or packed lists; the same for every row
  args.key_cap = len_max <= kSmemKeys ? ((len_max + 3) & ~3) : kSmemKeys;
  const size_t smem = (size_t)(args.key_cap > 0 ? args.key_cap : 4) * 4;
  const bool fused = a.hist0 != nullptr && (a.row_stride & 3) == 0 &&
                     (reinterpret_cast<uintptr_t>(a.scores) & 15) == 0 && args.key_cap >= kWarps * 4;
  if (fused && a.expand == 1 && a.t_max <= kRegMaxUnits) {
    const size_t row_smem = (size_t)((a.t_max + 3) & ~3) * 4;
    if (prepare_kernel((const void*)select_regs_kernel, row_smem, kThreads) < 1) return cudaErrorInvalidConfiguration;
    return launch_pdl(select_regs_kernel, dim3(args.n_rows), dim3(kThreads), row_smem, s, args);
  }
  auto kern = fused ? select_kernel<true> : select_kernel<false>;
  if (prepare_kernel((const void*)kern, smem, kThreads) < 1) return cudaErrorInvalidConfiguration;
  return launch_pdl(kern, dim3(args.n_rows), dim3(kThreads), smem, s, args);
}

ASP_STATUS_READER(read_status_select)

}  // namespace asp
