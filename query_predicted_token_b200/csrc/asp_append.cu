// asp_append.cu -- the new token's K and V appended to the cache.
//
// One CTA per sequence: every thread reads the sequence's length T before any
// write, the warps copy the KV heads' rows to position T (contiguous: row T of
// [b, h]; paged: row T % P of page page_table[b][T / P]) and, when page bounds
// are kept, fold the key into the bounds of the page that receives it (a token
// that opens a page sets them).  After a barrier one thread records T as the
// tail's start and advances the length to T + 1.  A sequence at capacity or
// whose page is not valid is left unchanged and ASP_DEV_BAD_PAGE is recorded.
#include "asp_common.cuh"
#include "asp_internal.h"

namespace asp {
namespace {

constexpr int kThreads = 256;

template <typename KT, int D>
__global__ void __launch_bounds__(kThreads) append_kernel(KvView kv, const KT* __restrict__ k_new,
                                                          const KT* __restrict__ v_new, int32_t* seq_lens,
                                                          int32_t* tail_begin, KT* meta, int quest_page, int npm) {
  using E = Elem<KT>;
  constexpr int CPV = E::kPerVec;           // elements per 16-byte vector
  constexpr int VPR = D / CPV;              // vectors per row
  const int b = blockIdx.x;
  const int T = seq_lens[b];
  const int cap = kv.page_size ? min(kv.t_max, kv.max_pages * kv.page_size) : kv.t_max;
  bool ok = T >= 0 && T < cap;
  int page = 0;
  if (ok && kv.page_size) {
    page = kv.page_table[(size_t)b * kv.max_pages + T / kv.page_size];
    ok = page >= 0 && page < kv.n_pages;
  }
  if (!ok) {
    if (threadIdx.x == 0) flag_status(ASP_DEV_BAD_PAGE);
    return;   // uniform over the CTA: every thread saw the same T and page
  }
  const int n = kv.n_kv * VPR;              // vectors of one token over the heads
  for (int i = threadIdx.x; i < n; i += kThreads) {
    const int h = i / VPR, c = i - h * VPR;
    size_t row;
    if (kv.page_size == 0) {
      row = ((size_t)b * kv.n_kv + h) * kv.t_max + T;
    } else {
      row = ((size_t)page * kv.n_kv + h) * kv.page_size + (T % kv.page_size);
    }
    const size_t src = ((size_t)b * kv.n_kv + h) * D + (size_t)c * CPV;
    const uint4 kv4 = *reinterpret_cast<const uint4*>(k_new + src);
    reinterpret_cast<uint4*>(const_cast<void*>(kv.k))[row * VPR + c] = kv4;
    reinterpret_cast<uint4*>(const_cast<void*>(kv.v))[row * VPR + c] = *reinterpret_cast<const uint4*>(v_new + src);
    if (meta) {
      KT* m = meta + (((size_t)b * kv.n_kv + h) * npm + T / quest_page) * 2 * D + (size_t)c * CPV;
      uint4 lo = kv4, hi = kv4;
      if (T % quest_page != 0) {   // fold into the page's bounds
        float2 f[CPV / 2], mn[CPV / 2], mx[CPV / 2];
        E::unpack(kv4, f);
        E::unpack(*reinterpret_cast<const uint4*>(m), mn);
        E::unpack(*reinterpret_cast<const uint4*>(m + D), mx);
        union {
          uint4 v;
          KT e[CPV];
        } l, u;
#pragma unroll
        for (int e = 0; e < CPV / 2; ++e) {
          l.e[2 * e] = E::from_float(fminf(mn[e].x, f[e].x));
          l.e[2 * e + 1] = E::from_float(fminf(mn[e].y, f[e].y));
          u.e[2 * e] = E::from_float(fmaxf(mx[e].x, f[e].x));
          u.e[2 * e + 1] = E::from_float(fmaxf(mx[e].y, f[e].y));
        }
        lo = l.v;
        hi = u.v;
      }
      *reinterpret_cast<uint4*>(m) = lo;
      *reinterpret_cast<uint4*>(m + D) = hi;
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    if (tail_begin) tail_begin[b] = T;
    seq_lens[b] = T + 1;
  }
}

template <typename KT, int D>
cudaError_t append_t(const KvView& kv, const void* k_new, const void* v_new, int32_t* seq_lens, int32_t* tail_begin,
                     void* meta, int quest_page, cudaStream_t s) {
  const int npm = meta ? (kv.t_max + quest_page - 1) / quest_page : 0;
  append_kernel<KT, D><<<kv.batch, kThreads, 0, s>>>(kv, static_cast<const KT*>(k_new), static_cast<const KT*>(v_new),
                                                     seq_lens, tail_begin, static_cast<KT*>(meta), quest_page, npm);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_append(const KvView& kv, const void* k_new, const void* v_new, int32_t* seq_lens,
                          int32_t* tail_begin, void* meta, int quest_page, cudaStream_t s) {
  if (kv.kv_f32)
    return kv.head_dim == 64 ? append_t<float, 64>(kv, k_new, v_new, seq_lens, tail_begin, meta, quest_page, s)
                             : append_t<float, 128>(kv, k_new, v_new, seq_lens, tail_begin, meta, quest_page, s);
  return kv.head_dim == 64
             ? append_t<__nv_bfloat16, 64>(kv, k_new, v_new, seq_lens, tail_begin, meta, quest_page, s)
             : append_t<__nv_bfloat16, 128>(kv, k_new, v_new, seq_lens, tail_begin, meta, quest_page, s);
}

namespace {
// One warp waits on a shared-memory barrier that nothing arrives on, with the
// library's bounded wait cut to `tries` attempts; it must give up, record
// ASP_DEV_WAIT_LIMIT and return, which *returned = 1 shows.
__global__ void wait_limit_kernel(uint32_t tries, int32_t* returned) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    mbar_init_fence();
  }
  __syncwarp();
  const bool ok = __all_sync(0xffffffffu, mbar_wait_n(&bar, 0u, tries));
  if (threadIdx.x == 0) *returned = ok ? 2 : 1;
}
}  // namespace

cudaError_t launch_wait_limit_check(int tries, int32_t* returned, cudaStream_t s) {
  wait_limit_kernel<<<1, 32, 0, s>>>((uint32_t)tries, returned);
  return cudaGetLastError();
}

ASP_STATUS_READER(read_status_append)

}  // namespace asp
