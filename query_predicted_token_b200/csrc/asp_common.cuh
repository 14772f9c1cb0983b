// asp_common.cuh -- device helpers shared by the libasp kernels (sm_100a).
//
// Bulk copies (cp.async.bulk, the 1-D form of the Tensor Memory Accelerator)
// move contiguous key/value rows from HBM into shared memory and signal an
// mbarrier with the number of bytes delivered.  Every wait on such a barrier is
// bounded: when the limit runs out the warp records ASP_DEV_WAIT_LIMIT in the
// device status word and stops instead of spinning forever.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "asp.h"

namespace asp {

// Device status word (ASP_DEV_* bits) of this translation unit.  Every kernel
// file defines a reader (ASP_STATUS_READER) that asp_device_status() calls.
namespace {
__device__ int g_dev_status = 0;
}

__device__ __forceinline__ void flag_status(int bits) { atomicOr(&g_dev_status, bits); }

// Defines `cudaError_t NAME(cudaStream_t, int* bits)`: ORs this translation
// unit's status word into *bits and clears it (synchronises the stream).
#define ASP_STATUS_READER(NAME)                                                                      \
  cudaError_t NAME(cudaStream_t s, int* bits) {                                                      \
    int v = 0;                                                                                       \
    static const int zero = 0;                                                                       \
    cudaError_t e = cudaMemcpyFromSymbolAsync(&v, g_dev_status, sizeof(int), 0, cudaMemcpyDeviceToHost, s); \
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);                                              \
    if (e == cudaSuccess && v) {                                                                     \
      e = cudaMemcpyToSymbolAsync(g_dev_status, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, s);   \
      if (e == cudaSuccess) e = cudaStreamSynchronize(s);                                            \
    }                                                                                                \
    *bits |= v;                                                                                      \
    return e;                                                                                        \
  }

// ---- shared-memory barriers -------------------------------------------------

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

// Makes barrier initialisation visible to the async proxy (bulk copies).
__device__ __forceinline__ void mbar_init_fence() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(1000u)   // suspend-time hint: 1 us
      : "memory");
  return ok != 0;
}

// Bounded wait: about 2^20 tries of at most ~1 us each, i.e. at most ~1 s.
constexpr uint32_t kWaitTries = 1u << 20;

// Waits for the barrier phase of `parity`, giving up after `tries` attempts: then
// ASP_DEV_WAIT_LIMIT is recorded and false returned.
__device__ __forceinline__ bool mbar_wait_n(uint64_t* bar, uint32_t parity, uint32_t tries) {
  for (uint32_t i = 0; i < tries; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  flag_status(ASP_DEV_WAIT_LIMIT);
  return false;
}

__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  return mbar_wait_n(bar, parity, kWaitTries);
}

// Orders earlier generic-proxy accesses of shared memory before later
// async-proxy writes into the same buffer.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// L2 policy for data read once (the key scan): evict first.
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

// 1-D bulk copy global -> shared, completion counted on `bar` in bytes.
// dst, src 16-byte aligned; bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void bulk_g2s_hint(void* dst, const void* src, uint32_t bytes, uint64_t* bar,
                                              uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], "
      "%4;" ::"r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// ---- programmatic dependent launch --------------------------------------------
// A kernel launched with programmatic stream serialisation may start while the
// previous kernel of its stream is still running; pdl_wait() blocks until that
// kernel has finished and its writes are visible (a no-op for normal launches).
// pdl_trigger() lets the next kernel of the stream launch early.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ---- selection keys ---------------------------------------------------------

// 32-bit key whose unsigned order is the IEEE order of the score (-0.0 == +0.0).
__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Width of the first radix digit of the selection (the key's top 11 bits).
constexpr int kTopBins = 2048;
constexpr int kTopShift = 21;

// ---- element conversion -----------------------------------------------------

// Two bf16 packed in a 32-bit word -> (low, high) as fp32 (exact).
__device__ __forceinline__ float2 bf16x2_to_float2(uint32_t w) {
  return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

template <typename T>
struct Elem;
template <>
struct Elem<float> {
  static constexpr int kBytes = 4;
  static constexpr int kPerVec = 4;   // elements per 16-byte vector
  // 16 bytes -> 2 float2 pairs (channel c, c+1), (c+2, c+3)
  __device__ __forceinline__ static void unpack(const uint4& v, float2* out) {
    out[0] = make_float2(__uint_as_float(v.x), __uint_as_float(v.y));
    out[1] = make_float2(__uint_as_float(v.z), __uint_as_float(v.w));
  }
  __device__ __forceinline__ static float load(const float* p) { return *p; }
  __device__ __forceinline__ static float from_float(float x) { return x; }
};
template <>
struct Elem<__nv_bfloat16> {
  static constexpr int kBytes = 2;
  static constexpr int kPerVec = 8;
  __device__ __forceinline__ static void unpack(const uint4& v, float2* out) {
    out[0] = bf16x2_to_float2(v.x);
    out[1] = bf16x2_to_float2(v.y);
    out[2] = bf16x2_to_float2(v.z);
    out[3] = bf16x2_to_float2(v.w);
  }
  __device__ __forceinline__ static float load(const __nv_bfloat16* p) { return __bfloat162float(*p); }
  __device__ __forceinline__ static __nv_bfloat16 from_float(float x) { return __float2bfloat16_rn(x); }
};

// ---- warp reduce-scatter ----------------------------------------------------
//
// N partial sums per lane, summed over the LPR lanes of an aligned lane group
// (xor offsets LPR/2 .. 1).  At each level a lane keeps half of its values and
// trades the other half with its partner, so the total number of shuffles is
// about N instead of N * log2(LPR).  Afterwards a lane holds
//   N >= LPR: values [ (N/LPR) * l, (N/LPR) * (l + 1) ) in vals[0 .. N/LPR)
//   N <  LPR: value  l / (LPR/N) in vals[0] (shared by LPR/N lanes)
// where l = lane % LPR.
template <int N, int OFF>
struct ReduceScatter {
  __device__ __forceinline__ static void run(float* vals, int lane) {
    if constexpr (OFF >= 1) {
      if constexpr (N >= 2) {
        constexpr int H = N / 2;
        const bool upper = (lane & OFF) != 0;
#pragma unroll
        for (int i = 0; i < H; ++i) {
          const float send = upper ? vals[i] : vals[i + H];
          const float keep = upper ? vals[i + H] : vals[i];
          vals[i] = keep + __shfl_xor_sync(0xffffffffu, send, OFF);
        }
        ReduceScatter<H, OFF / 2>::run(vals, lane);
      } else {
        vals[0] += __shfl_xor_sync(0xffffffffu, vals[0], OFF);
        ReduceScatter<1, OFF / 2>::run(vals, lane);
      }
    }
  }
};

// pre[0] = 0, pre[i + 1] = pre[i] + f(i) for i < n; the whole CTA participates.
template <typename F>
__device__ void cta_prefix_sum(int n, int* pre, F f, int* scratch) {
  const int tid = threadIdx.x, nt = blockDim.x, lane = tid & 31, wid = tid >> 5, nw = nt >> 5;
  int carry = 0;
  if (tid == 0) pre[0] = 0;
  for (int base = 0; base < n; base += nt) {
    const int i = base + tid;
    int x = i < n ? f(i) : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) scratch[wid] = x;
    __syncthreads();
    if (wid == 0) {
      int w = lane < nw ? scratch[lane] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, w, o);
        if (lane >= o) w += y;
      }
      if (lane < nw) scratch[lane] = w;
    }
    __syncthreads();
    if (i < n) pre[i + 1] = carry + (wid > 0 ? scratch[wid - 1] : 0) + x;
    carry += scratch[nw - 1];
    __syncthreads();
  }
}

__device__ __forceinline__ int ceil_div(int a, int b) { return (a + b - 1) / b; }

}  // namespace asp
