// Device-side helpers shared by the SureLock kernels (sm_100a).
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace sl {

typedef __nv_bfloat16 bf16;

// Error codes a kernel writes into the device error word.
enum : int { DEV_OK = 0, DEV_TIMEOUT_PRODUCER = 1, DEV_TIMEOUT_MMA = 2, DEV_TIMEOUT_EPI = 3,
             DEV_BAD_INDEX = 4 };

// Spin-wait limit for every wait on a barrier a kernel of this library can
// issue: after this many nanoseconds of globaltimer the wait gives up, the
// kernel records the failure and winds down instead of hanging the GPU.
constexpr unsigned long long WAIT_LIMIT_NS = 2000000000ull;

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(bf16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ bf16 from_f<bf16>(float x) { return __float2bfloat16_rn(x); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ int warp_sum_i(int v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ float silu_f(float x) { return x / (1.0f + __expf(-x)); }

// Programmatic dependent launch: every kernel of the step is launched with
// programmatic stream serialisation and waits for its predecessor's results
// with pdl_wait() before touching memory the predecessor writes (or reads).
// Light kernels (norms, finalize passes, merges) call pdl_trigger() right
// after that wait, so the next GEMM's CTAs become resident beside them and
// stream their weight tiles meanwhile; heavy kernels trigger once their main
// work is issued.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// 8 x bf16 <-> 16-byte vector
// Fire-and-forget L2 prefetch of this CTA's share of [ptr, ptr + bytes): the
// next kernel's weights, brought in while the running kernel leaves HBM idle.
// ptr 16-byte aligned; pieces of at most 64 KB.
__device__ __forceinline__ void l2_prefetch_share(const void *ptr, size_t bytes, int cta,
                                                  int ctas) {
  if (!ptr || bytes < 16) return;
  const size_t units = bytes >> 4;                        // 16-byte units
  const size_t per = (units + ctas - 1) / ctas;
  size_t u0 = per * (size_t)cta, u1 = u0 + per;
  if (u1 > units) u1 = units;
  const char *base = reinterpret_cast<const char *>(ptr);
  for (size_t u = u0; u < u1; u += 4096) {
    const uint32_t n = (uint32_t)((u1 - u < 4096 ? u1 - u : 4096) << 4);
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(base + (u << 4)), "r"(n)
                 : "memory");
  }
}

union Pack8 {
  uint4 u;
  bf16 h[8];
  __nv_bfloat162 h2[4];
};

}  // namespace sl
