// Device helpers shared by the kernels: type widening/narrowing, reductions.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

namespace dg {

typedef __nv_bfloat16 bf16;

// Programmatic dependent launch: wait until the preceding kernel on the stream has
// completed and its writes are visible, then let the next kernel be scheduled.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_enter() {
  pdl_wait();
  pdl_trigger();
}

// Load with acquire semantics at GPU scope (pairs with a writer's fence + atomic).
__device__ __forceinline__ int ld_acquire(const int32_t* p) {
  int v;
  asm volatile("ld.acquire.gpu.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ float widen(float x) { return x; }
__device__ __forceinline__ float widen(bf16 x) { return __bfloat162float(x); }
__device__ __forceinline__ double widen(double x) { return x; }

template <class T> __device__ __forceinline__ T narrow(float x);
template <> __device__ __forceinline__ float narrow<float>(float x) { return x; }
template <> __device__ __forceinline__ bf16 narrow<bf16>(float x) { return __float2bfloat16_rn(x); }
template <> __device__ __forceinline__ double narrow<double>(float x) { return x; }
template <class T> __device__ __forceinline__ T narrow(double x);
template <> __device__ __forceinline__ double narrow<double>(double x) { return x; }
template <> __device__ __forceinline__ float narrow<float>(double x) { return (float)x; }
template <> __device__ __forceinline__ bf16 narrow<bf16>(double x) {
  return __float2bfloat16_rn((float)x);
}

__device__ __forceinline__ float dexp(float x) { return expf(x); }
__device__ __forceinline__ double dexp(double x) { return exp(x); }
__device__ __forceinline__ float dlog(float x) { return logf(x); }
__device__ __forceinline__ double dlog(double x) { return log(x); }
__device__ __forceinline__ float dsqrt(float x) { return sqrtf(x); }
__device__ __forceinline__ double dsqrt(double x) { return sqrt(x); }

template <class T> __device__ __forceinline__ T silu(T z) { return z / (T(1) + dexp(-z)); }

// 8 consecutive elements moved with 16-byte accesses (p 16-byte aligned).
template <class T> __device__ __forceinline__ void ld8(const T* p, T (&v)[8]) {
  static_assert((sizeof(T) * 8) % 16 == 0, "16-byte vectors");
#pragma unroll
  for (int i = 0; i < (int)(sizeof(T) * 8 / 16); ++i)
    reinterpret_cast<uint4*>(v)[i] = reinterpret_cast<const uint4*>(p)[i];
}
template <class T> __device__ __forceinline__ void st8(T* p, const T (&v)[8]) {
#pragma unroll
  for (int i = 0; i < (int)(sizeof(T) * 8 / 16); ++i)
    reinterpret_cast<uint4*>(p)[i] = reinterpret_cast<const uint4*>(v)[i];
}

template <class T> __device__ __forceinline__ T warp_sum(T v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

template <class T> __device__ __forceinline__ T warp_max(T v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Block-wide sum with a fixed reduction shape (deterministic). blockDim % 32 == 0.
template <class T> __device__ T block_sum(T v, T* red /* >= 32 */) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
  v = warp_sum(v);
  __syncthreads();
  if (lane == 0) red[wid] = v;
  __syncthreads();
  T r = (threadIdx.x < nw) ? red[threadIdx.x] : T(0);
  if (wid == 0) r = warp_sum(r);
  if (threadIdx.x == 0) red[0] = r;
  __syncthreads();
  r = red[0];
  __syncthreads();
  return r;
}

}  // namespace dg
