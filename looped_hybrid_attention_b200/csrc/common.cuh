// Shared device/host helpers for the looped hybrid decoder kernels (sm_100a).
#pragma once
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include <mutex>
#include <set>
#include <utility>

namespace lk {

// ------------------------------------------------------------------ storage types
template <typename T> struct Io;
template <> struct Io<float> {
  static __device__ __forceinline__ float ld(const float* p) { return *p; }
  static __device__ __forceinline__ void st(float* p, float v) { *p = v; }
  static __device__ __forceinline__ float round(float v) { return v; }
};
template <> struct Io<__nv_bfloat16> {
  static __device__ __forceinline__ float ld(const __nv_bfloat16* p) { return __bfloat162float(*p); }
  static __device__ __forceinline__ void st(__nv_bfloat16* p, float v) { *p = __float2bfloat16(v); }
  static __device__ __forceinline__ float round(float v) { return __bfloat162float(__float2bfloat16(v)); }
};
template <typename T> __device__ __forceinline__ float ldf(const T* p) { return Io<T>::ld(p); }
template <typename T> __device__ __forceinline__ void stf(T* p, float v) { Io<T>::st(p, v); }

// 8 consecutive elements (16 B for bf16, 32 B for fp32) <-> 8 floats.
__device__ __forceinline__ void load8(const __nv_bfloat16* p, float* f) {
  uint4 u = *reinterpret_cast<const uint4*>(p);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) { float2 t = __bfloat1622float2(h[i]); f[2 * i] = t.x; f[2 * i + 1] = t.y; }
}
__device__ __forceinline__ void load8(const float* p, float* f) {
  float4 a = *reinterpret_cast<const float4*>(p), b = *reinterpret_cast<const float4*>(p + 4);
  f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w; f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}
__device__ __forceinline__ void store8(__nv_bfloat16* p, const float* f) {
  uint4 u;
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
  *reinterpret_cast<uint4*>(p) = u;
}
__device__ __forceinline__ void store8(float* p, const float* f) {
  *reinterpret_cast<float4*>(p) = make_float4(f[0], f[1], f[2], f[3]);
  *reinterpret_cast<float4*>(p + 4) = make_float4(f[4], f[5], f[6], f[7]);
}
// Round 8 floats to the storage type and back (what a store + reload would give).
template <typename T> __device__ __forceinline__ void round8(float* f) {
#pragma unroll
  for (int i = 0; i < 8; ++i) f[i] = Io<T>::round(f[i]);
}

// ------------------------------------------------------------------ reductions
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
// Block-wide sum; `red` must hold >= 32 floats. All threads get the result.
__device__ __forceinline__ float block_sum(float v, float* red) {
  int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
  v = warp_sum(v);
  __syncthreads();
  if (lane == 0) red[wid] = v;
  __syncthreads();
  float t = (threadIdx.x < (unsigned)nw) ? red[threadIdx.x] : 0.f;
  if (wid == 0) t = warp_sum(t);
  if (threadIdx.x == 0) red[0] = t;
  __syncthreads();
  return red[0];
}

__device__ __forceinline__ float sigmoidf_(float x) { return 1.f / (1.f + __expf(-x)); }
__device__ __forceinline__ float sigmoidf_acc(float x) { return 1.f / (1.f + expf(-x)); }

// ------------------------------------------------------------------ device error word
// Kernels that detect a bad input or give up a bounded wait record a code here
// instead of trapping; the host reads it with loop_device_error().
enum DeviceError : int {
  DEV_OK = 0,
  DEV_BAD_TOKEN = 1,      // a token id outside [0, vocab)
  DEV_WAIT_TIMEOUT = 2,   // an mbarrier wait exceeded its iteration limit
  DEV_BAD_POSITION = 3,   // a KV write past the slab capacity
};
extern __device__ int g_device_error;
__device__ __forceinline__ void set_device_error(int code) { atomicCAS(&g_device_error, 0, code); }

// Programmatic dependent launch: lets a kernel launched after this one as a programmatic
// dependent (the few-row projections) start its prologue and weight loads now.  The
// dependent still waits (griddepcontrol.wait) for this grid's completion before it reads
// what this grid writes; without such a dependent this is a no-op.
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

inline int ceil_div(long a, long b) { return (int)((a + b - 1) / b); }

// ------------------------------------------------------------------ host: launch set-up
// Raise a kernel's dynamic shared-memory limit once per (kernel, device): the attribute
// belongs to the current device, so a process that drives several GPUs sets it on each.
template <typename K>
inline cudaError_t set_smem_limit(K kernel, int bytes) {
  static std::mutex mu;
  static std::set<std::pair<const void*, int>> done;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const auto key = std::make_pair(reinterpret_cast<const void*>(kernel), dev);
  std::lock_guard<std::mutex> lock(mu);
  if (done.count(key)) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) done.insert(key);
  return e;
}

}  // namespace lk
