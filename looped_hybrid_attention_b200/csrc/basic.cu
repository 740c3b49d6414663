// RMSNorm (+ fused residual add), token-embedding gather, greedy argmax.
// All three are HBM-bound: one pass over their inputs with 16-byte accesses.
#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"

namespace lk {

__device__ int g_device_error = 0;

int read_and_clear_device_error() {
  int v = 0, z = 0;
  cudaMemcpyFromSymbol(&v, g_device_error, sizeof(int));
  cudaMemcpyToSymbol(g_device_error, &z, sizeof(int));
  return v;
}

// y = x / sqrt(mean(x^2) + eps) * w, with x optionally replaced by x + r (and that sum
// written out).  One CTA per row; the row is staged in shared memory as fp32.
template <typename T>
__global__ void rmsnorm_kernel(const T* __restrict__ x, const T* __restrict__ r, T* __restrict__ sum_out,
                               const T* __restrict__ w, T* __restrict__ y, int d, long ldx, float eps) {
  pdl_trigger();
  extern __shared__ float row[];
  __shared__ float red[32];
  const long base = (long)blockIdx.x * d;
  const long xbase = (long)blockIdx.x * ldx;
  float ss = 0.f;
  for (int j = threadIdx.x * 8; j < d; j += blockDim.x * 8) {
    float a[8];
    load8(x + xbase + j, a);
    if (r) {
      float b[8];
      load8(r + base + j, b);
#pragma unroll
      for (int i = 0; i < 8; ++i) a[i] += b[i];
      round8<T>(a);                       // the sum is what is stored and re-read downstream
      if (sum_out) store8(sum_out + base + j, a);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) { row[j + i] = a[i]; ss += a[i] * a[i]; }
  }
  ss = block_sum(ss, red);
  const float inv = rsqrtf(ss / (float)d + eps);
  for (int j = threadIdx.x * 8; j < d; j += blockDim.x * 8) {
    float g[8], o[8];
    load8(w + j, g);
#pragma unroll
    for (int i = 0; i < 8; ++i) o[i] = row[j + i] * inv * g[i];
    store8(y + base + j, o);
  }
}

// Register-resident variant for d = 8 * blockDim.x * CH: every thread keeps its CH
// 8-element pieces (piece c at (c * blockDim.x + tid) * 8, so a warp's accesses are
// contiguous) in registers across the row reduction: one read and one write per element.
template <typename T, int CH>
__global__ void __launch_bounds__(256) rmsnorm_reg_kernel(const T* __restrict__ x, const T* __restrict__ r,
                                                          T* __restrict__ sum_out, const T* __restrict__ w,
                                                          T* __restrict__ y, int d, long ldx, float eps) {
  pdl_trigger();
  __shared__ float red[32];
  const long base = (long)blockIdx.x * d;
  const long xbase = (long)blockIdx.x * ldx;
  float a[CH][8];
  float ss = 0.f;
#pragma unroll
  for (int c = 0; c < CH; ++c) {
    const int j = (c * blockDim.x + threadIdx.x) * 8;
    load8(x + xbase + j, a[c]);
    if (r) {
      float b[8];
      load8(r + base + j, b);
#pragma unroll
      for (int i = 0; i < 8; ++i) a[c][i] += b[i];
      round8<T>(a[c]);                    // the sum is what is stored and re-read downstream
      if (sum_out) store8(sum_out + base + j, a[c]);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) ss += a[c][i] * a[c][i];
  }
  ss = block_sum(ss, red);
  const float inv = rsqrtf(ss / (float)d + eps);
#pragma unroll
  for (int c = 0; c < CH; ++c) {
    const int j = (c * blockDim.x + threadIdx.x) * 8;
    float g[8], o[8];
    load8(w + j, g);
#pragma unroll
    for (int i = 0; i < 8; ++i) o[i] = a[c][i] * inv * g[i];
    store8(y + base + j, o);
  }
}

// Self-test of the bounded-wait path: one thread waits on an mbarrier that nothing
// completes.  After `limit` clock cycles the wait gives up, records DEV_WAIT_TIMEOUT in the
// device error word and the kernel returns normally, as every bounded wait in the library
// does -- the host reads the code with loop_device_error and the context stays usable.
__global__ void wait_selftest_kernel(long long limit) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  const uint32_t b = tc::smem_u32(&bar);
  if (threadIdx.x == 0) {
    tc::mbar_init(b, 1);
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  if (threadIdx.x == 0) tc::mbar_wait(b, 0, &abort_flag, limit);   // phase 0 never completes
}

cudaError_t wait_selftest(long long limit, cudaStream_t s) {
  wait_selftest_kernel<<<1, 32, 0, s>>>(limit);
  return cudaGetLastError();
}

cudaError_t rmsnorm(const void* x, const void* r, void* sum_out, const void* w, void* y, int M,
                    int d, float eps, int dtype, cudaStream_t s, long ldx) {
  if (ldx <= 0) ldx = d;
  if (M == 0) return cudaSuccess;
  auto al16 = [](const void* p) { return ((uintptr_t)p % 16) == 0; };
  const bool aligned = al16(x) && al16(w) && al16(y) && (!r || al16(r)) && (!sum_out || al16(sum_out)) && ldx % 8 == 0;
  if (aligned && d % 8 == 0) {
    const int pieces = d / 8;                    // 8-element pieces per row
    int ch = 0, th = 0;
    if (pieces <= 256 && pieces % 32 == 0) { ch = 1; th = pieces; }
    else if (pieces % 256 == 0 && pieces / 256 <= 4) { ch = pieces / 256; th = 256; }
    if (ch) {
#define RMS_REG(TT, C) rmsnorm_reg_kernel<TT, C><<<M, th, 0, s>>>((const TT*)x, (const TT*)r, (TT*)sum_out, \
                                                                  (const TT*)w, (TT*)y, d, ldx, eps)
      if (dtype == BF16) {
        if (ch == 1) RMS_REG(__nv_bfloat16, 1); else if (ch == 2) RMS_REG(__nv_bfloat16, 2);
        else if (ch == 3) RMS_REG(__nv_bfloat16, 3); else RMS_REG(__nv_bfloat16, 4);
      } else {
        if (ch == 1) RMS_REG(float, 1); else if (ch == 2) RMS_REG(float, 2);
        else if (ch == 3) RMS_REG(float, 3); else RMS_REG(float, 4);
      }
#undef RMS_REG
      return cudaGetLastError();
    }
  }
  int threads = d >= 4096 ? 256 : 128;
  size_t smem = (size_t)d * sizeof(float);
  if (dtype == BF16)
    rmsnorm_kernel<__nv_bfloat16><<<M, threads, smem, s>>>(
        (const __nv_bfloat16*)x, (const __nv_bfloat16*)r, (__nv_bfloat16*)sum_out,
        (const __nv_bfloat16*)w, (__nv_bfloat16*)y, d, ldx, eps);
  else
    rmsnorm_kernel<float><<<M, threads, smem, s>>>((const float*)x, (const float*)r, (float*)sum_out,
                                                   (const float*)w, (float*)y, d, ldx, eps);
  return cudaGetLastError();
}

// out[m] = E[ids[m]]: 16-byte vector copies; bad ids write zeros and flag the error word.
template <typename T>
__global__ void embed_kernel(const int32_t* __restrict__ ids, const T* __restrict__ E, T* __restrict__ out,
                             int d, int vocab) {
  const int m = blockIdx.x;
  const int id = ids[m];
  const bool ok = id >= 0 && id < vocab;
  if (!ok && threadIdx.x == 0) set_device_error(DEV_BAD_TOKEN);
  const int vec = 16 / sizeof(T);
  const uint4* src = reinterpret_cast<const uint4*>(E + (long)(ok ? id : 0) * d);
  uint4* dst = reinterpret_cast<uint4*>(out + (long)m * d);
  for (int j = threadIdx.x; j < d / vec; j += blockDim.x) dst[j] = ok ? src[j] : make_uint4(0, 0, 0, 0);
}

cudaError_t embed(const int32_t* ids, const void* E, void* out, int M, int d, int vocab, int dtype,
                  cudaStream_t s) {
  if (M == 0) return cudaSuccess;
  if (dtype == BF16)
    embed_kernel<__nv_bfloat16><<<M, 128, 0, s>>>(ids, (const __nv_bfloat16*)E, (__nv_bfloat16*)out, d, vocab);
  else
    embed_kernel<float><<<M, 128, 0, s>>>(ids, (const float*)E, (float*)out, d, vocab);
  return cudaGetLastError();
}

// Greedy token: argmax over one row of logits per CTA, lowest index on ties (NaN never wins).
__device__ __forceinline__ void better(float& bv, int& bi, float v, int i) {
  if (v > bv || (v == bv && i < bi)) { bv = v; bi = i; }
}

__global__ void argmax_kernel(const float* __restrict__ logits, int32_t* __restrict__ next, int V) {
  const float* row = logits + (long)blockIdx.x * V;
  float bv = -INFINITY;
  int bi = 0x7fffffff;
  for (int j = threadIdx.x; j < V; j += blockDim.x) better(bv, bi, row[j], j);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    float v = __shfl_xor_sync(0xffffffffu, bv, o);
    int i = __shfl_xor_sync(0xffffffffu, bi, o);
    better(bv, bi, v, i);
  }
  __shared__ float sv[32];
  __shared__ int si[32];
  int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  if (lane == 0) { sv[wid] = bv; si[wid] = bi; }
  __syncthreads();
  if (wid == 0) {
    int nw = blockDim.x >> 5;
    bv = lane < nw ? sv[lane] : -INFINITY;
    bi = lane < nw ? si[lane] : 0x7fffffff;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      float v = __shfl_xor_sync(0xffffffffu, bv, o);
      int i = __shfl_xor_sync(0xffffffffu, bi, o);
      better(bv, bi, v, i);
    }
    if (lane == 0) next[blockIdx.x] = bi == 0x7fffffff ? 0 : bi;
  }
}

cudaError_t argmax(const float* logits, int32_t* next, int B, int V, cudaStream_t s) {
  if (B == 0) return cudaSuccess;
  argmax_kernel<<<B, 1024, 0, s>>>(logits, next, V);
  return cudaGetLastError();
}

}  // namespace lk
