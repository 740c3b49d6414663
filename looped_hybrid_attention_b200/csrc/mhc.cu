// Two-stream mHC residual ("Loop-9B engineering teardown" §五, §六; "SenseNova-Loop-9B
// 是什么" §二): one kernel per layer boundary mixes the previous layer's output into
// the two streams, then computes the next layer's routing (FP32 logits, FP32
// Sinkhorn) and reads the layer input -- the streams cross HBM once per boundary.
//
// One warp per token.  Lane L owns elements [8L + 256c, 8L + 256c + 8) of each
// stream (16-byte accesses), so the 2x[d] stream pair and the [2d, 8] routing map
// are read fully coalesced.  The routing map (256 KiB at d = 4096) is L2-resident.
#include "common.cuh"
#include "internal.h"

namespace lk {

// 2x2 (or n x n, n <= 8) Sinkhorn in registers: rows then columns, `iters` times.
__device__ __forceinline__ void sinkhorn2(float m[4], int iters) {
  for (int it = 0; it < iters; ++it) {
    float r0 = m[0] + m[1], r1 = m[2] + m[3];
    m[0] /= r0; m[1] /= r0; m[2] /= r1; m[3] /= r1;
    float c0 = m[0] + m[2], c1 = m[1] + m[3];
    m[0] /= c0; m[2] /= c0; m[1] /= c1; m[3] /= c1;
  }
}

template <typename T>
__global__ void __launch_bounds__(256) mhc_kernel(int mode, const T* __restrict__ X_in, const T* __restrict__ F,
                                                  const float* __restrict__ coeffs_in,
                                                  const float* __restrict__ w_r, const float* __restrict__ b_r,
                                                  T* X_out, T* __restrict__ x_in, T* __restrict__ h_out,
                                                  float* __restrict__ coeffs_out, int N, int d, float eps,
                                                  int iters) {
  const int lane = threadIdx.x & 31;
  const long tok = (long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (tok >= N) return;

  float hp0 = 0.f, hp1 = 0.f, r00 = 0.f, r01 = 0.f, r10 = 0.f, r11 = 0.f;
  if (mode == MHC_MIX || mode == MHC_MERGE) {
    const float* c = coeffs_in + tok * 8;
    hp0 = c[2]; hp1 = c[3]; r00 = c[4]; r01 = c[5]; r10 = c[6]; r11 = c[7];
  }
  const T* X = (mode == MHC_OPEN) ? X_in + tok * d : X_in + tok * 2 * d;
  const T* Ft = F ? F + tok * d : nullptr;
  T* Xo = X_out ? X_out + tok * 2 * d : nullptr;

  float l[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  float ss = 0.f;
  for (int j = lane * 8; j < d; j += 256) {
    float y0[8], y1[8];
    if (mode == MHC_OPEN) {
      load8(X + j, y0);
#pragma unroll
      for (int i = 0; i < 8; ++i) y1[i] = y0[i];
    } else if (mode == MHC_ROUTE) {
      load8(X + j, y0);
      load8(X + d + j, y1);
    } else {
      float x0[8], x1[8], f[8];
      load8(X + j, x0);
      load8(X + d + j, x1);
      load8(Ft + j, f);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        y0[i] = r00 * x0[i] + r01 * x1[i] + hp0 * f[i];
        y1[i] = r10 * x0[i] + r11 * x1[i] + hp1 * f[i];
      }
      if (mode == MHC_MERGE) {
        float h[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) h[i] = 0.5f * (y0[i] + y1[i]);
        store8(h_out + tok * d + j, h);
        continue;
      }
      round8<T>(y0);
      round8<T>(y1);
    }
    if (Xo && mode != MHC_ROUTE) {
      store8(Xo + j, y0);
      store8(Xo + d + j, y1);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      ss += y0[i] * y0[i] + y1[i] * y1[i];
      const float4* w0 = reinterpret_cast<const float4*>(w_r + (long)(j + i) * 8);
      const float4* w1 = reinterpret_cast<const float4*>(w_r + (long)(d + j + i) * 8);
      float4 a0 = __ldg(w0), a1 = __ldg(w0 + 1), b0 = __ldg(w1), b1 = __ldg(w1 + 1);
      l[0] += y0[i] * a0.x + y1[i] * b0.x;
      l[1] += y0[i] * a0.y + y1[i] * b0.y;
      l[2] += y0[i] * a0.z + y1[i] * b0.z;
      l[3] += y0[i] * a0.w + y1[i] * b0.w;
      l[4] += y0[i] * a1.x + y1[i] * b1.x;
      l[5] += y0[i] * a1.y + y1[i] * b1.y;
      l[6] += y0[i] * a1.z + y1[i] * b1.z;
      l[7] += y0[i] * a1.w + y1[i] * b1.w;
    }
  }
  if (mode == MHC_MERGE) return;

  ss = warp_sum(ss);
#pragma unroll
  for (int o = 0; o < 8; ++o) l[o] = warp_sum(l[o]);
  const float inv = rsqrtf(ss / (float)(2 * d) + eps);
#pragma unroll
  for (int o = 0; o < 8; ++o) l[o] = l[o] * inv + b_r[o];

  const float pre0 = sigmoidf_acc(l[0]), pre1 = sigmoidf_acc(l[1]);
  float m[4];
  const float mx = fmaxf(fmaxf(l[4], l[5]), fmaxf(l[6], l[7]));
#pragma unroll
  for (int i = 0; i < 4; ++i) m[i] = expf(l[4 + i] - mx);
  sinkhorn2(m, iters);
  if (lane == 0) {
    float4* c = reinterpret_cast<float4*>(coeffs_out + tok * 8);
    c[0] = make_float4(pre0, pre1, 2.f * sigmoidf_acc(l[2]), 2.f * sigmoidf_acc(l[3]));
    c[1] = make_float4(m[0], m[1], m[2], m[3]);
  }
  // layer input from the streams as stored (this lane re-reads only what it wrote)
  const T* Xr = (mode == MHC_ROUTE) ? X : Xo;
  for (int j = lane * 8; j < d; j += 256) {
    float a[8], b[8], o[8];
    if (mode == MHC_OPEN) {
      load8(X + j, a);                    // both streams equal h
#pragma unroll
      for (int i = 0; i < 8; ++i) o[i] = (pre0 + pre1) * a[i];
    } else {
      load8(Xr + j, a);
      load8(Xr + d + j, b);
#pragma unroll
      for (int i = 0; i < 8; ++i) o[i] = pre0 * a[i] + pre1 * b[i];
    }
    store8(x_in + tok * d + j, o);
  }
}

cudaError_t mhc(int mode, const void* X_in, const void* F, const float* coeffs_in, const float* w_r,
                const float* b_r, void* X_out, void* x_in, void* h_out, float* coeffs_out, int N,
                int d, float eps, int iters, int dtype, cudaStream_t s) {
  if (N == 0) return cudaSuccess;
  const int warps = 8;
  dim3 grid((N + warps - 1) / warps);
  if (dtype == BF16)
    mhc_kernel<__nv_bfloat16><<<grid, warps * 32, 0, s>>>(
        mode, (const __nv_bfloat16*)X_in, (const __nv_bfloat16*)F, coeffs_in, w_r, b_r,
        (__nv_bfloat16*)X_out, (__nv_bfloat16*)x_in, (__nv_bfloat16*)h_out, coeffs_out, N, d, eps, iters);
  else
    mhc_kernel<float><<<grid, warps * 32, 0, s>>>(mode, (const float*)X_in, (const float*)F, coeffs_in,
                                                  w_r, b_r, (float*)X_out, (float*)x_in, (float*)h_out,
                                                  coeffs_out, N, d, eps, iters);
  return cudaGetLastError();
}

// Standalone FP32 Sinkhorn-Knopp: one thread per n x n matrix (n <= 8).
__global__ void sinkhorn_kernel(const float* __restrict__ L, float* __restrict__ out, int N, int n, int iters) {
  const long t = (long)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= N) return;
  float m[64];
  const float* x = L + t * n * n;
  float mx = -INFINITY;
  for (int i = 0; i < n * n; ++i) mx = fmaxf(mx, x[i]);
  for (int i = 0; i < n * n; ++i) m[i] = expf(x[i] - mx);
  for (int it = 0; it < iters; ++it) {
    for (int r = 0; r < n; ++r) {
      float sr = 0.f;
      for (int c = 0; c < n; ++c) sr += m[r * n + c];
      for (int c = 0; c < n; ++c) m[r * n + c] /= sr;
    }
    for (int c = 0; c < n; ++c) {
      float sc = 0.f;
      for (int r = 0; r < n; ++r) sc += m[r * n + c];
      for (int r = 0; r < n; ++r) m[r * n + c] /= sc;
    }
  }
  for (int i = 0; i < n * n; ++i) out[t * n * n + i] = m[i];
}

cudaError_t sinkhorn(const float* logits, float* out, int N, int n, int iters, cudaStream_t s) {
  if (N == 0) return cudaSuccess;
  sinkhorn_kernel<<<(N + 127) / 128, 128, 0, s>>>(logits, out, N, n, iters);
  return cudaGetLastError();
}

}  // namespace lk
