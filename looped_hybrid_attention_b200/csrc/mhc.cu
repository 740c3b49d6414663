// Two-stream mHC residual ("Loop-9B engineering teardown" §五, §六; "SenseNova-Loop-9B
// 是什么" §二): one kernel per layer boundary mixes the previous layer's output into
// the two streams, then computes the next layer's routing (FP32 logits, FP32
// Sinkhorn) and reads the layer input -- the streams cross HBM once per boundary.
//
// A warp owns 4 consecutive tokens.  Lane L owns elements [8L + 256c, 8L + 256c + 8)
// of each stream (16-byte accesses).  The routing map is read through its transposed
// copy [8, 2d] (w_rt, kept by the model) so that, per output, the warp reads one
// contiguous 1 KiB run; each value loaded serves all 4 tokens.  The per-op entry
// point, which has only the [2d, 8] map, reads it directly.
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

template <typename T, int TPW, bool WT>
__global__ void __launch_bounds__(128) mhc_kernel(int mode, const T* __restrict__ X_in, const T* __restrict__ F,
                                                  const float* __restrict__ coeffs_in,
                                                  const float* __restrict__ w_r, const float* __restrict__ b_r,
                                                  T* X_out, T* __restrict__ x_in, T* __restrict__ h_out,
                                                  float* __restrict__ coeffs_out, int N, int d, float eps,
                                                  int iters) {
  // A warp owns TPW consecutive tokens, so each routing-map row it loads serves TPW tokens.
  const int lane = threadIdx.x & 31;
  const long tok0 = ((long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5)) * TPW;
  if (tok0 >= N) return;
  const int nt = (int)min((long)TPW, N - tok0);

  float hp0[TPW], hp1[TPW], r00[TPW], r01[TPW], r10[TPW], r11[TPW];
#pragma unroll
  for (int t = 0; t < TPW; ++t) {
    hp0[t] = hp1[t] = r00[t] = r01[t] = r10[t] = r11[t] = 0.f;
    if ((mode == MHC_MIX || mode == MHC_MERGE) && t < nt) {
      const float* c = coeffs_in + (tok0 + t) * 8;
      hp0[t] = c[2]; hp1[t] = c[3]; r00[t] = c[4]; r01[t] = c[5]; r10[t] = c[6]; r11[t] = c[7];
    }
  }
  const long xs = (mode == MHC_OPEN) ? d : 2L * d;          // row stride of X_in

  float l[TPW][8], ss[TPW];
#pragma unroll
  for (int t = 0; t < TPW; ++t) {
    ss[t] = 0.f;
#pragma unroll
    for (int o = 0; o < 8; ++o) l[t][o] = 0.f;
  }
  for (int j = lane * 8; j < d; j += 256) {
    float y0[TPW][8], y1[TPW][8];
#pragma unroll
    for (int t = 0; t < TPW; ++t) {
      const long tok = tok0 + t;
      if (t >= nt) {
#pragma unroll
        for (int i = 0; i < 8; ++i) y0[t][i] = y1[t][i] = 0.f;
        continue;
      }
      const T* X = X_in + tok * xs;
      if (mode == MHC_OPEN) {
        load8(X + j, y0[t]);
#pragma unroll
        for (int i = 0; i < 8; ++i) y1[t][i] = y0[t][i];
      } else if (mode == MHC_ROUTE) {
        load8(X + j, y0[t]);
        load8(X + d + j, y1[t]);
      } else {
        float x0[8], x1[8], f[8];
        load8(X + j, x0);
        load8(X + d + j, x1);
        load8(F + tok * d + j, f);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          y0[t][i] = r00[t] * x0[i] + r01[t] * x1[i] + hp0[t] * f[i];
          y1[t][i] = r10[t] * x0[i] + r11[t] * x1[i] + hp1[t] * f[i];
        }
        if (mode == MHC_MERGE) {
          float h[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) h[i] = 0.5f * (y0[t][i] + y1[t][i]);
          store8(h_out + tok * d + j, h);
          continue;
        }
        round8<T>(y0[t]);
        round8<T>(y1[t]);
      }
      if (mode != MHC_ROUTE) {
        T* Xo = X_out + tok * 2 * d;
        store8(Xo + j, y0[t]);
        store8(Xo + d + j, y1[t]);
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) ss[t] += y0[t][i] * y0[t][i] + y1[t][i] * y1[t][i];
    }
    if (mode == MHC_MERGE) continue;
    if (WT) {
      // transposed map: output o reads w_r[o][j .. j+8) and w_r[o][d+j .. d+j+8), coalesced
#pragma unroll
      for (int o = 0; o < 8; ++o) {
        const float4* wa = reinterpret_cast<const float4*>(w_r + (long)o * 2 * d + j);
        const float4* wb = reinterpret_cast<const float4*>(w_r + (long)o * 2 * d + d + j);
        const float4 a0 = __ldg(wa), a1 = __ldg(wa + 1), b0 = __ldg(wb), b1 = __ldg(wb + 1);
        const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
        const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
        for (int t = 0; t < TPW; ++t) {
          float acc = l[t][o];
#pragma unroll
          for (int i = 0; i < 8; ++i) acc += y0[t][i] * av[i] + y1[t][i] * bv[i];
          l[t][o] = acc;
        }
      }
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float4* w0 = reinterpret_cast<const float4*>(w_r + (long)(j + i) * 8);
        const float4* w1 = reinterpret_cast<const float4*>(w_r + (long)(d + j + i) * 8);
        const float4 a0 = __ldg(w0), a1 = __ldg(w0 + 1), b0 = __ldg(w1), b1 = __ldg(w1 + 1);
#pragma unroll
        for (int t = 0; t < TPW; ++t) {
          const float u = y0[t][i], v = y1[t][i];
          l[t][0] += u * a0.x + v * b0.x;
          l[t][1] += u * a0.y + v * b0.y;
          l[t][2] += u * a0.z + v * b0.z;
          l[t][3] += u * a0.w + v * b0.w;
          l[t][4] += u * a1.x + v * b1.x;
          l[t][5] += u * a1.y + v * b1.y;
          l[t][6] += u * a1.z + v * b1.z;
          l[t][7] += u * a1.w + v * b1.w;
        }
      }
    }
  }
  if (mode == MHC_MERGE) return;

#pragma unroll
  for (int t = 0; t < TPW; ++t) {
    if (t >= nt) break;
    const long tok = tok0 + t;
    const float inv = rsqrtf(warp_sum(ss[t]) / (float)(2 * d) + eps);
    float lt[8];
#pragma unroll
    for (int o = 0; o < 8; ++o) lt[o] = warp_sum(l[t][o]) * inv + b_r[o];
    const float pre0 = sigmoidf_acc(lt[0]), pre1 = sigmoidf_acc(lt[1]);
    float m[4];
    const float mx = fmaxf(fmaxf(lt[4], lt[5]), fmaxf(lt[6], lt[7]));
#pragma unroll
    for (int i = 0; i < 4; ++i) m[i] = expf(lt[4 + i] - mx);
    sinkhorn2(m, iters);
    if (lane == 0) {
      float4* c = reinterpret_cast<float4*>(coeffs_out + tok * 8);
      c[0] = make_float4(pre0, pre1, 2.f * sigmoidf_acc(lt[2]), 2.f * sigmoidf_acc(lt[3]));
      c[1] = make_float4(m[0], m[1], m[2], m[3]);
    }
    // layer input from the streams as stored (this lane re-reads only what it wrote)
    const T* Xr = (mode == MHC_ROUTE) ? X_in + tok * 2 * d : X_out + tok * 2 * d;
    for (int j = lane * 8; j < d; j += 256) {
      float a[8], bb[8], o[8];
      if (mode == MHC_OPEN) {
        load8(X_in + tok * d + j, a);       // both streams equal h
#pragma unroll
        for (int i = 0; i < 8; ++i) o[i] = (pre0 + pre1) * a[i];
      } else {
        load8(Xr + j, a);
        load8(Xr + d + j, bb);
#pragma unroll
        for (int i = 0; i < 8; ++i) o[i] = pre0 * a[i] + pre1 * bb[i];
      }
      store8(x_in + tok * d + j, o);
    }
  }
}

// Few tokens (decode): one CTA per token, threads split the hidden dimension, and the
// 9 routing sums are reduced across the block.
template <typename T>
__global__ void __launch_bounds__(512) mhc_token_kernel(int mode, const T* __restrict__ X_in, const T* __restrict__ F,
                                                        const float* __restrict__ coeffs_in,
                                                        const float* __restrict__ w_r, const float* __restrict__ b_r,
                                                        T* X_out, T* __restrict__ x_in, T* __restrict__ h_out,
                                                        float* __restrict__ coeffs_out, int d, float eps, int iters) {
  __shared__ float red[9][16];
  __shared__ float coef[4];
  const long tok = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5, nw = blockDim.x >> 5;
  float hp0 = 0.f, hp1 = 0.f, r00 = 0.f, r01 = 0.f, r10 = 0.f, r11 = 0.f;
  if (mode == MHC_MIX || mode == MHC_MERGE) {
    const float* c = coeffs_in + tok * 8;
    hp0 = c[2]; hp1 = c[3]; r00 = c[4]; r01 = c[5]; r10 = c[6]; r11 = c[7];
  }
  const T* X = (mode == MHC_OPEN) ? X_in + tok * d : X_in + tok * 2 * d;
  float l[8] = {0, 0, 0, 0, 0, 0, 0, 0}, ss = 0.f;
  for (int j = tid * 8; j < d; j += blockDim.x * 8) {
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
      load8(F + tok * d + j, f);
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
    if (mode != MHC_ROUTE) {
      store8(X_out + tok * 2 * d + j, y0);
      store8(X_out + tok * 2 * d + d + j, y1);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      ss += y0[i] * y0[i] + y1[i] * y1[i];
      const float4* w0 = reinterpret_cast<const float4*>(w_r + (long)(j + i) * 8);
      const float4* w1 = reinterpret_cast<const float4*>(w_r + (long)(d + j + i) * 8);
      const float4 a0 = __ldg(w0), a1 = __ldg(w0 + 1), b0 = __ldg(w1), b1 = __ldg(w1 + 1);
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
  if (lane == 0) {
    red[8][wid] = ss;
#pragma unroll
    for (int o = 0; o < 8; ++o) red[o][wid] = l[o];
  }
  __syncthreads();
  if (wid == 0) {
    float v[9];
#pragma unroll
    for (int o = 0; o < 9; ++o) v[o] = warp_sum(lane < nw ? red[o][lane] : 0.f);
    const float inv = rsqrtf(v[8] / (float)(2 * d) + eps);
    float lt[8];
#pragma unroll
    for (int o = 0; o < 8; ++o) lt[o] = v[o] * inv + b_r[o];
    const float pre0 = sigmoidf_acc(lt[0]), pre1 = sigmoidf_acc(lt[1]);
    float m[4];
    const float mx = fmaxf(fmaxf(lt[4], lt[5]), fmaxf(lt[6], lt[7]));
#pragma unroll
    for (int i = 0; i < 4; ++i) m[i] = expf(lt[4 + i] - mx);
    sinkhorn2(m, iters);
    if (lane == 0) {
      float4* c = reinterpret_cast<float4*>(coeffs_out + tok * 8);
      c[0] = make_float4(pre0, pre1, 2.f * sigmoidf_acc(lt[2]), 2.f * sigmoidf_acc(lt[3]));
      c[1] = make_float4(m[0], m[1], m[2], m[3]);
      coef[0] = pre0;
      coef[1] = pre1;
    }
  }
  __syncthreads();
  const float pre0 = coef[0], pre1 = coef[1];
  const T* Xr = (mode == MHC_ROUTE) ? X : X_out + tok * 2 * d;
  for (int j = tid * 8; j < d; j += blockDim.x * 8) {
    float a[8], bb[8], o[8];
    if (mode == MHC_OPEN) {
      load8(X + j, a);
#pragma unroll
      for (int i = 0; i < 8; ++i) o[i] = (pre0 + pre1) * a[i];
    } else {
      load8(Xr + j, a);
      load8(Xr + d + j, bb);
#pragma unroll
      for (int i = 0; i < 8; ++i) o[i] = pre0 * a[i] + pre1 * bb[i];
    }
    store8(x_in + tok * d + j, o);
  }
}

// w_r [8, 2d] from the [2d, 8] routing map (run once per looped layer by the model).
__global__ void transpose_wr_kernel(const float* __restrict__ w, float* __restrict__ wt, int rows) {
  const long i = (long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (long)rows * 8) return;
  const long r = i / 8, o = i % 8;
  wt[o * rows + r] = w[i];
}

cudaError_t transpose_wr(const float* w, float* wt, int two_d, cudaStream_t s) {
  const long n = (long)two_d * 8;
  transpose_wr_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(w, wt, two_d);
  return cudaGetLastError();
}

cudaError_t mhc(int mode, const void* X_in, const void* F, const float* coeffs_in, const float* w_r,
                const float* b_r, void* X_out, void* x_in, void* h_out, float* coeffs_out, int N,
                int d, float eps, int iters, int dtype, cudaStream_t s, const float* w_rt) {
  if (N == 0) return cudaSuccess;
  if (N < 1024) {           // few tokens: spread each token over a CTA
    const int threads = d >= 4096 ? 512 : (d >= 2048 ? 256 : 128);
    if (dtype == BF16)
      mhc_token_kernel<__nv_bfloat16><<<N, threads, 0, s>>>(
          mode, (const __nv_bfloat16*)X_in, (const __nv_bfloat16*)F, coeffs_in, w_r, b_r, (__nv_bfloat16*)X_out,
          (__nv_bfloat16*)x_in, (__nv_bfloat16*)h_out, coeffs_out, d, eps, iters);
    else
      mhc_token_kernel<float><<<N, threads, 0, s>>>(mode, (const float*)X_in, (const float*)F, coeffs_in, w_r, b_r,
                                                    (float*)X_out, (float*)x_in, (float*)h_out, coeffs_out, d, eps,
                                                    iters);
    return cudaGetLastError();
  }
  constexpr int TPW = 4, warps = 4;
  dim3 grid((unsigned)(((long)N + TPW * warps - 1) / (TPW * warps)));
  const bool wt = w_rt != nullptr;
  const float* wmap = wt ? w_rt : w_r;
#define MHC_LAUNCH(TT, W)                                                                                            \
  mhc_kernel<TT, TPW, W><<<grid, warps * 32, 0, s>>>(mode, (const TT*)X_in, (const TT*)F, coeffs_in, wmap, b_r,      \
                                                     (TT*)X_out, (TT*)x_in, (TT*)h_out, coeffs_out, N, d, eps, iters)
  if (dtype == BF16) {
    if (wt) MHC_LAUNCH(__nv_bfloat16, true); else MHC_LAUNCH(__nv_bfloat16, false);
  } else {
    if (wt) MHC_LAUNCH(float, true); else MHC_LAUNCH(float, false);
  }
#undef MHC_LAUNCH
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
