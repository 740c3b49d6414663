// Gated-DeltaNet variant of the declared qwen3_5_text backbone ("原地套圈" investigation §01):
// the q | k | v channels of the input projection pass through a short causal depthwise
// convolution and SiLU before the recurrence, value heads (Hv) may outnumber key heads
// (Hk; value head h reads key head h / (Hv / Hk)), and each head's output is normalised
// and gated: y = RMSNorm(o_h) * w * silu(z_h).
//
// Input projection rows: q (Hk*dk) | k (Hk*dk) | v (Hv*dv) | z (Hv*dv) | a (Hv) | b (Hv).
// The conv taps K; y_t[c] = silu(sum_j w[c][j] x_{t-(K-1)+j}[c]), with the K-1 inputs
// before a call's first token taken from the per-execution conv state [B][K-1][C]
// (C = 2*Hk*dk + Hv*dv channels, zero at sequence start).
//
// Kernels (all HBM-bound, one pass):
//   gdn_conv_prep_kernel   one warp per (token, unit): a unit is a q head, a k head (conv,
//                          SiLU, L2 norm, written once per value head that reads it), a v
//                          head (conv, SiLU), or the token's gates g = -softplus(a + a_bias),
//                          beta = sigmoid(b + b_bias);
//   conv_state_kernel      one thread per (sequence, channel): the last K-1 inputs become
//                          the new state (a thread owns its channel's column, so the update
//                          is in place without a hazard);
//   gated_norm_kernel      one warp per (token, value head).
#include "common.cuh"
#include "internal.h"

namespace lk {

template <typename T, int KC>
__global__ void __launch_bounds__(256) gdn_conv_prep_kernel(
    const T* __restrict__ P, int ld_p, const T* __restrict__ conv_w, const T* __restrict__ conv_state,
    const float* __restrict__ a_bias, const float* __restrict__ b_bias, T* __restrict__ q, T* __restrict__ k,
    T* __restrict__ v, float* __restrict__ g, float* __restrict__ beta, int B, int T_len, int Hk, int Hv, int dk,
    int dv, float eps) {
  const int lane = threadIdx.x & 31;
  const int units = 2 * Hk + Hv + 1;
  const long w = (long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (w >= (long)B * T_len * units) return;
  const long m = w / units;                          // token row b * T + t
  const int u = (int)(w % units);
  const int b = (int)(m / T_len), t = (int)(m % T_len);
  const int C = 2 * Hk * dk + Hv * dv;
  const int rep = Hv / Hk;
  if (u == 2 * Hk + Hv) {                            // gates of every value head
    const T* row = P + m * ld_p + C + Hv * dv;
    for (int h = lane; h < Hv; h += 32) {
      const float a = ldf(row + h) + a_bias[h];
      const float bb = ldf(row + Hv + h) + b_bias[h];
      g[m * Hv + h] = -(a > 20.f ? a : log1pf(expf(a)));
      beta[m * Hv + h] = 1.f / (1.f + expf(-bb));
    }
    return;
  }
  // channel range of this unit
  int c0, width;
  if (u < Hk) {
    c0 = u * dk;
    width = dk;
  } else if (u < 2 * Hk) {
    c0 = Hk * dk + (u - Hk) * dk;
    width = dk;
  } else {
    c0 = 2 * Hk * dk + (u - 2 * Hk) * dv;
    width = dv;
  }
  constexpr int MAXPER = 8;                          // width <= 256
  float y[MAXPER];
  float ss = 0.f;
  const int per = width / 32;
#pragma unroll
  for (int i = 0; i < MAXPER; ++i) {
    y[i] = 0.f;
    if (i >= per) break;
    const int c = c0 + lane + 32 * i;
    float acc = 0.f;
#pragma unroll
    for (int j = 0; j < KC; ++j) {
      const int tt = t - (KC - 1) + j;               // input time of tap j
      const float x = tt >= 0 ? ldf(P + ((long)b * T_len + tt) * ld_p + c)
                              : ldf(conv_state + ((long)b * (KC - 1) + (KC - 1) + tt) * C + c);
      acc = fmaf(ldf(conv_w + (long)c * KC + j), x, acc);
    }
    y[i] = acc / (1.f + expf(-acc));                 // SiLU
    ss += y[i] * y[i];
  }
  if (u < 2 * Hk) {                                  // q or k head: L2 norm, then one copy per value head
    const float inv = rsqrtf(warp_sum(ss) + eps);
    const int kh = u < Hk ? u : u - Hk;
    T* dst = (u < Hk ? q : k) + (m * Hv + (long)kh * rep) * dk;
    for (int r = 0; r < rep; ++r)
#pragma unroll
      for (int i = 0; i < MAXPER; ++i) {
        if (i >= per) break;
        stf(dst + (long)r * dk + lane + 32 * i, y[i] * inv);
      }
  } else {
    T* dst = v + (m * Hv + (u - 2 * Hk)) * dv;
#pragma unroll
    for (int i = 0; i < MAXPER; ++i) {
      if (i >= per) break;
      stf(dst + lane + 32 * i, y[i]);
    }
  }
}

template <typename T, int KC>
__global__ void conv_state_kernel(const T* __restrict__ P, int ld_p, T* __restrict__ conv_state, int B, int T_len,
                                  int C) {
  const long i = (long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (long)B * C) return;
  const int b = (int)(i / C), c = (int)(i % C);
  T* st = conv_state + (long)b * (KC - 1) * C + c;
  T old[KC - 1];
#pragma unroll
  for (int j = 0; j < KC - 1; ++j) old[j] = st[(long)j * C];
  // inputs before and in this call: x_ext[0 .. KC-2] = old state, x_ext[KC-1 + t] = P row t;
  // the new state is x_ext[T .. T + KC-2]
#pragma unroll
  for (int j = 0; j < KC - 1; ++j) {
    const int e = T_len + j;
    st[(long)j * C] = e < KC - 1 ? old[e] : P[((long)b * T_len + (e - (KC - 1))) * ld_p + c];
  }
}

template <typename T>
__global__ void __launch_bounds__(256) gated_norm_kernel(const T* o, const T* __restrict__ z, int ld_z,
                                                         const T* __restrict__ w, T* y, long M, int H, int dv,
                                                         float eps) {
  // o and y may be the same array: a warp reads its whole row before it writes it
  const int lane = threadIdx.x & 31;
  const long wi = (long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (wi >= M * H) return;
  const long m = wi / H;
  const int h = (int)(wi % H);
  const T* op = o + wi * dv;
  const T* zp = z + m * ld_z + (long)h * dv;
  constexpr int MAXPER = 8;
  const int per = dv / 32;
  float x[MAXPER];
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < MAXPER; ++i) {
    x[i] = 0.f;
    if (i >= per) break;
    x[i] = ldf(op + lane + 32 * i);
    ss += x[i] * x[i];
  }
  const float inv = rsqrtf(warp_sum(ss) / (float)dv + eps);
#pragma unroll
  for (int i = 0; i < MAXPER; ++i) {
    if (i >= per) break;
    const int j = lane + 32 * i;
    const float zz = ldf(zp + j);
    stf(y + wi * dv + j, x[i] * inv * ldf(w + j) * (zz / (1.f + expf(-zz))));
  }
}

bool gdn_variant_supported(int Hk, int Hv, int dk, int dv, int conv) {
  return Hk > 0 && Hv >= Hk && Hv % Hk == 0 && gdn_supported(dk, dv) && conv == 4;
}

cudaError_t gdn_conv_prep(const void* P, int ld_p, const void* conv_w, void* conv_state, const float* a_bias,
                          const float* b_bias, void* q, void* k, void* v, float* g, float* beta, int B, int T, int Hk,
                          int Hv, int dk, int dv, int conv, float eps, int dtype, cudaStream_t s) {
  if (B == 0 || T == 0) return cudaSuccess;
  if (!gdn_variant_supported(Hk, Hv, dk, dv, conv)) return cudaErrorNotSupported;
  constexpr int KC = 4;
  const int units = 2 * Hk + Hv + 1;
  const long warps = (long)B * T * units;
  const unsigned blocks = (unsigned)((warps + 7) / 8);
  const int C = 2 * Hk * dk + Hv * dv;
  if (dtype == BF16) {
    using TT = __nv_bfloat16;
    gdn_conv_prep_kernel<TT, KC><<<blocks, 256, 0, s>>>((const TT*)P, ld_p, (const TT*)conv_w, (const TT*)conv_state,
                                                        a_bias, b_bias, (TT*)q, (TT*)k, (TT*)v, g, beta, B, T, Hk,
                                                        Hv, dk, dv, eps);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    conv_state_kernel<TT, KC><<<(unsigned)(((long)B * C + 255) / 256), 256, 0, s>>>((const TT*)P, ld_p,
                                                                                   (TT*)conv_state, B, T, C);
  } else {
    gdn_conv_prep_kernel<float, KC><<<blocks, 256, 0, s>>>((const float*)P, ld_p, (const float*)conv_w,
                                                           (const float*)conv_state, a_bias, b_bias, (float*)q,
                                                           (float*)k, (float*)v, g, beta, B, T, Hk, Hv, dk, dv, eps);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    conv_state_kernel<float, KC><<<(unsigned)(((long)B * C + 255) / 256), 256, 0, s>>>((const float*)P, ld_p,
                                                                                      (float*)conv_state, B, T, C);
  }
  return cudaGetLastError();
}

cudaError_t gdn_gated_norm(const void* o, const void* z, int ld_z, const void* w, void* y, long M, int H, int dv,
                           float eps, int dtype, cudaStream_t s) {
  if (M == 0) return cudaSuccess;
  if (dv % 32 != 0 || dv > 256) return cudaErrorNotSupported;
  const unsigned blocks = (unsigned)((M * H + 7) / 8);
  if (dtype == BF16)
    gated_norm_kernel<__nv_bfloat16><<<blocks, 256, 0, s>>>((const __nv_bfloat16*)o, (const __nv_bfloat16*)z, ld_z,
                                                            (const __nv_bfloat16*)w, (__nv_bfloat16*)y, M, H, dv, eps);
  else
    gated_norm_kernel<float><<<blocks, 256, 0, s>>>((const float*)o, (const float*)z, ld_z, (const float*)w,
                                                    (float*)y, M, H, dv, eps);
  return cudaGetLastError();
}

}  // namespace lk
