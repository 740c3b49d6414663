// Gated-DeltaNet ("Loop-9B engineering teardown" §三: a constant-size recurrent
// state updated with a gate and the delta rule).  Per sequence b and head h:
//   S <- exp(g_t) S;  S <- S + beta_t (v_t - S k_t) k_t^T;  o_t = scale * S q_t
// with S [dv, dk] fp32.
//
// gdn_chunk_kernel processes C = 64 tokens at a time in the UT-transform form
// (exact re-association of the recurrence; G = chunk-local cumulative log decay,
// gamma = exp(G)):
//   A_rs = beta_r exp(G_r - G_s) k_r.k_s  (s < r)
//   (I + A) [W | U'] = [beta*gamma*K | beta*V]         (forward substitution)
//   U  = U' - W S^T
//   O  = scale * (gamma * Q S^T + (Q K^T o exp(G_r - G_s) o [s <= r]) U)
//   S <- exp(G_C) S + U^T (exp(G_C - G) * K)
// Rows of S are independent, so each CTA owns DVS rows of one (b, h) and walks
// the chunks in order; the dv split gives B*H*dv/DVS CTAs.  All decay factors are
// exp of non-positive numbers, so nothing overflows.
#include "common.cuh"
#include "internal.h"

namespace lk {

// ------------------------------------------------------------------ prep
// One warp per (token, head): L2-normalise q and k, copy v, gates g and beta.
template <typename T>
__global__ void gdn_prep_kernel(const T* __restrict__ P, int ld_p, const float* __restrict__ a_bias,
                                const float* __restrict__ b_bias, T* __restrict__ q, T* __restrict__ k,
                                T* __restrict__ v, float* __restrict__ g, float* __restrict__ beta, int M,
                                int H, int dk, int dv, float eps) {
  const int lane = threadIdx.x & 31;
  const long w = (long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (w >= (long)M * H) return;
  const long m = w / H;
  const int h = (int)(w % H);
  const T* row = P + m * ld_p;
  const T* qs = row + h * dk;
  const T* ks = row + H * dk + h * dk;
  const T* vs = row + 2 * H * dk + h * dv;
  float sq = 0.f, sk = 0.f;
  for (int j = lane; j < dk; j += 32) {
    float a = ldf(qs + j), b = ldf(ks + j);
    sq += a * a;
    sk += b * b;
  }
  sq = rsqrtf(warp_sum(sq) + eps);
  sk = rsqrtf(warp_sum(sk) + eps);
  T* qo = q + w * dk;
  T* ko = k + w * dk;
  T* vo = v + w * dv;
  for (int j = lane; j < dk; j += 32) {
    stf(qo + j, ldf(qs + j) * sq);
    stf(ko + j, ldf(ks + j) * sk);
  }
  for (int j = lane; j < dv; j += 32) vo[j] = vs[j];
  if (lane == 0) {
    float a = ldf(row + 2 * H * dk + H * dv + h) + a_bias[h];
    float b = ldf(row + 2 * H * dk + H * dv + H + h) + b_bias[h];
    float sp = a > 20.f ? a : log1pf(expf(a));    // softplus
    g[w] = -sp;
    beta[w] = 1.f / (1.f + expf(-b));
  }
}

cudaError_t gdn_prep(const void* P, int ld_p, const float* a_bias, const float* b_bias, void* q,
                     void* k, void* v, float* g, float* beta, int M, int H, int dk, int dv,
                     float eps, int dtype, cudaStream_t s) {
  if (M == 0) return cudaSuccess;
  const int warps = 8;
  dim3 grid((unsigned)(((long)M * H + warps - 1) / warps));
  if (dtype == BF16)
    gdn_prep_kernel<__nv_bfloat16><<<grid, warps * 32, 0, s>>>(
        (const __nv_bfloat16*)P, ld_p, a_bias, b_bias, (__nv_bfloat16*)q, (__nv_bfloat16*)k,
        (__nv_bfloat16*)v, g, beta, M, H, dk, dv, eps);
  else
    gdn_prep_kernel<float><<<grid, warps * 32, 0, s>>>((const float*)P, ld_p, a_bias, b_bias, (float*)q,
                                                       (float*)k, (float*)v, g, beta, M, H, dk, dv, eps);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ chunked scan
constexpr int GDN_C = 64;

template <int DK, int DVS>
struct GdnSmem {
  static constexpr int KP = DK + 1, CP = GDN_C + 1, UP = DVS + 1;
  static constexpr int floats = 3 * GDN_C * KP + 2 * GDN_C * CP + GDN_C * UP + DVS * KP + 3 * GDN_C;
  static constexpr size_t bytes = floats * sizeof(float);
};

template <typename T, int DK, int DVS>
__global__ void __launch_bounds__(256) gdn_chunk_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                        const T* __restrict__ v, const float* __restrict__ g,
                                                        const float* __restrict__ beta, float* __restrict__ state,
                                                        T* __restrict__ out, int T_len, int H, int DV, float scale) {
  constexpr int C = GDN_C;
  using L = GdnSmem<DK, DVS>;
  constexpr int KP = L::KP, CP = L::CP, UP = L::UP;
  extern __shared__ float sm[];
  float* Ks = sm;                    // [C][KP] keys
  float* Qs = Ks + C * KP;           // [C][KP] queries
  float* Ws = Qs + C * KP;           // [C][KP] beta*gamma*K, then W
  float* As = Ws + C * KP;           // [C][CP] strictly lower A
  float* Ps = As + C * CP;           // [C][CP] (q.k) exp(G_r - G_s), s <= r
  float* Us = Ps + C * CP;           // [C][UP] beta*V slice, then U
  float* Ss = Us + C * UP;           // [DVS][KP] state rows i0 .. i0+DVS
  float* Gs = Ss + DVS * KP;         // [C] cumulative log decay
  float* Bs = Gs + C;                // [C] beta
  float* Es = Bs + C;                // [C] exp(G_last - G_s)

  const int tid = threadIdx.x, nth = blockDim.x;
  const int i0 = blockIdx.x * DVS, h = blockIdx.y, b = blockIdx.z;
  float* Sg = state + (((long)b * H + h) * DV + i0) * DK;
  for (int idx = tid; idx < DVS * DK; idx += nth) Ss[(idx / DK) * KP + idx % DK] = Sg[idx];

  for (int c0 = 0; c0 < T_len; c0 += C) {
    const int n = min(C, T_len - c0);
    __syncthreads();
    // ---- load the chunk (rows past the end act as identity steps: k = 0, beta = 0, g = 0)
    for (int idx = tid; idx < C * DK; idx += nth) {
      const int r = idx / DK, j = idx % DK;
      float kv = 0.f, qv = 0.f;
      if (r < n) {
        const long base = (((long)b * T_len + c0 + r) * H + h) * DK + j;
        kv = ldf(k + base);
        qv = ldf(q + base);
      }
      Ks[r * KP + j] = kv;
      Qs[r * KP + j] = qv;
    }
    for (int idx = tid; idx < C * DVS; idx += nth) {
      const int r = idx / DVS, i = idx % DVS;
      Us[r * UP + i] = r < n ? ldf(v + (((long)b * T_len + c0 + r) * H + h) * DV + i0 + i) : 0.f;
    }
    if (tid < C) {
      const long gi = ((long)b * T_len + c0 + tid) * H + h;
      Gs[tid] = tid < n ? g[gi] : 0.f;
      Bs[tid] = tid < n ? beta[gi] : 0.f;
    }
    __syncthreads();
    if (tid < 32) {                  // inclusive prefix sum of the log decays (2 per lane)
      float a0 = Gs[2 * tid], a1 = a0 + Gs[2 * tid + 1];
      float x = a1;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        float y = __shfl_up_sync(0xffffffffu, x, o);
        if (tid >= o) x += y;
      }
      const float excl = x - a1;
      Gs[2 * tid] = excl + a0;
      Gs[2 * tid + 1] = x;
    }
    __syncthreads();
    const float Glast = Gs[C - 1];
    if (tid < C) Es[tid] = expf(Glast - Gs[tid]);
    // ---- A (strict lower) and P (lower incl. diagonal)
    for (int idx = tid; idx < C * C; idx += nth) {
      const int r = idx / C, s = idx % C;
      float a = 0.f, p = 0.f;
      if (s <= r) {
        float kk = 0.f, qk = 0.f;
        const float* kr = Ks + r * KP;
        const float* qr = Qs + r * KP;
        const float* ks = Ks + s * KP;
#pragma unroll 8
        for (int j = 0; j < DK; ++j) {
          kk = fmaf(kr[j], ks[j], kk);
          qk = fmaf(qr[j], ks[j], qk);
        }
        const float dec = expf(Gs[r] - Gs[s]);
        p = qk * dec;
        if (s < r) a = Bs[r] * dec * kk;
      }
      As[r * CP + s] = a;
      Ps[r * CP + s] = p;
    }
    // ---- right-hand sides
    for (int idx = tid; idx < C * DK; idx += nth) {
      const int r = idx / DK, j = idx % DK;
      Ws[r * KP + j] = Bs[r] * expf(Gs[r]) * Ks[r * KP + j];
    }
    for (int idx = tid; idx < C * DVS; idx += nth) {
      const int r = idx / DVS;
      Us[r * UP + idx % DVS] *= Bs[r];
    }
    __syncthreads();
    // ---- forward substitution (I + A) X = RHS, one column per thread
    for (int col = tid; col < DK + DVS; col += nth) {
      float* X = col < DK ? Ws + col : Us + (col - DK);
      const int st = col < DK ? KP : UP;
      for (int r = 1; r < C; ++r) {
        float acc = X[r * st];
        const float* ar = As + r * CP;
        for (int s2 = 0; s2 < r; ++s2) acc = fmaf(-ar[s2], X[s2 * st], acc);
        X[r * st] = acc;
      }
    }
    __syncthreads();
    // ---- U = U' - W S^T
    for (int idx = tid; idx < C * DVS; idx += nth) {
      const int r = idx / DVS, i = idx % DVS;
      const float* wr = Ws + r * KP;
      const float* si = Ss + i * KP;
      float acc = 0.f;
#pragma unroll 8
      for (int j = 0; j < DK; ++j) acc = fmaf(wr[j], si[j], acc);
      Us[r * UP + i] -= acc;
    }
    __syncthreads();
    // ---- O = scale * (gamma Q S^T + P U)
    for (int idx = tid; idx < C * DVS; idx += nth) {
      const int r = idx / DVS, i = idx % DVS;
      if (r >= n) continue;
      const float* qr = Qs + r * KP;
      const float* si = Ss + i * KP;
      float a1 = 0.f, a2 = 0.f;
#pragma unroll 8
      for (int j = 0; j < DK; ++j) a1 = fmaf(qr[j], si[j], a1);
      const float* pr = Ps + r * CP;
      for (int s2 = 0; s2 <= r; ++s2) a2 = fmaf(pr[s2], Us[s2 * UP + i], a2);
      const float o = scale * (expf(Gs[r]) * a1 + a2);
      stf(out + (((long)b * T_len + c0 + r) * H + h) * DV + i0 + i, o);
    }
    __syncthreads();
    // ---- S <- exp(G_last) S + U^T (exp(G_last - G) K)
    const float gl = expf(Glast);
    for (int idx = tid; idx < DVS * DK; idx += nth) {
      const int i = idx / DK, j = idx % DK;
      float acc = gl * Ss[i * KP + j];
      for (int s2 = 0; s2 < C; ++s2) acc = fmaf(Us[s2 * UP + i] * Es[s2], Ks[s2 * KP + j], acc);
      Ss[i * KP + j] = acc;
    }
  }
  __syncthreads();
  for (int idx = tid; idx < DVS * DK; idx += nth) Sg[idx] = Ss[(idx / DK) * KP + idx % DK];
}

bool gdn_supported(int dk, int dv) { return (dk == 64 && dv == 64) || (dk == 128 && dv == 128); }

template <typename T, int DK, int DVS>
static cudaError_t launch_chunk(const void* q, const void* k, const void* v, const float* g,
                                const float* beta, float* state, void* out, int B, int T_len, int H,
                                int dv, float scale, cudaStream_t s) {
  using L = GdnSmem<DK, DVS>;
  auto kern = gdn_chunk_kernel<T, DK, DVS>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::bytes);
  if (e != cudaSuccess) return e;
  dim3 grid(dv / DVS, H, B);
  kern<<<grid, 256, L::bytes, s>>>((const T*)q, (const T*)k, (const T*)v, g, beta, state, (T*)out, T_len, H,
                                   dv, scale);
  return cudaGetLastError();
}

cudaError_t gdn_chunk(const void* q, const void* k, const void* v, const float* g,
                      const float* beta, float* state, void* out, int B, int T, int H, int dk,
                      int dv, float scale, int dtype, cudaStream_t s) {
  if (T == 0 || B == 0) return cudaSuccess;
  if (dk == 128 && dv == 128)
    return dtype == BF16 ? launch_chunk<__nv_bfloat16, 128, 16>(q, k, v, g, beta, state, out, B, T, H, dv, scale, s)
                         : launch_chunk<float, 128, 16>(q, k, v, g, beta, state, out, B, T, H, dv, scale, s);
  if (dk == 64 && dv == 64)
    return dtype == BF16 ? launch_chunk<__nv_bfloat16, 64, 16>(q, k, v, g, beta, state, out, B, T, H, dv, scale, s)
                         : launch_chunk<float, 64, 16>(q, k, v, g, beta, state, out, B, T, H, dv, scale, s);
  return cudaErrorNotSupported;
}

// ------------------------------------------------------------------ single-token step
// One warp per state row (b, h, i): the row streams through registers once
// (read 4*dk bytes, write 4*dk bytes), two warp reductions.
template <typename T, int DK>
__global__ void __launch_bounds__(256) gdn_step_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                       const T* __restrict__ v, const float* __restrict__ g,
                                                       const float* __restrict__ beta, float* __restrict__ state,
                                                       T* __restrict__ out, int BH, int DV, float scale) {
  constexpr int PER = DK / 32;
  const int lane = threadIdx.x & 31;
  const long row = (long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= (long)BH * DV) return;
  const long bh = row / DV;
  const int i = (int)(row % DV);
  float* S = state + row * DK;
  float s[PER], kk[PER], qq[PER];
#pragma unroll
  for (int u = 0; u < PER; ++u) {
    s[u] = S[lane * PER + u];
    kk[u] = ldf(k + bh * DK + lane * PER + u);
    qq[u] = ldf(q + bh * DK + lane * PER + u);
  }
  const float alpha = expf(g[bh]), bt = beta[bh];
  float pred = 0.f;
#pragma unroll
  for (int u = 0; u < PER; ++u) pred = fmaf(s[u], kk[u], pred);
  pred = warp_sum(pred) * alpha;
  const float uu = bt * (ldf(v + bh * DV + i) - pred);
  float o = 0.f;
#pragma unroll
  for (int u = 0; u < PER; ++u) {
    s[u] = fmaf(alpha, s[u], uu * kk[u]);
    o = fmaf(s[u], qq[u], o);
    S[lane * PER + u] = s[u];
  }
  o = warp_sum(o);
  if (lane == 0) stf(out + bh * DV + i, scale * o);
}

cudaError_t gdn_step(const void* q, const void* k, const void* v, const float* g, const float* beta,
                     float* state, void* out, int B, int H, int dk, int dv, float scale, int dtype,
                     cudaStream_t s) {
  if (B == 0) return cudaSuccess;
  const long rows = (long)B * H * dv;
  dim3 grid((unsigned)((rows + 7) / 8));
  if (dk == 128) {
    if (dtype == BF16)
      gdn_step_kernel<__nv_bfloat16, 128><<<grid, 256, 0, s>>>((const __nv_bfloat16*)q, (const __nv_bfloat16*)k,
                                                               (const __nv_bfloat16*)v, g, beta, state,
                                                               (__nv_bfloat16*)out, B * H, dv, scale);
    else
      gdn_step_kernel<float, 128><<<grid, 256, 0, s>>>((const float*)q, (const float*)k, (const float*)v, g, beta,
                                                       state, (float*)out, B * H, dv, scale);
  } else if (dk == 64) {
    if (dtype == BF16)
      gdn_step_kernel<__nv_bfloat16, 64><<<grid, 256, 0, s>>>((const __nv_bfloat16*)q, (const __nv_bfloat16*)k,
                                                              (const __nv_bfloat16*)v, g, beta, state,
                                                              (__nv_bfloat16*)out, B * H, dv, scale);
    else
      gdn_step_kernel<float, 64><<<grid, 256, 0, s>>>((const float*)q, (const float*)k, (const float*)v, g, beta,
                                                      state, (float*)out, B * H, dv, scale);
  } else {
    return cudaErrorNotSupported;
  }
  return cudaGetLastError();
}

}  // namespace lk
