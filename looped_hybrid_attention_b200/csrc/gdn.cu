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
#include <type_traits>

#include "common.cuh"
#include "internal.h"
#include "mma_sync.cuh"
#include "tc_common.cuh"

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

// bf16, dk = dv = 128, 16-byte aligned rows: one warp per R heads of one token with
// 16-byte vectors -- lanes 0-15 normalise q, lanes 16-31 normalise k (8 elements each,
// sums reduced within each half-warp), lanes 0-15 copy v; all R heads' loads are in
// flight together.
template <int R>
__global__ void gdn_prep_v128_kernel(const __nv_bfloat16* __restrict__ P, int ld_p, const float* __restrict__ a_bias,
                                     const float* __restrict__ b_bias, __nv_bfloat16* __restrict__ q,
                                     __nv_bfloat16* __restrict__ k, __nv_bfloat16* __restrict__ v,
                                     float* __restrict__ g, float* __restrict__ beta, int M, int H, float eps) {
  constexpr int D = 128;
  const int lane = threadIdx.x & 31, half = lane >> 4, hl = lane & 15;
  const int groups = H / R;
  const long w = (long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (w >= (long)M * groups) return;
  const long m = w / groups;
  const int h0 = (int)(w % groups) * R;
  const __nv_bfloat16* row = P + m * ld_p;
  float x[R][8];
  uint4 vv[R];
#pragma unroll
  for (int r = 0; r < R; ++r) load8(row + half * H * D + (h0 + r) * D + hl * 8, x[r]);   // q (half 0) or k
  if (!half) {
#pragma unroll
    for (int r = 0; r < R; ++r) vv[r] = *reinterpret_cast<const uint4*>(row + 2 * H * D + (h0 + r) * D + hl * 8);
  }
  float ss[R];
#pragma unroll
  for (int r = 0; r < R; ++r) {
    ss[r] = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) ss[r] += x[r][i] * x[r][i];
  }
#pragma unroll
  for (int o = 8; o > 0; o >>= 1)
#pragma unroll
    for (int r = 0; r < R; ++r) ss[r] += __shfl_xor_sync(0xffffffffu, ss[r], o);
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const float inv = rsqrtf(ss[r] + eps);
#pragma unroll
    for (int i = 0; i < 8; ++i) x[r][i] *= inv;
    const long wr = m * H + h0 + r;
    store8((half ? k : q) + wr * D + hl * 8, x[r]);
    if (!half) *reinterpret_cast<uint4*>(v + wr * D + hl * 8) = vv[r];
  }
  if (lane >= 16 && lane < 16 + R) {
    const int h = h0 + lane - 16;
    const long wr = m * H + h;
    const float a = __bfloat162float(row[2 * H * D + H * D + h]) + a_bias[h];
    const float b = __bfloat162float(row[2 * H * D + H * D + H + h]) + b_bias[h];
    const float sp = a > 20.f ? a : log1pf(expf(a));    // softplus
    g[wr] = -sp;
    beta[wr] = 1.f / (1.f + expf(-b));
  }
}

cudaError_t gdn_prep(const void* P, int ld_p, const float* a_bias, const float* b_bias, void* q,
                     void* k, void* v, float* g, float* beta, int M, int H, int dk, int dv,
                     float eps, int dtype, cudaStream_t s) {
  if (M == 0) return cudaSuccess;
  const int warps = 8;
  dim3 grid((unsigned)(((long)M * H + warps - 1) / warps));
  auto al16 = [](const void* p) { return ((uintptr_t)p % 16) == 0; };
  if (dtype == BF16 && dk == 128 && dv == 128 && ld_p % 8 == 0 && al16(P) && al16(q) && al16(k) && al16(v)) {
    if (H % 4 == 0) {                             // four heads per warp
      const dim3 g4((unsigned)(((long)M * (H / 4) + warps - 1) / warps));
      gdn_prep_v128_kernel<4><<<g4, warps * 32, 0, s>>>((const __nv_bfloat16*)P, ld_p, a_bias, b_bias,
                                                        (__nv_bfloat16*)q, (__nv_bfloat16*)k, (__nv_bfloat16*)v, g,
                                                        beta, M, H, eps);
    } else {
      gdn_prep_v128_kernel<1><<<grid, warps * 32, 0, s>>>((const __nv_bfloat16*)P, ld_p, a_bias, b_bias,
                                                          (__nv_bfloat16*)q, (__nv_bfloat16*)k, (__nv_bfloat16*)v,
                                                          g, beta, M, H, eps);
    }
    return cudaGetLastError();
  }
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

// ------------------------------------------------------------------ two-pass chunked scan
// Pass 1 (gdn_intra_kernel, every chunk in parallel): cumulative log decay G, the
// strictly lower A and the causal P = (q.k) exp(G_r - G_s), and the solve
// (I + A) [W | U'] = [beta*gamma*K | beta*V] -- one thread per right-hand-side column,
// the column held in registers.  Written to the workspace: W [64, dk], U' [64, dv],
// P [64, 64], G [64] (fp32) per (b, h, chunk).
// Pass 2 (gdn_scan_kernel, chunks in order per (b, h, dv-slice)): U = U' - W S^T,
// O = scale (gamma Q S^T + P U), S <- exp(G_last) S + U^T (exp(G_last - G) K).  The next
// chunk's operands are prefetched with cp.async while the current one is processed.
template <int DK, int DV>
struct GdnWs {
  static constexpr int W_OFF = 0, U_OFF = GDN_C * DK, P_OFF = U_OFF + GDN_C * DV, G_OFF = P_OFF + GDN_C * GDN_C;
  static constexpr int FLOATS = G_OFF + GDN_C;
};

size_t gdn_workspace_bytes(int B, int T, int H, int dk, int dv) {
  const long chunks = (T + GDN_C - 1) / GDN_C;
  return (size_t)B * H * chunks * (GDN_C * (dk + dv) + GDN_C * GDN_C + GDN_C) * sizeof(float);
}

// Workspace block of the tensor-core scan (bf16 models), byte offsets within one
// (b, h, chunk) block: the left factor Aw = (I + A)^-1 diag(beta gamma) as two bf16
// terms, hi rows 0..63 then lo rows 64..127 of a [128][64] array (the scan forms
// W S^T = Aw (K S^T), so W itself is never rounded); U' fp32 [64][dv]; P bf16 [64][64];
// G fp32 [64].
template <int DK, int DV>
struct GdnWsB {
  static constexpr int AW_OFF = 0, U_OFF = 2 * GDN_C * GDN_C * 2, P_OFF = U_OFF + GDN_C * DV * 4,
                       G_OFF = P_OFF + GDN_C * GDN_C * 2, BYTES = G_OFF + GDN_C * 4;
};

template <typename T, int DK, int DV>
__global__ void __launch_bounds__(256, 2) gdn_intra_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                        const T* __restrict__ v, const float* __restrict__ g,
                                                        const float* __restrict__ beta, float* __restrict__ ws,
                                                        int T_len, int H, int n_chunks) {
  constexpr int C = GDN_C, CP = GDN_C + 4;
  using WL = GdnWs<DK, DV>;
  extern __shared__ float sm[];
  float* Kt = sm;                 // [DK][CP] keys, transposed
  float* Qt = Kt + DK * CP;       // [DK][CP] queries, transposed
  float* As = Qt + DK * CP;       // [C][CP] strictly lower A
  float* Gs = As + C * CP;        // [C]
  float* Bs = Gs + C;             // [C]
  const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  const int c0 = c * C, n = min(C, T_len - c0);
  float* blk = ws + (((long)b * H + h) * n_chunks + c) * WL::FLOATS;
  for (int idx = tid; idx < C * DK; idx += 256) {
    const int r = idx / DK, j = idx % DK;
    float kv = 0.f, qv = 0.f;
    if (r < n) {
      const long base = (((long)b * T_len + c0 + r) * H + h) * DK + j;
      kv = ldf(k + base);
      qv = ldf(q + base);
    }
    Kt[j * CP + r] = kv;
    Qt[j * CP + r] = qv;
  }
  if (tid < C) {
    const long gi = ((long)b * T_len + c0 + tid) * H + h;
    Gs[tid] = tid < n ? g[gi] : 0.f;
    Bs[tid] = tid < n ? beta[gi] : 0.f;
  }
  __syncthreads();
  if (tid < 32) {                 // inclusive prefix sum of the log decays
    float a0 = Gs[2 * tid], a1 = a0 + Gs[2 * tid + 1];
    float x = a1;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      float y = __shfl_up_sync(0xffffffffu, x, o);
      if (tid >= o) x += y;
    }
    Gs[2 * tid] = x - a1 + a0;
    Gs[2 * tid + 1] = x;
  }
  __syncthreads();
  if (tid < C) blk[WL::G_OFF + tid] = Gs[tid];
  {
    // 4 x 4 blocks of K K^T and Q K^T on and below the diagonal
    const int r0 = (tid >> 4) * 4, s0 = (tid & 15) * 4;
    float ak[4][4], aq[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int e = 0; e < 4; ++e) ak[a][e] = aq[a][e] = 0.f;
    if (s0 <= r0 + 3) {
#pragma unroll 4
      for (int j = 0; j < DK; ++j) {
        const float4 kr = *reinterpret_cast<const float4*>(Kt + j * CP + r0);
        const float4 qr = *reinterpret_cast<const float4*>(Qt + j * CP + r0);
        const float4 ks = *reinterpret_cast<const float4*>(Kt + j * CP + s0);
        const float krv[4] = {kr.x, kr.y, kr.z, kr.w}, qrv[4] = {qr.x, qr.y, qr.z, qr.w};
        const float ksv[4] = {ks.x, ks.y, ks.z, ks.w};
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            ak[a][e] = fmaf(krv[a], ksv[e], ak[a][e]);
            aq[a][e] = fmaf(qrv[a], ksv[e], aq[a][e]);
          }
      }
    }
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      const int r = r0 + a;
      float av[4], pv[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int s2 = s0 + e;
        const float dec = s2 <= r ? expf(Gs[r] - Gs[s2]) : 0.f;
        av[e] = s2 < r ? Bs[r] * dec * ak[a][e] : 0.f;
        pv[e] = aq[a][e] * dec;
      }
      *reinterpret_cast<float4*>(As + r * CP + s0) = make_float4(av[0], av[1], av[2], av[3]);
      *reinterpret_cast<float4*>(blk + WL::P_OFF + r * C + s0) = make_float4(pv[0], pv[1], pv[2], pv[3]);
    }
  }
  __syncthreads();
  if (tid < DK + DV) {
    const int j = tid;
    float x[C];
    if (j < DK) {
#pragma unroll
      for (int r = 0; r < C; ++r) x[r] = Bs[r] * expf(Gs[r]) * Kt[j * CP + r];
    } else {
#pragma unroll
      for (int r = 0; r < C; ++r)
        x[r] = r < n ? Bs[r] * ldf(v + (((long)b * T_len + c0 + r) * H + h) * DV + (j - DK)) : 0.f;
    }
    // forward substitution with the unit lower-triangular I + A (A[r][s] = 0 for s >= r)
#pragma unroll
    for (int r = 1; r < C; ++r) {
      float acc = x[r];
#pragma unroll
      for (int s4 = 0; s4 < (r + 3) / 4; ++s4) {
        const float4 a = *reinterpret_cast<const float4*>(As + r * CP + 4 * s4);
        acc = fmaf(-a.x, x[4 * s4], acc);
        acc = fmaf(-a.y, x[4 * s4 + 1], acc);
        acc = fmaf(-a.z, x[4 * s4 + 2], acc);
        acc = fmaf(-a.w, x[4 * s4 + 3], acc);
      }
      x[r] = acc;
    }
    {
      float* dst = j < DK ? blk + WL::W_OFF + j : blk + WL::U_OFF + (j - DK);
      const int stride = j < DK ? DK : DV;
#pragma unroll
      for (int r = 0; r < C; ++r) dst[r * stride] = x[r];
    }
  }
}

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem, bool valid) {
  const uint32_t d = (uint32_t)__cvta_generic_to_shared(smem);
  const int sz = valid ? 16 : 0;                       // 0: fill zeros, read nothing
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(gmem), "r"(sz) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

template <typename T, int DK, int DV, int DVS>
struct ScanSmem {
  static constexpr int WP = DK + 4;                    // fp32 row pitch of W
  static constexpr int PP = GDN_C + 4;                 // fp32 row pitch of P
  static constexpr int QP = DK + 16 / sizeof(T);       // row pitch of Q and K (elements of T)
  static constexpr int W_B = GDN_C * WP * 4, P_B = GDN_C * PP * 4, UP_B = GDN_C * DVS * 4,
                       Q_B = GDN_C * QP * sizeof(T), G_B = GDN_C * 4;
  static constexpr int BUF = W_B + P_B + UP_B + 2 * Q_B + G_B;
  static constexpr int ST_B = DK * DVS * 4;
  static constexpr int NBUF = (2 * BUF + 2 * ST_B + UP_B + 3 * GDN_C * 4 + 64) <= 225 * 1024 ? 2 : 1;
  static constexpr size_t BYTES = (size_t)NBUF * BUF + 2 * ST_B + UP_B + 3 * GDN_C * 4 + 64;
};

template <typename T, int DK, int DV, int DVS>
__global__ void __launch_bounds__(256) gdn_scan_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                       const float* __restrict__ ws, float* __restrict__ state,
                                                       T* __restrict__ out, int T_len, int H, int n_chunks, float scale) {
  constexpr int C = GDN_C;
  using L = ScanSmem<T, DK, DV, DVS>;
  using WL = GdnWs<DK, DV>;
  constexpr int NBUF = L::NBUF;
  extern __shared__ __align__(16) uint8_t smb[];
  float* St[2] = {(float*)(smb + NBUF * L::BUF), (float*)(smb + NBUF * L::BUF + L::ST_B)};   // [DK][DVS]
  float* Us = (float*)(smb + NBUF * L::BUF + 2 * L::ST_B);                                     // [C][DVS]
  float* gam = Us + C * DVS;                                                                     // exp(G_r)
  float* ex = gam + C;                                                                           // exp(G_last - G_s)
  const int tid = threadIdx.x;
  const int i0 = blockIdx.x * DVS, h = blockIdx.y, b = blockIdx.z;
  float* Sg = state + (((long)b * H + h) * DV + i0) * DK;
  for (int idx = tid; idx < DVS * DK; idx += 256) St[0][(idx % DK) * DVS + idx / DK] = Sg[idx];

  auto buf_ptr = [&](int bi) { return smb + bi * L::BUF; };
  auto issue = [&](int c, int bi) {
    uint8_t* base = buf_ptr(bi);
    float* Ws = (float*)base;
    float* Ps = (float*)(base + L::W_B);
    float* Ups = (float*)(base + L::W_B + L::P_B);
    T* Qs = (T*)(base + L::W_B + L::P_B + L::UP_B);
    T* Ks = (T*)(base + L::W_B + L::P_B + L::UP_B + L::Q_B);
    float* Gs = (float*)(base + L::W_B + L::P_B + L::UP_B + 2 * L::Q_B);
    const float* blk = ws + (((long)b * H + h) * n_chunks + c) * WL::FLOATS;
    const int c0 = c * C, n = min(C, T_len - c0);
    for (int idx = tid; idx < C * DK / 4; idx += 256) {
      const int r = idx / (DK / 4), p = idx % (DK / 4);
      cp_async16(Ws + r * L::WP + 4 * p, blk + WL::W_OFF + r * DK + 4 * p, true);
    }
    for (int idx = tid; idx < C * C / 4; idx += 256) {
      const int r = idx / (C / 4), p = idx % (C / 4);
      cp_async16(Ps + r * L::PP + 4 * p, blk + WL::P_OFF + r * C + 4 * p, true);
    }
    for (int idx = tid; idx < C * DVS / 4; idx += 256) {
      const int r = idx / (DVS / 4), p = idx % (DVS / 4);
      cp_async16(Ups + r * DVS + 4 * p, blk + WL::U_OFF + r * DV + i0 + 4 * p, true);
    }
    constexpr int PER_ROW = DK * (int)sizeof(T) / 16;
    for (int idx = tid; idx < C * PER_ROW; idx += 256) {
      const int r = idx / PER_ROW, p = idx % PER_ROW;
      const bool ok = r < n;
      const long row = (((long)b * T_len + c0 + (ok ? r : 0)) * H + h) * DK;
      cp_async16((uint8_t*)(Qs + r * L::QP) + 16 * p, (const uint8_t*)(q + row) + 16 * p, ok);
      cp_async16((uint8_t*)(Ks + r * L::QP) + 16 * p, (const uint8_t*)(k + row) + 16 * p, ok);
    }
    if (tid < C / 4) cp_async16(Gs + 4 * tid, blk + WL::G_OFF + 4 * tid, true);
    cp_async_commit();
  };

  issue(0, 0);
  int cur = 0;
  for (int c = 0; c < n_chunks; ++c) {
    const int bi = NBUF == 2 ? (c & 1) : 0;
    if (NBUF == 2 && c + 1 < n_chunks) {
      issue(c + 1, (c + 1) & 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    uint8_t* base = buf_ptr(bi);
    const float* Ws = (const float*)base;
    const float* Ps = (const float*)(base + L::W_B);
    const float* Ups = (const float*)(base + L::W_B + L::P_B);
    const T* Qs = (const T*)(base + L::W_B + L::P_B + L::UP_B);
    const T* Ks = (const T*)(base + L::W_B + L::P_B + L::UP_B + L::Q_B);
    const float* Gs = (const float*)(base + L::W_B + L::P_B + L::UP_B + 2 * L::Q_B);
    const float* S0 = St[cur];
    float* S1 = St[cur ^ 1];
    const int c0 = c * C, n = min(C, T_len - c0);
    if (tid < C) {
      gam[tid] = expf(Gs[tid]);
      ex[tid] = expf(Gs[C - 1] - Gs[tid]);
    }
    // U = U' - W S^T : thread (r, 4 consecutive i)
    const int r = tid >> 2, ib = (tid & 3) * 4;
    for (int it = 0; it < DVS / 16; ++it) {
      const int i = ib + it * 16;
      float4 acc = *reinterpret_cast<const float4*>(Ups + r * DVS + i);
#pragma unroll 8
      for (int kk = 0; kk < DK; ++kk) {
        const float w = Ws[r * L::WP + kk];
        const float4 sv = *reinterpret_cast<const float4*>(S0 + kk * DVS + i);
        acc.x = fmaf(-w, sv.x, acc.x);
        acc.y = fmaf(-w, sv.y, acc.y);
        acc.z = fmaf(-w, sv.z, acc.z);
        acc.w = fmaf(-w, sv.w, acc.w);
      }
      *reinterpret_cast<float4*>(Us + r * DVS + i) = acc;
    }
    __syncthreads();
    // O = scale (gamma Q S^T + P U)
    for (int it = 0; it < DVS / 16; ++it) {
      const int i = ib + it * 16;
      float4 a1 = make_float4(0, 0, 0, 0), a2 = make_float4(0, 0, 0, 0);
#pragma unroll 8
      for (int kk = 0; kk < DK; ++kk) {
        const float qv = ldf(Qs + r * L::QP + kk);
        const float4 sv = *reinterpret_cast<const float4*>(S0 + kk * DVS + i);
        a1.x = fmaf(qv, sv.x, a1.x);
        a1.y = fmaf(qv, sv.y, a1.y);
        a1.z = fmaf(qv, sv.z, a1.z);
        a1.w = fmaf(qv, sv.w, a1.w);
      }
      for (int s2 = 0; s2 <= r; ++s2) {
        const float pv = Ps[r * L::PP + s2];
        const float4 uv = *reinterpret_cast<const float4*>(Us + s2 * DVS + i);
        a2.x = fmaf(pv, uv.x, a2.x);
        a2.y = fmaf(pv, uv.y, a2.y);
        a2.z = fmaf(pv, uv.z, a2.z);
        a2.w = fmaf(pv, uv.w, a2.w);
      }
      if (r < n) {
        const float gr = gam[r];
        T* op = out + (((long)b * T_len + c0 + r) * H + h) * DV + i0 + i;
        stf(op + 0, scale * fmaf(gr, a1.x, a2.x));
        stf(op + 1, scale * fmaf(gr, a1.y, a2.y));
        stf(op + 2, scale * fmaf(gr, a1.z, a2.z));
        stf(op + 3, scale * fmaf(gr, a1.w, a2.w));
      }
    }
    // S1 = exp(G_last) S0 + U^T (exp(G_last - G) K) : thread (kk, 4 consecutive i)
    const float gl = expf(Gs[C - 1]);
    for (int idx = tid; idx < DK * (DVS / 4); idx += 256) {
      const int kk = idx % DK, i = (idx / DK) * 4;
      float4 acc = *reinterpret_cast<const float4*>(S0 + kk * DVS + i);
      acc.x *= gl;
      acc.y *= gl;
      acc.z *= gl;
      acc.w *= gl;
#pragma unroll 8
      for (int s2 = 0; s2 < C; ++s2) {
        const float kv = ex[s2] * ldf(Ks + s2 * L::QP + kk);
        const float4 uv = *reinterpret_cast<const float4*>(Us + s2 * DVS + i);
        acc.x = fmaf(uv.x, kv, acc.x);
        acc.y = fmaf(uv.y, kv, acc.y);
        acc.z = fmaf(uv.z, kv, acc.z);
        acc.w = fmaf(uv.w, kv, acc.w);
      }
      *reinterpret_cast<float4*>(S1 + kk * DVS + i) = acc;
    }
    __syncthreads();
    cur ^= 1;
    if (NBUF == 1 && c + 1 < n_chunks) issue(c + 1, 0);
  }
  for (int idx = tid; idx < DVS * DK; idx += 256) Sg[idx] = St[cur][(idx % DK) * DVS + idx / DK];
}


// ------------------------------------------------------------------ tensor-core sequential pass (bf16)
// The bf16 two-pass scan runs its chunk recurrence with the per-chunk products on the tensor
// cores (mma.sync m16n8k16, bf16 operands, fp32 accumulation):
//   Y  = K S^T               (64 x 16, K = dk)      A = K (exact),  B = S as bf16 hi + lo
//   U  = U' - Aw Y           (64 x 16, K = 64)      A = Aw hi + lo, B = Y hi + lo   (W S^T = Aw K S^T)
//   O  = gamma Q S^T + P U   (64 x 16, K = dk, 64)  A = Q, P; B = S hi, U (output: bf16 operands)
//   S <- exp(G_last) S + (exp(G_last - G) U)^T K   (16 x dk, K = 64)  A = as bf16 hi + lo, B = K
// Every product on the state's path has exact operands or operands carried as two bf16
// terms (hi + lo, relative error ~2^-17; the lo x lo term is dropped), so the state is
// updated with fp32-grade accuracy; only the output products use single bf16 operands.
__device__ __forceinline__ void st_bf2(__nv_bfloat16* p, float x, float y) {
  *reinterpret_cast<__nv_bfloat162*>(p) = __floats2bfloat162_rn(x, y);
}


// ------------------------------------------------------------------ warp-specialised sequential pass (bf16)
// The products above split by role, so that the state's chain of dependent
// products runs on warps of its own and no A fragment is loaded twice:
//   warps 0-3 (state):  Y = K S^T and U = U' - Aw Y with each warp owning one 16-row m-tile
//                       of the chunk and both 8-column n-tiles of the CTA's 16 state rows;
//                       S <- exp(G_C) S + (eU)^T K with each warp owning a quarter of the dk
//                       columns.  State-path operands as hi + lo bf16 pairs, as above.
//   warps 4-7 (output): O = scale (gamma Q S_c^T + P U) for the same m-tiles (bf16 hi
//                       operands), at most one chunk behind the state warps.
//   warp 8 (producer):  the chunk's tiles by TMA into a 3-stage ring.
// Hand-offs: mbarriers full[s] (the stage's tiles landed), empty[s] (the 8 compute warps
// are done with the stage), go[c % 2] (U of chunk c and the state it started from are in
// shared memory), done (the output warps finished a chunk: its U buffer and the state copy
// it read may be reused); named barrier 1 among the 128 state threads.  Shared-memory
// addresses of the fragments are fixed per lane and computed once.
template <int DK, int DV>
struct ScanWs {
  static constexpr int C = GDN_C, DVS = 16, KP = DK + 8, UP = DVS + 8;
  static constexpr int HALF = C * 128;
  static constexpr int AW_B = 2 * HALF, Q_B = (DK / 64) * HALF, K_B = Q_B, P_B = HALF, UPF_B = C * DVS * 4,
                       G_B = C * 4;
  static constexpr int TX = AW_B + Q_B + K_B + P_B + UPF_B + G_B;
  static constexpr int STAGE = (TX + 1023) / 1024 * 1024;
  static constexpr int NSTAGE = 3;
  static constexpr int S_B = DVS * KP * 2, U_B = C * UP * 2;
  // state copies [2 buffers][hi, lo]; U for the output [2 buffers]; (eU) hi, lo; Y hi, lo
  static constexpr int OFF_S = NSTAGE * STAGE, OFF_U = OFF_S + 4 * S_B, OFF_UE = OFF_U + 2 * U_B,
                       OFF_Y = OFF_UE + 2 * U_B, BAR_OFF = OFF_Y + 2 * U_B;
  static constexpr int N_BARS = 2 * NSTAGE + 3;                 // full[3], empty[3], go[2], done
  static constexpr size_t BYTES = (size_t)BAR_OFF + 8 * N_BARS + 16 + 1024;
  static_assert(BAR_OFF % 8 == 0, "mbarrier alignment");
  static_assert(BYTES <= 232448, "shared memory per CTA");
};

// Shared-memory accesses by address (explicit shared-window loads and stores).
__device__ __forceinline__ float lds_f(uint32_t a) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ void sts_bf2(uint32_t a, float x, float y) {
  asm volatile("st.shared.b32 [%0], %1;" ::"r"(a), "r"(pack_bf2(x, y)) : "memory");
}
__device__ __forceinline__ void sts_bf2_split(uint32_t hi, uint32_t lo, float x, float y) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(x, y);
  const float2 f = __bfloat1622float2(h);
  asm volatile("st.shared.b32 [%0], %1;" ::"r"(hi), "r"(*reinterpret_cast<const uint32_t*>(&h)) : "memory");
  sts_bf2(lo, x - f.x, y - f.y);
}

template <int DK, int DV>
__global__ void __launch_bounds__(288, 1) gdn_scan_ws_kernel(const __grid_constant__ CUtensorMap mA,
                                                             const __grid_constant__ CUtensorMap mP,
                                                             const __grid_constant__ CUtensorMap mU,
                                                             const __grid_constant__ CUtensorMap mG,
                                                             const __grid_constant__ CUtensorMap mQ,
                                                             const __grid_constant__ CUtensorMap mK,
                                                             float* __restrict__ state, __nv_bfloat16* __restrict__ out,
                                                             int T_len, int H, int n_chunks, float scale) {
  using L = ScanWs<DK, DV>;
  constexpr int C = L::C, DVS = L::DVS, KP = L::KP, UP = L::UP;
  extern __shared__ __align__(16) uint8_t smw_raw[];
  uint8_t* smb = (uint8_t*)(((uintptr_t)smw_raw + 1023) & ~(uintptr_t)1023);
  const uint32_t sbase = tc::smem_u32(smb);
  const uint32_t bar0 = sbase + L::BAR_OFF;
  auto full = [&](int i) { return bar0 + 8u * i; };
  auto empty = [&](int i) { return bar0 + 8u * (L::NSTAGE + i); };
  auto go = [&](int i) { return bar0 + 8u * (2 * L::NSTAGE + i); };
  const uint32_t done = bar0 + 8u * (2 * L::NSTAGE + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smb + L::BAR_OFF + 8 * L::N_BARS);
  const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31, gq = lane >> 2, tq = lane & 3;
  const int i0 = blockIdx.x * DVS, h = blockIdx.y, b = blockIdx.z;
  if (tid == 0) {
    for (int i = 0; i < L::NSTAGE; ++i) {
      tc::mbar_init(full(i), 1);
      tc::mbar_init(empty(i), 8);                              // one arrival per compute warp
    }
    tc::mbar_init(go(0), 4);
    tc::mbar_init(go(1), 4);
    tc::mbar_init(done, 4);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  float* Sg = state + (((long)b * H + h) * DV + i0) * DK;
  // byte offsets (from sbase) of the shared arrays
  auto s_copy = [&](int buf, int lo) { return (uint32_t)(L::OFF_S + (2 * buf + lo) * L::S_B); };
  const uint32_t u_out0 = L::OFF_U, ueh = L::OFF_UE, uel = L::OFF_UE + L::U_B, yh = L::OFF_Y, yl = L::OFF_Y + L::U_B;
  auto stage_off = [&](int c) { return (uint32_t)((c % L::NSTAGE) * L::STAGE); };
  // per-lane fragment offsets
  const int mt = w & 3;                                        // the m-tile of a state or output warp
  uint32_t a_off[4];                                           // A fragments of a swizzled 64-row piece
#pragma unroll
  for (int kk = 0; kk < 4; ++kk)
    a_off[kk] = (uint32_t)((mt * 16 + (lane & 15)) * 128 + ((((2 * kk + (lane >> 4)) ^ (lane & 7)) & 7) << 4));
  const uint32_t b_s = (uint32_t)(((lane & 7) + (lane >> 4) * 8) * KP * 2 + ((lane >> 3) & 1) * 16);  // state copy
  const uint32_t b_y = (uint32_t)((lane & 15) * UP * 2 + (lane >> 4) * 16);                            // [C][UP], trans
  const uint32_t a_ue = (uint32_t)((((lane >> 4) * 8) + (lane & 7)) * UP * 2 + ((lane >> 3) & 1) * 16);  // (eU)^T
  const int r0 = mt * 16 + gq, r1 = r0 + 8;

  __syncthreads();                                             // barriers initialised

  if (w == 8) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&mA) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&mQ) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&mK) : "memory");
      for (int c = 0; c < n_chunks; ++c) {
        const int st = c % L::NSTAGE;
        if (c >= L::NSTAGE && !tc::mbar_wait(empty(st), (uint32_t)((c / L::NSTAGE - 1) & 1), abort_flag)) break;
        tc::fence_proxy_async();                               // the consumers' reads before the new tiles
        const uint32_t base = sbase + stage_off(c);
        const int blk = (b * H + h) * n_chunks + c;
        const uint32_t fb = full(st);
        tc::mbar_expect_tx(fb, (uint32_t)L::TX);
        tc::tma_load_3d(base, &mA, fb, 0, 0, blk);
#pragma unroll
        for (int hf = 0; hf < DK / 64; ++hf) {
          tc::tma_load_4d(base + L::AW_B + hf * L::HALF, &mQ, fb, hf * 64, h, c * C, b);
          tc::tma_load_4d(base + L::AW_B + L::Q_B + hf * L::HALF, &mK, fb, hf * 64, h, c * C, b);
        }
        const uint32_t off_p = L::AW_B + L::Q_B + L::K_B;
        tc::tma_load_3d(base + off_p, &mP, fb, 0, 0, blk);
        tc::tma_load_3d(base + off_p + L::P_B, &mU, fb, i0, 0, blk);
        tc::tma_load_2d(base + off_p + L::P_B + L::UPF_B, &mG, fb, 0, blk);
      }
    }
  } else if (w < 4) {
    // ---------------------------------------------------------------- state warps
    constexpr int NT = DK / 32;                                // 8-column state tiles per warp
    const int cb = w * NT;                                     // first state tile of this warp
    // B fragments of K (trans) for the tile pairs (cb, cb+1), (cb+2, cb+3), ...
    uint32_t b_k[NT / 2];
#pragma unroll
    for (int p = 0; p < NT / 2; ++p) {
      const int col = (cb + 2 * p + (lane >> 4)) * 8;
      b_k[p] = (uint32_t)((col >> 6) * L::HALF + (lane & 15) * 128 + ((((col & 63) >> 3) ^ (lane & 7)) << 4));
    }
    float st[NT][4];
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      const int col = (cb + j) * 8 + 2 * tq;
      st[j][0] = Sg[gq * DK + col];
      st[j][1] = Sg[gq * DK + col + 1];
      st[j][2] = Sg[(gq + 8) * DK + col];
      st[j][3] = Sg[(gq + 8) * DK + col + 1];
      const uint32_t sh = sbase + s_copy(0, 0), sl = sbase + s_copy(0, 1);
      sts_bf2_split(sh + (gq * KP + col) * 2, sl + (gq * KP + col) * 2, st[j][0], st[j][1]);
      sts_bf2_split(sh + ((gq + 8) * KP + col) * 2, sl + ((gq + 8) * KP + col) * 2, st[j][2], st[j][3]);
    }
    asm volatile("bar.sync 1, 128;" ::: "memory");
    for (int c = 0; c < n_chunks; ++c) {
      const int sb = c & 1;
      if (!tc::mbar_wait(full(c % L::NSTAGE), (uint32_t)((c / L::NSTAGE) & 1), abort_flag)) break;
      const uint32_t base = sbase + stage_off(c);
      const uint32_t kb = base + L::AW_B + L::Q_B;
      const uint32_t upf = base + L::AW_B + L::Q_B + L::K_B + L::P_B;     // U' slice [C][DVS] fp32
      const uint32_t gsa = upf + L::UPF_B;                                 // G [C] fp32
      // 1a: Y = K S^T with S as hi + lo (m-tile mt, both n-tiles)
      float cy[2][2][4] = {}, cyl[2][2][4] = {};               // [n-tile][k parity]
      {
        const uint32_t sh = sbase + s_copy(sb, 0) + b_s, sl = sbase + s_copy(sb, 1) + b_s;
#pragma unroll
        for (int ks = 0; ks < DK / 16; ++ks) {
          uint32_t ak[4], bh[4], bl[4];
          ldsm_x4_s(ak, kb + (ks >> 2) * L::HALF + a_off[ks & 3]);
          ldsm_x4_s(bh, sh + ks * 32);
          ldsm_x4_s(bl, sl + ks * 32);
#pragma unroll
          for (int nt = 0; nt < 2; ++nt) {
            mma16816_h(cy[nt][ks & 1], ak, bh[2 * nt], bh[2 * nt + 1]);
            mma16816_h(cyl[nt][ks & 1], ak, bl[2 * nt], bl[2 * nt + 1]);
          }
        }
      }
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        float y[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) y[e] = (cy[nt][0][e] + cy[nt][1][e]) + (cyl[nt][0][e] + cyl[nt][1][e]);
        const int col = nt * 8 + 2 * tq;
        sts_bf2_split(sbase + yh + (r0 * UP + col) * 2, sbase + yl + (r0 * UP + col) * 2, y[0], y[1]);
        sts_bf2_split(sbase + yh + (r1 * UP + col) * 2, sbase + yl + (r1 * UP + col) * 2, y[2], y[3]);
      }
      asm volatile("bar.sync 1, 128;" ::: "memory");
      // the output warps are done with chunk c - 1: U buffer sb and state copy 1 - sb are free
      if (c >= 1 && !tc::mbar_wait(done, (uint32_t)((c - 1) & 1), abort_flag)) break;
      // 1b: W S^T = Aw Y with both as hi + lo (lo x lo dropped); U = U' - W S^T
      const float Glast = lds_f(gsa + (C - 1) * 4);
      const float e0 = expf(Glast - lds_f(gsa + r0 * 4)), e1 = expf(Glast - lds_f(gsa + r1 * 4)), gl = expf(Glast);
      {
        float cw[2][2][4] = {}, cx[2][2][4] = {};
#pragma unroll
        for (int ks = 0; ks < C / 16; ++ks) {
          uint32_t ah[4], al[4], bh[4], bl[4];
          ldsm_x4_s(ah, base + a_off[ks]);
          ldsm_x4_s(al, base + L::HALF + a_off[ks]);
          ldsm_x4_t_s(bh, sbase + yh + b_y + ks * 16 * UP * 2);
          ldsm_x4_t_s(bl, sbase + yl + b_y + ks * 16 * UP * 2);
#pragma unroll
          for (int nt = 0; nt < 2; ++nt) {
            mma16816_h(cw[nt][ks & 1], ah, bh[2 * nt], bh[2 * nt + 1]);
            mma16816_h(cx[nt][ks & 1], ah, bl[2 * nt], bl[2 * nt + 1]);
            mma16816_h(cx[nt][ks & 1], al, bh[2 * nt], bh[2 * nt + 1]);
          }
        }
        const uint32_t uo = sbase + u_out0 + sb * L::U_B;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          const int col = nt * 8 + 2 * tq;
          float wv[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) wv[e] = (cw[nt][0][e] + cw[nt][1][e]) + (cx[nt][0][e] + cx[nt][1][e]);
          const float u00 = lds_f(upf + (r0 * DVS + col) * 4) - wv[0], u01 = lds_f(upf + (r0 * DVS + col + 1) * 4) - wv[1];
          const float u10 = lds_f(upf + (r1 * DVS + col) * 4) - wv[2], u11 = lds_f(upf + (r1 * DVS + col + 1) * 4) - wv[3];
          sts_bf2(uo + (r0 * UP + col) * 2, u00, u01);
          sts_bf2(uo + (r1 * UP + col) * 2, u10, u11);
          sts_bf2_split(sbase + ueh + (r0 * UP + col) * 2, sbase + uel + (r0 * UP + col) * 2, u00 * e0, u01 * e0);
          sts_bf2_split(sbase + ueh + (r1 * UP + col) * 2, sbase + uel + (r1 * UP + col) * 2, u10 * e1, u11 * e1);
        }
      }
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(go(sb));                  // U of chunk c (and its start state) for the output warps
      asm volatile("bar.sync 1, 128;" ::: "memory");
      // 3: S <- exp(G_last) S + (eU)^T K on this warp's dk columns
      {
        float s1[NT][4], l0[NT][4], l1[NT][4];
#pragma unroll
        for (int j = 0; j < NT; ++j)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            st[j][e] *= gl;
            s1[j][e] = l0[j][e] = l1[j][e] = 0.f;
          }
#pragma unroll
        for (int ks = 0; ks < C / 16; ++ks) {
          uint32_t au[4], al[4];
          ldsm_x4_t_s(au, sbase + ueh + a_ue + ks * 16 * UP * 2);
          ldsm_x4_t_s(al, sbase + uel + a_ue + ks * 16 * UP * 2);
#pragma unroll
          for (int p = 0; p < NT / 2; ++p) {
            uint32_t bk[4];
            ldsm_x4_t_s(bk, kb + b_k[p] + ks * 16 * 128);
#pragma unroll
            for (int q = 0; q < 2; ++q) {
              const int j = 2 * p + q;
              mma16816_h((ks & 1) ? s1[j] : st[j], au, bk[2 * q], bk[2 * q + 1]);
              mma16816_h((ks & 1) ? l1[j] : l0[j], al, bk[2 * q], bk[2 * q + 1]);
            }
          }
        }
        const uint32_t sh = sbase + s_copy(sb ^ 1, 0), sl = sbase + s_copy(sb ^ 1, 1);
#pragma unroll
        for (int j = 0; j < NT; ++j) {
#pragma unroll
          for (int e = 0; e < 4; ++e) st[j][e] += s1[j][e] + (l0[j][e] + l1[j][e]);
          const int col = (cb + j) * 8 + 2 * tq;
          sts_bf2_split(sh + (gq * KP + col) * 2, sl + (gq * KP + col) * 2, st[j][0], st[j][1]);
          sts_bf2_split(sh + ((gq + 8) * KP + col) * 2, sl + ((gq + 8) * KP + col) * 2, st[j][2], st[j][3]);
        }
      }
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(empty(c % L::NSTAGE));
      asm volatile("bar.sync 1, 128;" ::: "memory");           // the new state copy, before the next Y
    }
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      const int col = (cb + j) * 8 + 2 * tq;
      Sg[gq * DK + col] = st[j][0];
      Sg[gq * DK + col + 1] = st[j][1];
      Sg[(gq + 8) * DK + col] = st[j][2];
      Sg[(gq + 8) * DK + col + 1] = st[j][3];
    }
  } else {
    // ---------------------------------------------------------------- output warps
    for (int c = 0; c < n_chunks; ++c) {
      const int sb = c & 1;
      if (!tc::mbar_wait(full(c % L::NSTAGE), (uint32_t)((c / L::NSTAGE) & 1), abort_flag)) break;
      if (!tc::mbar_wait(go(sb), (uint32_t)((c >> 1) & 1), abort_flag)) break;
      const uint32_t base = sbase + stage_off(c);
      const uint32_t qb = base + L::AW_B, pb = base + L::AW_B + L::Q_B + L::K_B;
      const uint32_t gsa = base + L::AW_B + L::Q_B + L::K_B + L::P_B + L::UPF_B;
      float cq[2][2][4] = {}, cp[2][2][4] = {};
      const uint32_t sh = sbase + s_copy(sb, 0) + b_s;
#pragma unroll
      for (int ks = 0; ks < DK / 16; ++ks) {
        uint32_t aq[4], bs[4];
        ldsm_x4_s(aq, qb + (ks >> 2) * L::HALF + a_off[ks & 3]);
        ldsm_x4_s(bs, sh + ks * 32);
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) mma16816_h(cq[nt][ks & 1], aq, bs[2 * nt], bs[2 * nt + 1]);
      }
      const uint32_t uo = sbase + u_out0 + sb * L::U_B + b_y;
#pragma unroll
      for (int ks = 0; ks < C / 16; ++ks) {
        uint32_t ap[4], bu[4];
        ldsm_x4_s(ap, pb + a_off[ks]);
        ldsm_x4_t_s(bu, uo + ks * 16 * UP * 2);
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) mma16816_h(cp[nt][ks & 1], ap, bu[2 * nt], bu[2 * nt + 1]);
      }
      const float g0 = expf(lds_f(gsa + r0 * 4)), g1 = expf(lds_f(gsa + r1 * 4));   // the last reads of the stage
      const int c0 = c * C, n = min(C, T_len - c0);
      __syncwarp();
      if (lane == 0) {
        tc::mbar_arrive(done);                                 // U buffer sb and state copy sb may be reused
        tc::mbar_arrive(empty(c % L::NSTAGE));
      }
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        const int col = nt * 8 + 2 * tq;
        if (r0 < n)
          st_bf2(out + (((long)b * T_len + c0 + r0) * H + h) * DV + i0 + col,
                 scale * fmaf(g0, cq[nt][0][0] + cq[nt][1][0], cp[nt][0][0] + cp[nt][1][0]),
                 scale * fmaf(g0, cq[nt][0][1] + cq[nt][1][1], cp[nt][0][1] + cp[nt][1][1]));
        if (r1 < n)
          st_bf2(out + (((long)b * T_len + c0 + r1) * H + h) * DV + i0 + col,
                 scale * fmaf(g1, cq[nt][0][2] + cq[nt][1][2], cp[nt][0][2] + cp[nt][1][2]),
                 scale * fmaf(g1, cq[nt][0][3] + cq[nt][1][3], cp[nt][0][3] + cp[nt][1][3]));
      }
    }
  }
}

// ------------------------------------------------------------------ tensor-core pass 1 (bf16)
// Pass 1 for bf16 models with the chunk-local products on the tensor cores (mma.sync
// m16n8k16, bf16 operands, fp32 accumulation).  Per (b, h, chunk), C = 64 tokens:
//   G = inclusive cumsum of the log decays g;  KK = K K^T, QK = Q K^T        (tensor cores)
//   A[r][s] = beta_r exp(G_r - G_s) KK[r][s]  (s < r),  P[r][s] = exp(G_r - G_s) QK[r][s]  (s <= r)
//   T = (I + A)^-1 in fp32: the four 16 x 16 diagonal blocks by substitution, then block
//       row i = 1..3:  T_ij = -T_ii sum_{k=j}^{i-1} A_ik T_kj
//   Aw = T diag(beta gamma) (gamma_s = exp(G_s)) as two bf16 terms, hi + lo, so its
//       rounding error is about 2^-17 instead of 2^-9; the sequential pass forms
//       W S^T = Aw (K S^T) from it
//   U' = (T diag(beta)) V   (tensor cores, the fp32 left factor split the same way)
// Aw, P (bf16), U', G (fp32) go to the workspace block the tensor-core sequential pass reads.
template <int DK, int DV>
struct IntraTc {
  static constexpr int C = GDN_C;
  static constexpr int KS = DK + 8, VS = DV + 8;           // bf16 row pitches (odd multiples of 16 B)
  static constexpr int FP = C + 4;                         // fp32 row pitch of A and T
  static constexpr int SP = C + 8;                         // bf16 row pitch of the split factors
  static constexpr int K_B = C * KS * 2, V_B = C * VS * 2;
  static constexpr int SPLIT_B = 2 * C * SP * 2;           // hi + lo
  static constexpr int QA_B = (K_B > SPLIT_B ? K_B : SPLIT_B);      // Q, later the W factors
  static constexpr int AU_B = (C * FP * 4 > SPLIT_B ? C * FP * 4 : SPLIT_B);   // A, later the U' factors
  static constexpr int T_B = C * FP * 4, M_B = 3 * 256 * 4, G_B = 3 * C * 4;
  static constexpr int KT_B = K_B > T_B ? K_B : T_B;       // K, then T (K's last use is K K^T, Q K^T)
  static constexpr int OFF_K = 0, OFF_T = 0, OFF_V = KT_B, OFF_QA = OFF_V + V_B, OFF_AU = OFF_QA + QA_B,
                       OFF_M = OFF_AU + AU_B, OFF_G = OFF_M + M_B;
  static constexpr size_t BYTES = (size_t)OFF_G + G_B;     // 75.5 KB at dk = dv = 128: three CTAs per SM
};

template <int DK, int DV>
__global__ void __launch_bounds__(256, 3)
    gdn_intra_tc_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                        const __nv_bfloat16* __restrict__ v, const float* __restrict__ g,
                        const float* __restrict__ beta, uint8_t* __restrict__ ws, int T_len, int H, int n_chunks) {
  using L = IntraTc<DK, DV>;
  using WLB = GdnWsB<DK, DV>;
  constexpr int C = L::C, KS = L::KS, VS = L::VS, FP = L::FP, SP = L::SP;
  extern __shared__ __align__(16) uint8_t smi[];
  __nv_bfloat16* Ks = (__nv_bfloat16*)(smi + L::OFF_K);
  __nv_bfloat16* Vs = (__nv_bfloat16*)(smi + L::OFF_V);
  __nv_bfloat16* Qs = (__nv_bfloat16*)(smi + L::OFF_QA);
  __nv_bfloat16* Awh = (__nv_bfloat16*)(smi + L::OFF_QA);    // after Q K^T
  __nv_bfloat16* Awl = Awh + C * SP;
  float* As = (float*)(smi + L::OFF_AU);
  __nv_bfloat16* Auh = (__nv_bfloat16*)(smi + L::OFF_AU);    // after T is complete
  __nv_bfloat16* Aul = Auh + C * SP;
  float* Ts = (float*)(smi + L::OFF_T);
  float* Ms = (float*)(smi + L::OFF_M);
  float* Gs = (float*)(smi + L::OFF_G);
  float* Bs = Gs + C;
  float* Es = Bs + C;                                       // gamma = exp(G)
  const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  const int w = tid >> 5, lane = tid & 31, gq = lane >> 2, tq = lane & 3;
  const int c0 = c * C, n = min(C, T_len - c0);
  uint8_t* blk = ws + (((long)b * H + h) * n_chunks + c) * (long)WLB::BYTES;
  __nv_bfloat16* Pg = reinterpret_cast<__nv_bfloat16*>(blk + WLB::P_OFF);
  __nv_bfloat16* Awg = reinterpret_cast<__nv_bfloat16*>(blk + WLB::AW_OFF);
  float* Ug = reinterpret_cast<float*>(blk + WLB::U_OFF);

  // ---- 1. the chunk's K, Q, V rows (zeros past the sequence end), decays and betas
  {
    constexpr int RK = DK * 2 / 16, RV = DV * 2 / 16;     // 16-byte pieces per row
    for (int idx = tid; idx < C * RK; idx += 256) {
      const int r = idx / RK, p = idx % RK;
      const bool ok = r < n;
      const long row = (((long)b * T_len + c0 + (ok ? r : 0)) * H + h) * DK;
      cp_async16(Ks + r * KS + 8 * p, k + row + 8 * p, ok);
      cp_async16(Qs + r * KS + 8 * p, q + row + 8 * p, ok);
    }
    for (int idx = tid; idx < C * RV; idx += 256) {
      const int r = idx / RV, p = idx % RV;
      const bool ok = r < n;
      const long row = (((long)b * T_len + c0 + (ok ? r : 0)) * H + h) * DV;
      cp_async16(Vs + r * VS + 8 * p, v + row + 8 * p, ok);
    }
    cp_async_commit();
    if (tid < C) {
      const long gi = ((long)b * T_len + c0 + tid) * H + h;
      Gs[tid] = tid < n ? g[gi] : 0.f;
      Bs[tid] = tid < n ? beta[gi] : 0.f;
    }
    __syncthreads();
    if (tid < 32) {                 // inclusive prefix sum of the log decays
      const float a0 = Gs[2 * tid], a1 = a0 + Gs[2 * tid + 1];
      float x = a1;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, x, o);
        if (tid >= o) x += y;
      }
      Gs[2 * tid] = x - a1 + a0;
      Gs[2 * tid + 1] = x;
      Es[2 * tid] = expf(x - a1 + a0);
      Es[2 * tid + 1] = expf(x);
    }
    cp_async_wait<0>();
    __syncthreads();
  }
  if (tid < C) reinterpret_cast<float*>(blk + WLB::G_OFF)[tid] = Gs[tid];

  // ---- 2. K K^T and Q K^T on and below the diagonal; A (smem, fp32) and P (workspace, bf16)
  {
    const int mt = w >> 1;                                  // rows 16 mt .. 16 mt + 15
    float akk[4][4], aqk[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int e = 0; e < 4; ++e) akk[i][e] = aqk[i][e] = 0.f;
#pragma unroll
    for (int ks = 0; ks < DK / 16; ++ks) {
      uint32_t ak[4], aq[4];
      ldsm_x4(ak, Ks + (mt * 16 + (lane & 15)) * KS + ks * 16 + (lane >> 4) * 8);
      ldsm_x4(aq, Qs + (mt * 16 + (lane & 15)) * KS + ks * 16 + (lane >> 4) * 8);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int nt = (w & 1) + 2 * i;                     // 8-column tiles
        if (nt > 2 * mt + 1) break;                         // above the diagonal
        uint32_t bk[2];
        ldsm_x2(bk, Ks + (nt * 8 + (lane & 7)) * KS + ks * 16 + ((lane >> 3) & 1) * 8);
        mma16816(akk[i], ak, bk);
        mma16816(aqk[i], aq, bk);
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int nt = (w & 1) + 2 * i;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int r = mt * 16 + gq + 8 * half, s0 = nt * 8 + 2 * tq;
        float pv[2] = {0.f, 0.f};
        if (nt <= 2 * mt + 1) {
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int s2 = s0 + e;
            const float dec = s2 <= r ? expf(Gs[r] - Gs[s2]) : 0.f;
            As[r * FP + s2] = s2 < r ? Bs[r] * dec * akk[i][2 * half + e] : 0.f;
            pv[e] = dec * aqk[i][2 * half + e];
          }
        }
        st_bf2(Pg + r * C + s0, pv[0], pv[1]);              // zeros above the diagonal
      }
    }
  }
  __syncthreads();

  // ---- 3. T = (I + A)^-1: diagonal 16 x 16 blocks by forward substitution (one column each)
  if (tid < C) {
    const int d = tid >> 4, cc = tid & 15, o = 16 * d;
    float x[16];
#pragma unroll
    for (int r = 0; r < 16; ++r) {
      float acc = r == cc ? 1.f : 0.f;
#pragma unroll
      for (int s2 = 0; s2 < r; ++s2) acc = fmaf(-As[(o + r) * FP + o + s2], x[s2], acc);
      x[r] = r < cc ? 0.f : acc;
    }
#pragma unroll
    for (int r = 0; r < 16; ++r) Ts[(o + r) * FP + o + cc] = x[r];
  }
  __syncthreads();
  // block rows 1..3: M_j = sum_{k=j}^{i-1} A_ik T_kj, then T_ij = -T_ii M_j
  for (int i = 1; i < 4; ++i) {
    for (int e = tid; e < 256 * i; e += 256) {
      const int j = e >> 8, rr = (e >> 4) & 15, cc = e & 15;
      float acc = 0.f;
      for (int kb = j; kb < i; ++kb)
#pragma unroll
        for (int m = 0; m < 16; ++m) acc = fmaf(As[(16 * i + rr) * FP + 16 * kb + m], Ts[(16 * kb + m) * FP + 16 * j + cc], acc);
      Ms[e] = acc;
    }
    __syncthreads();
    for (int e = tid; e < 256 * i; e += 256) {
      const int j = e >> 8, rr = (e >> 4) & 15, cc = e & 15;
      float acc = 0.f;
#pragma unroll
      for (int m = 0; m < 16; ++m)
        if (m <= rr) acc = fmaf(Ts[(16 * i + rr) * FP + 16 * i + m], Ms[(j << 8) + (m << 4) + cc], acc);
      Ts[(16 * i + rr) * FP + 16 * j + cc] = -acc;
    }
    __syncthreads();
  }

  // ---- 4. left factors T diag(beta gamma) and T diag(beta), each as bf16 hi + lo
  for (int e = tid; e < C * C / 2; e += 256) {
    const int r = e / (C / 2), s2 = 2 * (e % (C / 2));
    float tw[2], tu[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const float t = (s2 + u) <= r ? Ts[r * FP + s2 + u] : 0.f;
      tu[u] = t * Bs[s2 + u];
      tw[u] = tu[u] * Es[s2 + u];
    }
    const __nv_bfloat162 wh = __floats2bfloat162_rn(tw[0], tw[1]), uh = __floats2bfloat162_rn(tu[0], tu[1]);
    const float2 whf = __bfloat1622float2(wh), uhf = __bfloat1622float2(uh);
    *reinterpret_cast<__nv_bfloat162*>(Awh + r * SP + s2) = wh;
    *reinterpret_cast<__nv_bfloat162*>(Awl + r * SP + s2) = __floats2bfloat162_rn(tw[0] - whf.x, tw[1] - whf.y);
    *reinterpret_cast<__nv_bfloat162*>(Auh + r * SP + s2) = uh;
    *reinterpret_cast<__nv_bfloat162*>(Aul + r * SP + s2) = __floats2bfloat162_rn(tu[0] - uhf.x, tu[1] - uhf.y);
  }
  __syncthreads();

  // ---- 5. Aw (hi rows, then lo rows) to the workspace; U' = Au V (fp32 out): warp = (16-row
  //         tile, half of the columns)
  for (int e = tid; e < 2 * C * C / 8; e += 256) {           // 16-byte pieces of [2C][C]
    const int r = e / (C / 8), p8 = e % (C / 8);
    const __nv_bfloat16* src = (r < C ? Awh + r * SP : Awl + (r - C) * SP) + 8 * p8;
    *reinterpret_cast<uint4*>(Awg + r * C + 8 * p8) = *reinterpret_cast<const uint4*>(src);
  }
  {
    const int mt = w & 3, nh = w >> 2;
    auto product = [&](const __nv_bfloat16* Ah, const __nv_bfloat16* Al, const __nv_bfloat16* Bm, int BP, int NC,
                       auto&& store) {
      constexpr int NTW = (DK > DV ? DK : DV) / 16;          // 8-column tiles per warp (upper bound)
      const int ntw = NC / 16;
      float acc[NTW][4];
#pragma unroll
      for (int t2 = 0; t2 < NTW; ++t2)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[t2][e] = 0.f;
#pragma unroll
      for (int ks = 0; ks < C / 16; ++ks) {
        uint32_t ah[4], al[4];
        ldsm_x4(ah, Ah + (mt * 16 + (lane & 15)) * SP + ks * 16 + (lane >> 4) * 8);
        ldsm_x4(al, Al + (mt * 16 + (lane & 15)) * SP + ks * 16 + (lane >> 4) * 8);
#pragma unroll
        for (int t2 = 0; t2 < NTW; ++t2) {
          if (t2 >= ntw) break;
          uint32_t bb[2];
          ldsm_x2_t(bb, Bm + (ks * 16 + (lane & 15)) * BP + (nh * ntw + t2) * 8);
          mma16816(acc[t2], ah, bb);
          mma16816(acc[t2], al, bb);
        }
      }
#pragma unroll
      for (int t2 = 0; t2 < NTW; ++t2) {
        if (t2 >= ntw) break;
        const int col = (nh * ntw + t2) * 8 + 2 * tq, r0 = mt * 16 + gq;
        store(r0, col, acc[t2][0], acc[t2][1]);
        store(r0 + 8, col, acc[t2][2], acc[t2][3]);
      }
    };
    product(Auh, Aul, Vs, VS, DV, [&](int r, int col, float x0, float x1) {
      *reinterpret_cast<float2*>(Ug + r * DV + col) = make_float2(x0, x1);
    });
  }
}

template <typename T, int DK, int DV>
static cudaError_t launch_two_pass(const void* q, const void* k, const void* v, const float* g, const float* beta,
                                   float* state, void* out, int B, int T_len, int H, float scale, void* workspace,
                                   cudaStream_t s) {
  constexpr int DVS = 16;
  const int n_chunks = (T_len + GDN_C - 1) / GDN_C;
  const size_t smem1 = (size_t)(2 * DK * (GDN_C + 4) + GDN_C * (GDN_C + 4) + 2 * GDN_C) * sizeof(float);
  constexpr bool TC = std::is_same<T, __nv_bfloat16>::value;   // bf16: tensor-core sequential pass
  auto k1 = gdn_intra_kernel<T, DK, DV>;
  auto k2 = gdn_scan_kernel<T, DK, DV, DVS>;
  using L = ScanSmem<T, DK, DV, DVS>;
  using LW = ScanWs<DK, DV>;
  {
    cudaError_t e = set_smem_limit(k1, (int)smem1);
    if (e == cudaSuccess) e = set_smem_limit(k2, (int)L::BYTES);
    if (e != cudaSuccess) return e;
  }
  if (TC) {
    using LI = IntraTc<DK, DV>;
    auto k1t = gdn_intra_tc_kernel<DK, DV>;
    {
      cudaError_t e = set_smem_limit(k1t, (int)LI::BYTES);
      if (e != cudaSuccess) return e;
    }
    k1t<<<dim3(n_chunks, H, B), 256, LI::BYTES, s>>>((const __nv_bfloat16*)q, (const __nv_bfloat16*)k,
                                                      (const __nv_bfloat16*)v, g, beta, (uint8_t*)workspace, T_len, H,
                                                      n_chunks);
  } else {
    k1<<<dim3(n_chunks, H, B), 256, smem1, s>>>((const T*)q, (const T*)k, (const T*)v, g, beta, (float*)workspace,
                                                 T_len, H, n_chunks);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (TC) {
    // tensor maps of the workspace blocks and of q, k [B, T, H, dk] for the scan's tile loads
    using WLB = GdnWsB<DK, DV>;
    const uint8_t* wsb = (const uint8_t*)workspace;
    const cuuint64_t nblk = (cuuint64_t)B * H * n_chunks, bs = (cuuint64_t)WLB::BYTES;
    CUtensorMap mA, mP, mU, mG, mQ, mK;
    const cuuint64_t dA[3] = {GDN_C, 2 * GDN_C, nblk}, sA[2] = {GDN_C * 2, bs};
    const cuuint64_t dP[3] = {GDN_C, GDN_C, nblk}, sP[2] = {GDN_C * 2, bs};
    const cuuint64_t dU[3] = {DV, GDN_C, nblk}, sU[2] = {DV * 4, bs};
    const cuuint64_t dG[2] = {GDN_C, nblk}, sG[1] = {bs};
    const cuuint64_t dQ[4] = {DK, (cuuint64_t)H, (cuuint64_t)T_len, (cuuint64_t)B};
    const cuuint64_t sQ[3] = {DK * 2, (cuuint64_t)H * DK * 2, (cuuint64_t)T_len * H * DK * 2};
    const cuuint32_t b64[3] = {64, GDN_C, 1}, bA[3] = {64, 2 * GDN_C, 1}, bU[3] = {LW::DVS, GDN_C, 1},
                     bG[2] = {GDN_C, 1}, bQ[4] = {64, 1, GDN_C, 1};
    const auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, F32 = CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
    if (!tc::make_map_nd(&mA, BF, 3, wsb + WLB::AW_OFF, dA, sA, bA, true) ||
        !tc::make_map_nd(&mP, BF, 3, wsb + WLB::P_OFF, dP, sP, b64, true) ||
        !tc::make_map_nd(&mU, F32, 3, wsb + WLB::U_OFF, dU, sU, bU, false) ||
        !tc::make_map_nd(&mG, F32, 2, wsb + WLB::G_OFF, dG, sG, bG, false) ||
        !tc::make_map_nd(&mQ, BF, 4, q, dQ, sQ, bQ, true) || !tc::make_map_nd(&mK, BF, 4, k, dQ, sQ, bQ, true))
      return cudaErrorNotSupported;
    auto k2w = gdn_scan_ws_kernel<DK, DV>;
    {
      cudaError_t e2 = set_smem_limit(k2w, (int)LW::BYTES);
      if (e2 != cudaSuccess) return e2;
    }
    k2w<<<dim3(DV / LW::DVS, H, B), 288, LW::BYTES, s>>>(mA, mP, mU, mG, mQ, mK, state, (__nv_bfloat16*)out, T_len, H,
                                                          n_chunks, scale);
  } else
    k2<<<dim3(DV / DVS, H, B), 256, L::BYTES, s>>>((const T*)q, (const T*)k, (const float*)workspace, state, (T*)out,
                                                    T_len, H, n_chunks, scale);
  return cudaGetLastError();
}

bool gdn_supported(int dk, int dv) { return (dk == 64 && dv == 64) || (dk == 128 && dv == 128); }

template <typename T, int DK, int DVS>
static cudaError_t launch_chunk(const void* q, const void* k, const void* v, const float* g,
                                const float* beta, float* state, void* out, int B, int T_len, int H,
                                int dv, float scale, cudaStream_t s) {
  using L = GdnSmem<DK, DVS>;
  auto kern = gdn_chunk_kernel<T, DK, DVS>;
  cudaError_t e = set_smem_limit(kern, (int)L::bytes);
  if (e != cudaSuccess) return e;
  dim3 grid(dv / DVS, H, B);
  kern<<<grid, 256, L::bytes, s>>>((const T*)q, (const T*)k, (const T*)v, g, beta, state, (T*)out, T_len, H,
                                   dv, scale);
  return cudaGetLastError();
}

cudaError_t gdn_chunk(const void* q, const void* k, const void* v, const float* g,
                      const float* beta, float* state, void* out, int B, int T, int H, int dk,
                      int dv, float scale, int dtype, cudaStream_t s, void* workspace) {
  if (T == 0 || B == 0) return cudaSuccess;
  // the two-pass kernels copy 16-byte pieces of q, k, v rows and of the workspace
  auto al16 = [](const void* p) { return ((uintptr_t)p % 16) == 0; };
  if (workspace && !(al16(q) && al16(k) && al16(v) && al16(workspace))) return cudaErrorNotSupported;
  if (workspace) {
    if (dk == 128 && dv == 128)
      return dtype == BF16
                 ? launch_two_pass<__nv_bfloat16, 128, 128>(q, k, v, g, beta, state, out, B, T, H, scale, workspace, s)
                 : launch_two_pass<float, 128, 128>(q, k, v, g, beta, state, out, B, T, H, scale, workspace, s);
    if (dk == 64 && dv == 64)
      return dtype == BF16
                 ? launch_two_pass<__nv_bfloat16, 64, 64>(q, k, v, g, beta, state, out, B, T, H, scale, workspace, s)
                 : launch_two_pass<float, 64, 64>(q, k, v, g, beta, state, out, B, T, H, scale, workspace, s);
    return cudaErrorNotSupported;
  }
  if (dk == 128 && dv == 128)
    return dtype == BF16 ? launch_chunk<__nv_bfloat16, 128, 16>(q, k, v, g, beta, state, out, B, T, H, dv, scale, s)
                         : launch_chunk<float, 128, 16>(q, k, v, g, beta, state, out, B, T, H, dv, scale, s);
  if (dk == 64 && dv == 64)
    return dtype == BF16 ? launch_chunk<__nv_bfloat16, 64, 16>(q, k, v, g, beta, state, out, B, T, H, dv, scale, s)
                         : launch_chunk<float, 64, 16>(q, k, v, g, beta, state, out, B, T, H, dv, scale, s);
  return cudaErrorNotSupported;
}

// ------------------------------------------------------------------ single-token step
// One warp per R state rows (b, h, i0 .. i0 + R - 1) of one head: every row streams
// through registers once (read 4*dk bytes, write 4*dk bytes, 16-byte accesses), all R
// rows' loads are in flight together, and the head's k and q are read once for them.
// VEC: 16-byte (dk 128) or 8-byte (dk 64) state accesses, for an aligned state.
template <int PER>
struct Vec;
template <>
struct Vec<4> {
  static __device__ __forceinline__ void ld(const float* p, float* x) {
    const float4 a = *reinterpret_cast<const float4*>(p);
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
  }
  static __device__ __forceinline__ void st(float* p, const float* x) {
    *reinterpret_cast<float4*>(p) = make_float4(x[0], x[1], x[2], x[3]);
  }
};
template <>
struct Vec<2> {
  static __device__ __forceinline__ void ld(const float* p, float* x) {
    const float2 a = *reinterpret_cast<const float2*>(p);
    x[0] = a.x; x[1] = a.y;
  }
  static __device__ __forceinline__ void st(float* p, const float* x) {
    *reinterpret_cast<float2*>(p) = make_float2(x[0], x[1]);
  }
};

template <typename T, int DK, int R, bool VEC>
__global__ void __launch_bounds__(256) gdn_step_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                       const T* __restrict__ v, const float* __restrict__ g,
                                                       const float* __restrict__ beta, float* __restrict__ state,
                                                       T* __restrict__ out, int BH, int DV, float scale) {
  pdl_trigger();
  constexpr int PER = DK / 32;
  const int lane = threadIdx.x & 31;
  const long row0 = ((long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5)) * R;
  if (row0 >= (long)BH * DV) return;
  const long bh = row0 / DV;                     // DV % R == 0: the R rows share the head
  const int i0 = (int)(row0 % DV);
  float* S = state + row0 * DK + lane * PER;
  float s[R][PER], kk[PER], qq[PER];
#pragma unroll
  for (int r = 0; r < R; ++r) {
    if (VEC) {
      Vec<PER>::ld(S + r * DK, s[r]);
    } else {
#pragma unroll
      for (int u = 0; u < PER; ++u) s[r][u] = S[r * DK + u];
    }
  }
#pragma unroll
  for (int u = 0; u < PER; ++u) {
    kk[u] = ldf(k + bh * DK + lane * PER + u);
    qq[u] = ldf(q + bh * DK + lane * PER + u);
  }
  const float alpha = expf(g[bh]), bt = beta[bh];
#pragma unroll
  for (int r = 0; r < R; ++r) {
    float pred = 0.f;
#pragma unroll
    for (int u = 0; u < PER; ++u) pred = fmaf(s[r][u], kk[u], pred);
    pred = warp_sum(pred) * alpha;
    const float uu = bt * (ldf(v + bh * DV + i0 + r) - pred);
    float o = 0.f;
#pragma unroll
    for (int u = 0; u < PER; ++u) {
      s[r][u] = fmaf(alpha, s[r][u], uu * kk[u]);
      o = fmaf(s[r][u], qq[u], o);
    }
    if (VEC) {
      Vec<PER>::st(S + r * DK, s[r]);
    } else {
#pragma unroll
      for (int u = 0; u < PER; ++u) S[r * DK + u] = s[r][u];
    }
    o = warp_sum(o);
    if (lane == 0) stf(out + bh * DV + i0 + r, scale * o);
  }
}

// The decode step straight from the stored input projection (rows q | k | v | a | b per
// token, H heads): each warp L2-normalises its head's q and k (eps inside the root) and
// rounds them to the storage type, forms g = -softplus(a + a_bias) and beta = sigmoid(b +
// b_bias) -- what the GDN preparation would have stored -- then updates its R state rows as
// gdn_step_kernel does.  The preparation's launch and its q, k, v, g, beta round trip are
// gone from the decode step.
template <typename T, int DK, int R, bool VEC>
__global__ void __launch_bounds__(256) gdn_step_proj_kernel(const T* __restrict__ P, int ld_p,
                                                            const float* __restrict__ a_bias,
                                                            const float* __restrict__ b_bias, float eps, int H,
                                                            float* __restrict__ state, T* __restrict__ out, int BH,
                                                            int DV, float scale) {
  pdl_trigger();
  constexpr int PER = DK / 32;
  const int lane = threadIdx.x & 31;
  const long row0 = ((long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5)) * R;
  if (row0 >= (long)BH * DV) return;
  const long bh = row0 / DV;                     // DV % R == 0: the R rows share the head
  const int i0 = (int)(row0 % DV);
  const long b = bh / H;
  const int h = (int)(bh % H);
  const T* prow = P + b * ld_p;
  float* S = state + row0 * DK + lane * PER;
  float s[R][PER], kk[PER], qq[PER];
#pragma unroll
  for (int r = 0; r < R; ++r) {
    if (VEC) {
      Vec<PER>::ld(S + r * DK, s[r]);
    } else {
#pragma unroll
      for (int u = 0; u < PER; ++u) s[r][u] = S[r * DK + u];
    }
  }
  float sq = 0.f, sk = 0.f;
#pragma unroll
  for (int u = 0; u < PER; ++u) {
    qq[u] = ldf(prow + (long)h * DK + lane * PER + u);
    kk[u] = ldf(prow + (long)(H + h) * DK + lane * PER + u);
    sq = fmaf(qq[u], qq[u], sq);
    sk = fmaf(kk[u], kk[u], sk);
  }
  const T* gates = prow + 2L * H * DK + (long)H * DV;
  const float a = ldf(gates + h) + a_bias[h];
  const float bb = ldf(gates + H + h) + b_bias[h];
  const float iq = rsqrtf(warp_sum(sq) + eps), ik = rsqrtf(warp_sum(sk) + eps);
#pragma unroll
  for (int u = 0; u < PER; ++u) {
    qq[u] = Io<T>::round(qq[u] * iq);
    kk[u] = Io<T>::round(kk[u] * ik);
  }
  const float sp = a > 20.f ? a : log1pf(expf(a));    // softplus
  const float alpha = expf(-sp), bt = 1.f / (1.f + expf(-bb));
  const T* vrow = prow + 2L * H * DK + (long)h * DV;
#pragma unroll
  for (int r = 0; r < R; ++r) {
    float pred = 0.f;
#pragma unroll
    for (int u = 0; u < PER; ++u) pred = fmaf(s[r][u], kk[u], pred);
    pred = warp_sum(pred) * alpha;
    const float uu = bt * (ldf(vrow + i0 + r) - pred);
    float o = 0.f;
#pragma unroll
    for (int u = 0; u < PER; ++u) {
      s[r][u] = fmaf(alpha, s[r][u], uu * kk[u]);
      o = fmaf(s[r][u], qq[u], o);
    }
    if (VEC) {
      Vec<PER>::st(S + r * DK, s[r]);
    } else {
#pragma unroll
      for (int u = 0; u < PER; ++u) S[r * DK + u] = s[r][u];
    }
    o = warp_sum(o);
    if (lane == 0) stf(out + bh * DV + i0 + r, scale * o);
  }
}

cudaError_t gdn_step_proj(const void* P, int ld_p, const float* a_bias, const float* b_bias, float eps, float* state,
                          void* out, int B, int H, int dk, int dv, float scale, int dtype, cudaStream_t s) {
  if (B == 0) return cudaSuccess;
  const long rows = (long)B * H * dv;
  const bool r4 = dv % 4 == 0 && (uintptr_t)state % (dk == 128 ? 16 : 8) == 0;
  const dim3 grid((unsigned)((rows + (r4 ? 31 : 7)) / (r4 ? 32 : 8)));
#define GDN_STEP_P(TT, DKK, RR)                                                                             \
  gdn_step_proj_kernel<TT, DKK, RR, (RR > 1)><<<grid, 256, 0, s>>>((const TT*)P, ld_p, a_bias, b_bias, eps, H, \
                                                                   state, (TT*)out, B * H, dv, scale)
  if (dk == 128) {
    if (dtype == BF16) {
      if (r4) GDN_STEP_P(__nv_bfloat16, 128, 4); else GDN_STEP_P(__nv_bfloat16, 128, 1);
    } else {
      if (r4) GDN_STEP_P(float, 128, 4); else GDN_STEP_P(float, 128, 1);
    }
  } else if (dk == 64) {
    if (dtype == BF16) {
      if (r4) GDN_STEP_P(__nv_bfloat16, 64, 4); else GDN_STEP_P(__nv_bfloat16, 64, 1);
    } else {
      if (r4) GDN_STEP_P(float, 64, 4); else GDN_STEP_P(float, 64, 1);
    }
  } else {
    return cudaErrorNotSupported;
  }
#undef GDN_STEP_P
  return cudaGetLastError();
}

cudaError_t gdn_step(const void* q, const void* k, const void* v, const float* g, const float* beta,
                     float* state, void* out, int B, int H, int dk, int dv, float scale, int dtype,
                     cudaStream_t s) {
  if (B == 0) return cudaSuccess;
  const long rows = (long)B * H * dv;
  // four rows of one head per warp, 16/8-byte state accesses; else the plain form
  const bool r4 = dv % 4 == 0 && (uintptr_t)state % (dk == 128 ? 16 : 8) == 0;
  const dim3 grid((unsigned)((rows + (r4 ? 31 : 7)) / (r4 ? 32 : 8)));
#define GDN_STEP(TT, DKK, RR)                                                                                      \
  gdn_step_kernel<TT, DKK, RR, (RR > 1)><<<grid, 256, 0, s>>>((const TT*)q, (const TT*)k, (const TT*)v, g, beta, state,      \
                                                    (TT*)out, B * H, dv, scale)
  if (dk == 128) {
    if (dtype == BF16) {
      if (r4) GDN_STEP(__nv_bfloat16, 128, 4); else GDN_STEP(__nv_bfloat16, 128, 1);
    } else {
      if (r4) GDN_STEP(float, 128, 4); else GDN_STEP(float, 128, 1);
    }
  } else if (dk == 64) {
    if (dtype == BF16) {
      if (r4) GDN_STEP(__nv_bfloat16, 64, 4); else GDN_STEP(__nv_bfloat16, 64, 1);
    } else {
      if (r4) GDN_STEP(float, 64, 4); else GDN_STEP(float, 64, 1);
    }
  } else {
    return cudaErrorNotSupported;
  }
#undef GDN_STEP
  return cudaGetLastError();
}

}  // namespace lk
