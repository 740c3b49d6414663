// Two-stream mHC residual ("Loop-9B engineering teardown" §五, §六; "SenseNova-Loop-9B
// 是什么" §二): one kernel per layer boundary mixes the previous layer's output into
// the two streams, then computes the next layer's routing (FP32 logits, FP32
// Sinkhorn) and reads the layer input -- the streams cross HBM once per boundary.
//
// bf16 streams, many tokens (mhc_cluster_kernel): a cluster of CL CTAs shares a block
// of TB tokens and CTA r owns the slice [r S, (r+1) S) of both streams.  Each CTA mixes
// its slice (16-byte loads, results kept in shared memory), forms its slice's share of
// the 8 routing dot products on the tensor cores (mma.sync; the FP32 map enters as the
// exact sum of three bf16 terms, the streams are bf16 already, so every product is
// exact and the sums are FP32), and the CTAs exchange their partial sums through
// distributed shared memory.  Every CTA adds the partials in rank order, so all of them
// hold bit-identical coefficients, and each writes its slice of the layer input from
// shared memory -- nothing is re-read from HBM.
//
// fp32 streams or few tokens: the warp-per-4-tokens kernel (mhc_kernel) or the
// CTA-per-token kernel (mhc_token_kernel), FP32 FMAs throughout.
//
// MERGE (the last boundary) is a plain streaming kernel: h = (X0' + X1') / 2.
#include "common.cuh"
#include "internal.h"
#include "mma_sync.cuh"
#include "tc_common.cuh"

namespace lk {

// 2x2 Sinkhorn in registers: rows then columns, `iters` times, on m = exp(l - max l)
// whose smallest entry is exp(-spread).  Every entry stays <= 1, so every row or column
// sum is <= 2 and no normalisation shrinks an entry by more than 2: after k steps the
// entries are >= exp(-spread) 2^-k.  When that bound stays above exp(-80) (a normal
// float, whose reciprocal cannot overflow) for all 2 iters steps, each sum's reciprocal
// comes from the hardware (rcp.approx, within about one ulp) and scales two entries;
// otherwise the loop divides (IEEE) instead.
__device__ __forceinline__ float rcp_hw(float x) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}
__device__ __forceinline__ void sinkhorn2(float m[4], int iters, float spread) {
  if (spread + 1.38629436f * (float)iters <= 80.f) {
    for (int it = 0; it < iters; ++it) {
      const float r0 = rcp_hw(m[0] + m[1]), r1 = rcp_hw(m[2] + m[3]);
      m[0] *= r0; m[1] *= r0; m[2] *= r1; m[3] *= r1;
      const float c0 = rcp_hw(m[0] + m[2]), c1 = rcp_hw(m[1] + m[3]);
      m[0] *= c0; m[2] *= c0; m[1] *= c1; m[3] *= c1;
    }
  } else {
    for (int it = 0; it < iters; ++it) {
      const float r0 = m[0] + m[1], r1 = m[2] + m[3];
      m[0] /= r0; m[1] /= r0; m[2] /= r1; m[3] /= r1;
      const float c0 = m[0] + m[2], c1 = m[1] + m[3];
      m[0] /= c0; m[2] /= c0; m[1] /= c1; m[3] /= c1;
    }
  }
}

// exp(l - max) of the four residual logits, then the Sinkhorn above.
__device__ __forceinline__ void residual_map(const float* l4, int iters, float m[4]) {
  const float mx = fmaxf(fmaxf(l4[0], l4[1]), fmaxf(l4[2], l4[3]));
  const float mn = fminf(fminf(l4[0], l4[1]), fminf(l4[2], l4[3]));
#pragma unroll
  for (int i = 0; i < 4; ++i) m[i] = expf(l4[i] - mx);
  sinkhorn2(m, iters, mx - mn);
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
    residual_map(lt + 4, iters, m);
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
    residual_map(lt + 4, iters, m);
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


// ------------------------------------------------------------------ cluster kernel (bf16)
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_arrive() { asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory"); }
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory"); }
// Address of the same shared variable in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t peer_addr(uint32_t a, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(rank));
  return r;
}
// Bulk copy of this CTA's shared memory into a peer's (dst, bar: peer addresses),
// completing on the peer's mbarrier.
__device__ __forceinline__ void bulk_s2peer(uint32_t dst, uint32_t src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "r"(src), "r"(bytes), "r"(bar)
               : "memory");
}

// 1-D bulk copy global -> this CTA's shared memory, completing on an mbarrier.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}

// Shared-memory plan of mhc_cluster_kernel.
template <int TB, int NCH>
struct MhcCl {
  static constexpr int S = 256 * NCH;          // slice of each stream owned by a CTA
  static constexpr int RS = 2 * S + 8;         // row stride (elements) of the stream rows; +16 B vs. bank conflicts
  static constexpr int X_B = TB * RS * 2;      // the two streams' slices [TB][2S], mixed in place
  static constexpr int F_B = TB * S * 2;       // the layer output's slice [TB][S]; afterwards the per-warp
                                               // routing partials [8][TB][8] fp32
  static constexpr int PART_B = TB * 9 * 4;    // this slice's 8 routing sums + sum of squares [TB][9]
  static constexpr int GATH_B = 8 * PART_B;    // the same from every CTA of the cluster [CL <= 8][TB][9]
  static constexpr int SS_B = TB * 4, COEF_B = TB * 2 * 4, CIN_B = TB * 8 * 4, BR_B = 8 * 4;
  static constexpr int OFF_F = X_B, OFF_PART = OFF_F + F_B, OFF_GATH = OFF_PART + PART_B,
                       OFF_SS = OFF_GATH + GATH_B, OFF_COEF = OFF_SS + SS_B, OFF_CIN = OFF_COEF + COEF_B,
                       OFF_BR = OFF_CIN + CIN_B, OFF_BAR = (OFF_BR + BR_B + 15) / 16 * 16;
  static constexpr size_t BYTES = (size_t)OFF_BAR + 32;   // two mbarriers + the abort flag
  static_assert(PART_B % 16 == 0 && OFF_PART % 16 == 0 && OFF_GATH % 16 == 0, "bulk-copy alignment");
  static_assert(F_B >= 8 * TB * 8 * 4, "routing partials overlay the F rows");
};

template <int TB, int NCH, int MODE>
__global__ void __launch_bounds__(256, 2) mhc_cluster_kernel(const __nv_bfloat16* X_in, const __nv_bfloat16* F,
                                                            const float* __restrict__ coeffs_in,
                                                            const float* __restrict__ w_r,
                                                            const float* __restrict__ b_r, __nv_bfloat16* X_out,
                                                            __nv_bfloat16* __restrict__ x_in,
                                                            float* __restrict__ coeffs_out, int N, int d, int CL,
                                                            float eps, int iters) {
  using P = MhcCl<TB, NCH>;
  constexpr int S = P::S, RS = P::RS;
  constexpr int KT = S / 64;                   // 16-deep k-steps of the routing product per warp (2S / 16 / 8)
  static_assert(TB % 16 == 0 && TB * 8 <= 256, "token block");
  extern __shared__ __align__(16) unsigned char smem[];
  __nv_bfloat16* Ys = reinterpret_cast<__nv_bfloat16*>(smem);
  __nv_bfloat16* Fs = reinterpret_cast<__nv_bfloat16*>(smem + P::OFF_F);
  float* red = reinterpret_cast<float*>(smem + P::OFF_F);
  float* part = reinterpret_cast<float*>(smem + P::OFF_PART);
  float* gath = reinterpret_cast<float*>(smem + P::OFF_GATH);
  float* ssv = reinterpret_cast<float*>(smem + P::OFF_SS);
  float* coef = reinterpret_cast<float*>(smem + P::OFF_COEF);
  float* cin = reinterpret_cast<float*>(smem + P::OFF_CIN);
  float* brs = reinterpret_cast<float*>(smem + P::OFF_BR);
  const uint32_t bar = su32(smem + P::OFF_BAR);          // the staged rows
  const uint32_t bar_x = su32(smem + P::OFF_BAR + 8);    // the partial sums of all CTAs
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + P::OFF_BAR + 16);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_rank();
  const long t0 = (long)(blockIdx.x / CL) * TB;
  const int j0 = (int)rank * S;
  const int nt = (int)min((long)TB, (long)N - t0);   // tokens of this block that exist (>= 1)

  // ---- 1a. stage the slices of the block's tokens: one bulk copy per row, all in flight at once
  if (tid == 0) {
    tc::mbar_init(bar, 1);
    tc::mbar_init(bar_x, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    tc::mbar_expect_tx(bar_x, (uint32_t)(CL * P::PART_B));
  }
  __syncthreads();
  cluster_arrive();                            // every CTA's mbarriers exist before any peer copies into them
  if (warp == 0) {
    constexpr uint32_t rowb = S * 2;
    const uint32_t per_tok = (MODE == MHC_OPEN) ? rowb : (MODE == MHC_MIX ? 3 * rowb : 2 * rowb);
    if (lane == 0) tc::mbar_expect_tx(bar, per_tok * (uint32_t)nt);
    __syncwarp();
    for (int t = lane; t < nt; t += 32) {
      const long tok = t0 + t;
      const uint32_t dx = su32(Ys + t * RS);
      if (MODE == MHC_OPEN) {
        bulk_g2s(dx, X_in + tok * d + j0, rowb, bar);
      } else {
        bulk_g2s(dx, X_in + tok * 2 * d + j0, rowb, bar);
        bulk_g2s(dx + rowb, X_in + tok * 2 * d + d + j0, rowb, bar);
        if (MODE == MHC_MIX) bulk_g2s(su32(Fs + t * S), F + tok * d + j0, rowb, bar);
      }
    }
  }
  // while the rows are in flight: zero rows past the end of the sequence (they enter the
  // routing products), fetch the mixing coefficients, the routing bias and this warp's
  // share of the routing map
  for (int i = nt * (2 * S / 8) + tid; i < TB * (2 * S / 8); i += 256) {
    const int t = i / (2 * S / 8), e = (i % (2 * S / 8)) * 8;
    *reinterpret_cast<uint4*>(Ys + t * RS + e) = make_uint4(0, 0, 0, 0);
  }
  if (MODE == MHC_MIX && tid < nt * 8) cin[tid] = coeffs_in[t0 * 8 + tid];
  if (tid < 8) brs[tid] = b_r[tid];
  const int q = lane & 3, n = lane >> 2;
  const int kw = warp * (S / 4);               // this warp's k range [kw, kw + S/4) of the local 2S
  float wf[KT][4];
#pragma unroll
  for (int kt = 0; kt < KT; ++kt) {
    const int k = kw + kt * 16;                // stream k / S, element k % S of the slice
    const long row = (k < S) ? (long)j0 + k : (long)d + j0 + (k - S);
    wf[kt][0] = __ldg(w_r + (row + 2 * q) * 8 + n);
    wf[kt][1] = __ldg(w_r + (row + 2 * q + 1) * 8 + n);
    wf[kt][2] = __ldg(w_r + (row + 2 * q + 8) * 8 + n);
    wf[kt][3] = __ldg(w_r + (row + 2 * q + 9) * 8 + n);
  }
  tc::mbar_wait(bar, 0, abort_flag);
  __syncthreads();                             // cin, brs, zero rows

  // ---- 1b. mix in place; warp w owns tokens w, w + 8, ...
#pragma unroll 1
  for (int i = 0; i < TB / 8; ++i) {
    const int t = warp + 8 * i;
    if (t >= nt) {
      if (lane == 0) ssv[t] = 0.f;
      continue;
    }
    const long tok = t0 + t;
    float co[6] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    if (MODE == MHC_MIX) {
#pragma unroll
      for (int k = 0; k < 6; ++k) co[k] = cin[t * 8 + 2 + k];   // H_post (2), H_res (2x2)
    }
    float ss = 0.f;
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
      const int e = c * 256 + lane * 8;
      float x0[8], x1[8], y0[8], y1[8];
      load8(Ys + t * RS + e, x0);
      if (MODE == MHC_OPEN) {
#pragma unroll
        for (int k = 0; k < 8; ++k) x1[k] = x0[k];
      } else {
        load8(Ys + t * RS + S + e, x1);
      }
      if (MODE == MHC_MIX) {
        float f[8];
        load8(Fs + t * S + e, f);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          y0[k] = co[2] * x0[k] + co[3] * x1[k] + co[0] * f[k];
          y1[k] = co[4] * x0[k] + co[5] * x1[k] + co[1] * f[k];
        }
        round8<__nv_bfloat16>(y0);
        round8<__nv_bfloat16>(y1);
      } else {
#pragma unroll
        for (int k = 0; k < 8; ++k) { y0[k] = x0[k]; y1[k] = x1[k]; }
      }
#pragma unroll
      for (int k = 0; k < 8; ++k) ss += y0[k] * y0[k] + y1[k] * y1[k];
      if (MODE != MHC_ROUTE) {
        store8(Ys + t * RS + e, y0);
        store8(Ys + t * RS + S + e, y1);
        store8(X_out + tok * 2 * d + j0 + e, y0);
        store8(X_out + tok * 2 * d + d + j0 + e, y1);
      }
    }
    ss = warp_sum(ss);
    if (lane == 0) ssv[t] = ss;
  }
  __syncthreads();                             // mixed rows complete; the F rows are free

  // ---- 2. this slice's routing sums: [TB x 2S] (bf16) x [2S x 8] (FP32 = hi + mid + lo, bf16 each)
  {
    constexpr int MT = TB / 16;
    float acc[MT][4];
#pragma unroll
    for (int m = 0; m < MT; ++m) acc[m][0] = acc[m][1] = acc[m][2] = acc[m][3] = 0.f;
#pragma unroll
    for (int kt = 0; kt < KT; ++kt) {
      const int k = kw + kt * 16;
      float hi[4], mid[4], lo[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        hi[i] = __bfloat162float(__float2bfloat16(wf[kt][i]));
        const float r1 = wf[kt][i] - hi[i];
        mid[i] = __bfloat162float(__float2bfloat16(r1));
        lo[i] = r1 - mid[i];
      }
      const uint32_t bh[2] = {pack_bf2(hi[0], hi[1]), pack_bf2(hi[2], hi[3])};
      const uint32_t bm[2] = {pack_bf2(mid[0], mid[1]), pack_bf2(mid[2], mid[3])};
      const uint32_t bl[2] = {pack_bf2(lo[0], lo[1]), pack_bf2(lo[2], lo[3])};
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        uint32_t af[4];
        const int r = m * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
        ldsm_x4(af, Ys + r * RS + k + (lane >> 4) * 8);
        mma16816(acc[m], af, bl);
        mma16816(acc[m], af, bm);
        mma16816(acc[m], af, bh);
      }
    }
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      const int t = m * 16 + n;
      float* rw = red + (warp * TB + t) * 8 + 2 * q;
      rw[0] = acc[m][0];
      rw[1] = acc[m][1];
      rw[8 * 8] = acc[m][2];                   // token t + 8
      rw[8 * 8 + 1] = acc[m][3];
    }
  }
  __syncthreads();
  // ---- 3. this slice's 9 sums per token, copied into slot [rank] of every CTA of the cluster
  for (int i = tid; i < TB * 9; i += 256) {
    const int t = i / 9, o = i - t * 9;
    float v;
    if (o < 8) {
      v = 0.f;
#pragma unroll
      for (int w = 0; w < 8; ++w) v += red[(w * TB + t) * 8 + o];
    } else {
      v = ssv[t];
    }
    part[i] = v;
  }
  tc::fence_proxy_async();                     // the copies read `part` through the async proxy
  __syncthreads();
  cluster_wait();                              // (pairs with the arrive after the mbarrier set-up)
  if (tid == 0) {
    const uint32_t src = su32(part), dst = su32(gath + (int)rank * TB * 9);
    for (int r = 0; r < CL; ++r)
      bulk_s2peer(peer_addr(dst, (uint32_t)r), src, (uint32_t)P::PART_B, peer_addr(bar_x, (uint32_t)r));
  }
  tc::mbar_wait(bar_x, 0, abort_flag);         // all CL slices' sums have landed here
  cluster_arrive();                            // ... so this CTA's own copies into its peers are done too
                                               // once every CTA has arrived (matched at the end)

  // ---- 4. full sums in rank order (bit-identical in every CTA), coefficients; the Sinkhorn
  //         of token t runs in CTA t mod CL
  if (tid < TB) {
    const int t = tid;
    const long tok = t0 + t;
    float v[9];
#pragma unroll
    for (int o = 0; o < 9; ++o) v[o] = 0.f;
    for (int r = 0; r < CL; ++r) {
#pragma unroll
      for (int o = 0; o < 9; ++o) v[o] += gath[(r * TB + t) * 9 + o];
    }
    const float inv = rsqrtf(v[8] / (float)(2 * d) + eps);
    float lt[8];
#pragma unroll
    for (int o = 0; o < 8; ++o) lt[o] = v[o] * inv + brs[o];
    const float pre0 = sigmoidf_acc(lt[0]), pre1 = sigmoidf_acc(lt[1]);
    coef[2 * t] = pre0;
    coef[2 * t + 1] = pre1;
    if (t % CL == (int)rank && tok < N) {
      float m[4];
      residual_map(lt + 4, iters, m);
      float4* c = reinterpret_cast<float4*>(coeffs_out + tok * 8);
      c[0] = make_float4(pre0, pre1, 2.f * sigmoidf_acc(lt[2]), 2.f * sigmoidf_acc(lt[3]));
      c[1] = make_float4(m[0], m[1], m[2], m[3]);
    }
  }
  __syncthreads();

  // ---- 5. layer input for this slice from the mixed streams held in shared memory
#pragma unroll 1
  for (int i = 0; i < TB / 8; ++i) {
    const int t = warp + 8 * i;
    if (t >= nt) break;
    const long tok = t0 + t;
    const float p0 = coef[2 * t], p1 = coef[2 * t + 1];
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
      const int e = c * 256 + lane * 8;
      float y0[8], y1[8], o[8];
      load8(Ys + t * RS + e, y0);
      load8(Ys + t * RS + S + e, y1);
#pragma unroll
      for (int k = 0; k < 8; ++k) o[k] = p0 * y0[k] + p1 * y1[k];
      store8(x_in + tok * d + j0 + e, o);
    }
  }
  cluster_wait();                              // no CTA leaves while a copy out of its shared memory may run
}

// MERGE: h = (y0 + y1) / 2 with y = H_res X + H_post F, one thread per 8 elements.
template <typename T>
__global__ void __launch_bounds__(256) mhc_merge_kernel(const T* __restrict__ X, const T* __restrict__ F,
                                                        const float* __restrict__ coeffs, T* __restrict__ h,
                                                        long N, int d) {
  const long groups = (long)d / 8;
  const long i = (long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= N * groups) return;
  const long tok = i / groups;
  const int j = (int)(i - tok * groups) * 8;
  const float4 c0 = __ldg(reinterpret_cast<const float4*>(coeffs + tok * 8));
  const float4 c1 = __ldg(reinterpret_cast<const float4*>(coeffs + tok * 8 + 4));
  float x0[8], x1[8], f[8], o[8];
  load8(X + tok * 2 * d + j, x0);
  load8(X + tok * 2 * d + d + j, x1);
  load8(F + tok * d + j, f);
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const float y0 = c1.x * x0[k] + c1.y * x1[k] + c0.z * f[k];
    const float y1 = c1.z * x0[k] + c1.w * x1[k] + c0.w * f[k];
    o[k] = 0.5f * (y0 + y1);
  }
  store8(h + tok * d + j, o);
}

// Smallest token count sent to the cluster kernel (below it the CTA-per-token kernel
// spreads the work over more SMs).
constexpr int kClusterMinTokens = 1024;

// Cluster shape for width d: CL CTAs x NCH 256-element chunks per stream slice.
static bool cluster_shape(int d, int& CL, int& nch) {
  if (d <= 0 || d % 256) return false;
  const int u = d / 256;
  for (int c : {1, 2, 4}) {
    if (u % c == 0 && u / c <= 8 && ((u / c) & (u / c - 1)) == 0) {
      nch = c;
      CL = u / c;
      return true;
    }
  }
  return false;
}

template <int TB, int NCH, int MODE>
static cudaError_t launch_cluster(const void* X_in, const void* F, const float* coeffs_in, const float* w_r,
                                  const float* b_r, void* X_out, void* x_in, float* coeffs_out, int N, int d, int CL,
                                  float eps, int iters, cudaStream_t s) {
  auto kern = mhc_cluster_kernel<TB, NCH, MODE>;
  const size_t bytes = MhcCl<TB, NCH>::BYTES;
  cudaError_t e = set_smem_limit(kern, (int)bytes);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(((long)N + TB - 1) / TB * CL));
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = bytes;
  cfg.stream = s;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = (unsigned)CL;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, (const __nv_bfloat16*)X_in, (const __nv_bfloat16*)F, coeffs_in, w_r, b_r,
                            (__nv_bfloat16*)X_out, (__nv_bfloat16*)x_in, coeffs_out, N, d, CL, eps, iters);
}

template <int NCH>
static cudaError_t cluster_mode(int mode, const void* X_in, const void* F, const float* coeffs_in, const float* w_r,
                                const float* b_r, void* X_out, void* x_in, float* coeffs_out, int N, int d, int CL,
                                float eps, int iters, cudaStream_t s) {
  constexpr int TB = 32;
  switch (mode) {
    case MHC_OPEN:
      return launch_cluster<TB, NCH, MHC_OPEN>(X_in, F, coeffs_in, w_r, b_r, X_out, x_in, coeffs_out, N, d, CL, eps,
                                               iters, s);
    case MHC_MIX:
      return launch_cluster<TB, NCH, MHC_MIX>(X_in, F, coeffs_in, w_r, b_r, X_out, x_in, coeffs_out, N, d, CL, eps,
                                              iters, s);
    default:
      return launch_cluster<TB, NCH, MHC_ROUTE>(X_in, F, coeffs_in, w_r, b_r, X_out, x_in, coeffs_out, N, d, CL,
                                                eps, iters, s);
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
  if (mode == MHC_MERGE && d % 8 == 0) {
    const long n = (long)N * (d / 8);
    const unsigned blocks = (unsigned)((n + 255) / 256);
    if (dtype == BF16)
      mhc_merge_kernel<__nv_bfloat16><<<blocks, 256, 0, s>>>((const __nv_bfloat16*)X_in, (const __nv_bfloat16*)F,
                                                              coeffs_in, (__nv_bfloat16*)h_out, N, d);
    else
      mhc_merge_kernel<float><<<blocks, 256, 0, s>>>((const float*)X_in, (const float*)F, coeffs_in, (float*)h_out,
                                                     N, d);
    return cudaGetLastError();
  }
  int CL = 0, nch = 0;
  if (dtype == BF16 && mode != MHC_MERGE && N >= kClusterMinTokens && cluster_shape(d, CL, nch)) {
    switch (nch) {
      case 1: return cluster_mode<1>(mode, X_in, F, coeffs_in, w_r, b_r, X_out, x_in, coeffs_out, N, d, CL, eps, iters, s);
      case 2: return cluster_mode<2>(mode, X_in, F, coeffs_in, w_r, b_r, X_out, x_in, coeffs_out, N, d, CL, eps, iters, s);
      default: return cluster_mode<4>(mode, X_in, F, coeffs_in, w_r, b_r, X_out, x_in, coeffs_out, N, d, CL, eps, iters, s);
    }
  }
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
