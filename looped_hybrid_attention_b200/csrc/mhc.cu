// Two-stream mHC residual ("Loop-9B engineering teardown" §五, §六; "SenseNova-Loop-9B
// 是什么" §二): one kernel per layer boundary mixes the previous layer's output into
// the two streams, then computes the next layer's routing (FP32 logits, FP32
// Sinkhorn) and reads the layer input -- the streams cross HBM once per boundary.
//
// bf16 streams, many tokens (mhc_cluster_kernel): a persistent cluster of CL CTAs walks
// blocks of TB tokens; CTA r owns the slice [r S, (r+1) S) of both streams.  A block's
// rows arrive as single TMA boxes (double-buffered: the next block loads while this one
// is processed).  Each CTA mixes its slice in shared memory and sends it back out by TMA,
// forms its slice's share of the 8 routing dot products and of the sum of squares on the
// tensor cores (mma.sync; the FP32 map enters as the exact sum of three bf16 terms and
// the streams are bf16 already, so every product is exact and the sums are FP32), and the
// CTAs exchange their partial sums through distributed shared memory.  Every CTA adds the
// partials in rank order, so all of them hold bit-identical coefficients, and each writes
// its slice of the layer input from shared memory -- nothing is re-read from HBM.
//
// fp32 streams or few tokens: the warp-per-4-tokens kernel (mhc_kernel) or the
// CTA-per-token kernel (mhc_token_kernel), FP32 FMAs throughout.
//
// MERGE (the last boundary) is a plain streaming kernel: h = (X0' + X1') / 2.
#include "common.cuh"
#include "internal.h"
#include "mma_sync.cuh"
#include "tc_common.cuh"

#include <algorithm>
#include <map>
#include <mutex>
#include <tuple>

namespace lk {

// 2x2 Sinkhorn in registers: `iters` rounds of row then column normalisation, on
// m = exp(l - max l), whose smallest entry is exp(-spread).
//
// Row normalisation keeps each row's odds x = m0/m1, y = m2/m3; the column normalisation
// that follows multiplies both by c1/c0, the ratio of the column sums of the row-
// normalised matrix [[x/(1+x), 1/(1+x)], [y/(1+y), 1/(1+y)]], which is
// (2 + x + y) / (x + y + 2xy).  So the rounds before the last one update the two odds
// (one reciprocal each), and the last round writes the column-normalised matrix from
// them.  The odds stay within exp(+-spread) and their product within exp(+-2 spread):
// for spread <= 40 nothing overflows and the reciprocals come from the hardware
// (rcp.approx, within about one ulp).  Wider spreads run the same rounds in the log domain
// (each row, then each column, minus its log-sum-exp): in the linear domain the smallest
// entries exp(-spread) would lose their precision to fp32 denormals (spread > ~87) or to
// the row and column sums they are divided by.
__device__ __forceinline__ float rcp_hw(float x) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}
__device__ __forceinline__ void sinkhorn2(float m[4], int iters) {
  if (iters <= 0) return;
  {
    float x = m[0] / m[1], y = m[2] / m[3];
#pragma unroll 4
    for (int it = 1; it < iters; ++it) {
      const float s = x + y;
      const float f = (2.f + s) * rcp_hw(fmaf(x + x, y, s));
      x *= f;
      y *= f;
    }
    const float px = rcp_hw(1.f + x), py = rcp_hw(1.f + y);   // the row-normalised second column
    const float a = x * px, b = y * py;                         // ... and first column
    const float r0 = rcp_hw(a + b), r1 = rcp_hw(px + py);
    m[0] = a * r0;
    m[2] = b * r0;
    m[1] = px * r1;
    m[3] = py * r1;
  }
}

// log(e^a + e^b)
__device__ __forceinline__ float lse2(float a, float b) { return fmaxf(a, b) + log1pf(expf(-fabsf(a - b))); }

// The rounds of sinkhorn2 in the log domain, from x = l - max l; writes exp(x).
__device__ __forceinline__ void sinkhorn2_log(const float x_in[4], int iters, float m[4]) {
  float x0 = x_in[0], x1 = x_in[1], x2 = x_in[2], x3 = x_in[3];
  for (int it = 0; it < iters; ++it) {
    const float r0 = lse2(x0, x1), r1 = lse2(x2, x3);
    x0 -= r0; x1 -= r0; x2 -= r1; x3 -= r1;
    const float c0 = lse2(x0, x2), c1 = lse2(x1, x3);
    x0 -= c0; x2 -= c0; x1 -= c1; x3 -= c1;
  }
  m[0] = expf(x0); m[1] = expf(x1); m[2] = expf(x2); m[3] = expf(x3);
}

// exp(l - max) of the four residual logits, then the Sinkhorn above.
__device__ __forceinline__ void residual_map(const float* l4, int iters, float m[4]) {
  const float mx = fmaxf(fmaxf(l4[0], l4[1]), fmaxf(l4[2], l4[3]));
  const float mn = fminf(fminf(l4[0], l4[1]), fminf(l4[2], l4[3]));
  if (mx - mn <= 40.f) {
#pragma unroll
    for (int i = 0; i < 4; ++i) m[i] = expf(l4[i] - mx);
    sinkhorn2(m, iters);
  } else {
    const float x[4] = {l4[0] - mx, l4[1] - mx, l4[2] - mx, l4[3] - mx};
    sinkhorn2_log(x, iters, m);
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
// Arrival without release semantics: for hand-offs whose data moves by bulk copies that
// complete on mbarriers (the waits on those mbarriers order the data; the cluster barrier
// only says that a CTA is past them).
__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
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


// Shared-memory plan of mhc_cluster_kernel.  Two token-block buffers (the block in use and
// the next one, in flight).  Each holds the two streams' slices as S/64 runs of
// [TB tokens][2 streams][64] bf16 (128-byte line 2t + s), a row slice as S/64 runs of
// [TB][64] (line t): the layer output F (mix), the stream h (open), later the layer input
// being written; and the block's incoming coefficients.  Each of the three arrives as ONE
// TMA box: the tensors are viewed with the 64-column chunk as their outermost dimension,
// so a box spans the whole slice, and the 128-byte swizzle keeps every access pattern
// below free of bank conflicts (ldmatrix rows 2t + s: two-way at most).
template <int TB, int NCH>
struct MhcCl {
  static constexpr int S = 256 * NCH;          // slice of each stream owned by a CTA
  static constexpr int XBOX = TB * 2 * 128, FBOX = TB * 128;
  static constexpr int X_B = (S / 64) * XBOX, F_B = (S / 64) * FBOX;
  static constexpr int CIN_B = TB * 8 * 4;     // the block's incoming coefficients [TB][8] fp32 (mix)
  static constexpr int BUF_B = (X_B + F_B + CIN_B + 1023) / 1024 * 1024;
  static constexpr int PART_B = TB * 9 * 4;    // this slice's 8 routing sums + sum of squares [TB][9]
  static constexpr int GATH_B = 8 * PART_B;    // the same from every CTA of the cluster [CL <= 8][TB][9]
  static constexpr int COEF_B = TB * 2 * 4, BR_B = 8 * 4;
  static constexpr int OFF_PART = 2 * BUF_B, OFF_GATH = OFF_PART + PART_B, OFF_COEF = OFF_GATH + GATH_B,
                       OFF_BR = OFF_COEF + COEF_B,
                       OFF_BAR = (OFF_BR + BR_B + 15) / 16 * 16;
  static constexpr size_t BYTES = (size_t)OFF_BAR + 32 + 1024;   // rows landed [2], sums landed, abort; alignment
  static_assert(BUF_B % 1024 == 0, "swizzled boxes start on 1024-byte boundaries");
  static_assert(PART_B % 16 == 0 && OFF_PART % 16 == 0 && OFF_GATH % 16 == 0, "bulk-copy alignment");
  static_assert(F_B >= 8 * TB * 9 * 4, "routing partials overlay the row slice");
};

// 8 floats -> 8 bf16 (round to nearest even) and back.
__device__ __forceinline__ uint4 pack8_bf(const float* f) {
  uint4 u;
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
  return u;
}
__device__ __forceinline__ void unpack8_bf(const uint4& u, float* f) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) { const float2 t = __bfloat1622float2(h[i]); f[2 * i] = t.x; f[2 * i + 1] = t.y; }
}
// An FP32 value as the exact sum of three bf16 terms (hi + mid + lo), two values per word.
__device__ __forceinline__ void split3_bf(const float (&w)[4], uint32_t (&b)[6]) {
  float hi[4], mid[4], lo[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    hi[i] = __bfloat162float(__float2bfloat16(w[i]));
    const float r1 = w[i] - hi[i];
    mid[i] = __bfloat162float(__float2bfloat16(r1));
    lo[i] = r1 - mid[i];
  }
  b[0] = pack_bf2(hi[0], hi[1]);
  b[1] = pack_bf2(hi[2], hi[3]);
  b[2] = pack_bf2(mid[0], mid[1]);
  b[3] = pack_bf2(mid[2], mid[3]);
  b[4] = pack_bf2(lo[0], lo[1]);
  b[5] = pack_bf2(lo[2], lo[3]);
}

// Byte offset of elements k..k+7 (k a multiple of 8) of 128-byte line `line` in a run of
// 64-column boxes of box_b bytes each, 128-byte swizzled.
__device__ __forceinline__ uint32_t swz(int box_b, int line, int k) {
  return (uint32_t)((k >> 6) * box_b + line * 128 + ((((k & 63) >> 3) ^ (line & 7)) << 4));
}

// Persistent: cluster c takes token blocks c, c + n_clusters, ...; while one block is mixed,
// routed and written, the next block's rows are already being loaded.  Rows come in and go
// out as TMA boxes (rows past the sequence end load as zeros and are not stored).
template <int TB, int NCH, int MODE>
__global__ void __launch_bounds__(256, NCH <= 2 ? 2 : 1) mhc_cluster_kernel(const __grid_constant__ CUtensorMap mX,
                                                          const __grid_constant__ CUtensorMap mF,
                                                          const __grid_constant__ CUtensorMap mXo,
                                                          const __grid_constant__ CUtensorMap mXi,
                                                          const __grid_constant__ CUtensorMap mC,
                                                          const float* __restrict__ w_r, const float* __restrict__ b_r,
                                                          float* __restrict__ coeffs_out, int N, int d, int CL,
                                                          float eps, int iters) {
  using P = MhcCl<TB, NCH>;
  constexpr int S = P::S, NB = S / 64;
  constexpr int KT = S / 64;                   // 16-deep k-steps of the routing product per warp (2S / 16 / 8)
  static_assert(TB % 16 == 0 && TB * 8 <= 256, "token block");
  extern __shared__ __align__(16) unsigned char smem_raw[];
  unsigned char* smem = (unsigned char*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  float* part = reinterpret_cast<float*>(smem + P::OFF_PART);
  float* gath = reinterpret_cast<float*>(smem + P::OFF_GATH);
  float* coef = reinterpret_cast<float*>(smem + P::OFF_COEF);
  float* brs = reinterpret_cast<float*>(smem + P::OFF_BR);
  const uint32_t bar_rows = su32(smem + P::OFF_BAR);     // + 8 * buffer: that buffer's rows landed
  const uint32_t bar_x = bar_rows + 16;                  // the partial sums of all CTAs landed
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + P::OFF_BAR + 24);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_rank();
  const long n_cl = gridDim.x / CL, n_blk = ((long)N + TB - 1) / TB;
  const int j0 = (int)rank * S;
  constexpr uint32_t TX = (MODE == MHC_OPEN) ? P::F_B : (MODE == MHC_MIX ? P::X_B + P::F_B + P::CIN_B : P::X_B);

  if (tid == 0) {
    tc::mbar_init(bar_rows, 1);
    tc::mbar_init(bar_rows + 8, 1);
    tc::mbar_init(bar_x, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    tc::mbar_expect_tx(bar_x, (uint32_t)(CL * P::PART_B));   // the first block's exchange
    asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&mX) : "memory");
    if (MODE == MHC_MIX) asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&mF) : "memory");
    if (MODE == MHC_MIX) asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&mC) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&mXi) : "memory");
    if (MODE != MHC_ROUTE) asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&mXo) : "memory");
  }
  __syncthreads();
  cluster_arrive();                            // every CTA's mbarriers exist before any peer copies into them

  // the rows of block `blk` into buffer `bf` (one thread; the buffer's earlier readers are done)
  auto issue = [&](long blk, int bf) {
    unsigned char* buf = smem + bf * P::BUF_B;
    const uint32_t bar = bar_rows + 8 * bf;
    const int y = (int)(blk * TB), ch = j0 / 64;
    tc::bulk_wait_read<0>();                   // stores out of this buffer have read it
    tc::fence_proxy_async();
    tc::mbar_expect_tx(bar, TX);
    if (MODE == MHC_OPEN) {
      tc::tma_load_3d(su32(buf + P::X_B), &mX, bar, 0, y, ch);
    } else {
      tc::tma_load_4d(su32(buf), &mX, bar, 0, 0, y, ch);
      if (MODE == MHC_MIX) {
        tc::tma_load_3d(su32(buf + P::X_B), &mF, bar, 0, y, ch);
        tc::tma_load_2d(su32(buf + P::X_B + P::F_B), &mC, bar, 0, y);
      }
    }
  };
  const long first = blockIdx.x / CL;
  if (tid == 0 && first < n_blk) issue(first, 0);

  // this warp's share of the routing map (kept for every block) and the routing bias
  if (tid < 8) brs[tid] = b_r[tid];
  const int q = lane & 3, n = lane >> 2;
  const int kw = warp * (S / 4);               // this warp's k range [kw, kw + S/4) of the local 2S
  constexpr bool PRE = KT <= 8;               // few k-steps: keep the bf16 split, not the FP32 values
  float wf[PRE ? 1 : KT][4];
  uint32_t wb[PRE ? KT : 1][6];
#pragma unroll
  for (int kt = 0; kt < KT; ++kt) {
    const int k = kw + kt * 16;                // stream k / S, element k % S of the slice
    const long row = (k < S) ? (long)j0 + k : (long)d + j0 + (k - S);
    float w4[4];
    w4[0] = __ldg(w_r + (row + 2 * q) * 8 + n);
    w4[1] = __ldg(w_r + (row + 2 * q + 1) * 8 + n);
    w4[2] = __ldg(w_r + (row + 2 * q + 8) * 8 + n);
    w4[3] = __ldg(w_r + (row + 2 * q + 9) * 8 + n);
    if constexpr (PRE) {
      split3_bf(w4, wb[kt]);
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i) wf[kt][i] = w4[i];
    }
  }
  using bf = __nv_bfloat16;
  // the Sinkhorn of a token runs one block later, while this CTA waits for the next
  // block's exchange: its residual logits and token index wait in registers
  float sk_l[4] = {0.f, 0.f, 0.f, 0.f};
  long sk_tok = -1;
  auto sinkhorn_pending = [&]() {
    if (sk_tok >= 0) {
      float m[4];
      residual_map(sk_l, iters, m);
      *reinterpret_cast<float4*>(coeffs_out + sk_tok * 8 + 4) = make_float4(m[0], m[1], m[2], m[3]);
      sk_tok = -1;
    }
  };
  int it = 0;
#pragma unroll 1
  for (long blk = first; blk < n_blk; blk += n_cl, ++it) {
    const int bi = it & 1;
    unsigned char* Xb = smem + bi * P::BUF_B;  // stream boxes
    unsigned char* Fb = Xb + P::X_B;           // row-slice boxes
    const float* cin = reinterpret_cast<const float*>(Fb + P::F_B);
    float* red = reinterpret_cast<float*>(Fb);
    const long t0 = blk * TB;
    const int nt = (int)min((long)TB, (long)N - t0);   // tokens of this block that exist (>= 1)
    tc::mbar_wait(bar_rows + 8 * bi, (uint32_t)((it >> 1) & 1), abort_flag);
    __syncthreads();                           // rows, coefficients (zeros past the end)

    // ---- 1. mix in place; warp w owns tokens w, w + 8, ... (rows past the end are zeros)
    if (MODE != MHC_ROUTE) {
#pragma unroll
      for (int i = 0; i < TB / 8; ++i) {
        const int t = warp + 8 * i;
        float co[6] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        if (MODE == MHC_MIX) {
#pragma unroll
          for (int k = 0; k < 6; ++k) co[k] = cin[t * 8 + 2 + k];   // H_post (2), H_res (2x2)
        }
#pragma unroll
        for (int c = 0; c < NCH; ++c) {
          const int e = c * 256 + lane * 8;
          uint4* p0 = reinterpret_cast<uint4*>(Xb + swz(P::XBOX, 2 * t, e));
          uint4* p1 = reinterpret_cast<uint4*>(Xb + swz(P::XBOX, 2 * t + 1, e));
          const uint4* pf = reinterpret_cast<const uint4*>(Fb + swz(P::FBOX, t, e));
          if (MODE == MHC_OPEN) {
            const uint4 u = *pf;               // h into both streams
            *p0 = u;
            *p1 = u;
          } else {
            float x0[8], x1[8], f[8], y0[8], y1[8];
            unpack8_bf(*p0, x0);
            unpack8_bf(*p1, x1);
            unpack8_bf(*pf, f);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              y0[k] = co[2] * x0[k] + co[3] * x1[k] + co[0] * f[k];
              y1[k] = co[4] * x0[k] + co[5] * x1[k] + co[1] * f[k];
            }
            *p0 = pack8_bf(y0);
            *p1 = pack8_bf(y1);
          }
        }
      }
    }
    if (MODE != MHC_ROUTE) tc::fence_proxy_async();   // the mixed rows leave by TMA stores
    __syncthreads();                           // mixed rows complete; the row slice is free
    if (tid == 0) {
      // the next block's rows into the other buffer (free since the end of the last block),
      // then this block's mixed streams out
      if (blk + n_cl < n_blk) issue(blk + n_cl, bi ^ 1);
      if (MODE != MHC_ROUTE) {
        tc::tma_store_4d(&mXo, su32(Xb), 0, 0, (int)t0, j0 / 64);
        tc::bulk_commit();
      }
    }

    // ---- 2. this slice's routing sums: [TB x 2S] (bf16) x [2S x 8] (FP32 = hi + mid + lo, bf16
    //         each), and its sums of squares as the diagonal of the Gram matrix X X^T (the A
    //         fragment of X is also the B fragment of X^T: no extra loads); bf16 products are
    //         exact in FP32
    {
      constexpr int MT = TB / 16;
      float acc[MT][4], acm[MT][4], ach[MT][4];  // lo, mid, hi terms: three independent chains
      float g0[MT][4], g1[MT][4];                // Gram blocks: columns = tokens 0-7, 8-15 of the tile
#pragma unroll
      for (int m = 0; m < MT; ++m)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[m][i] = acm[m][i] = ach[m][i] = g0[m][i] = g1[m][i] = 0.f;
#pragma unroll
      for (int kt = 0; kt < KT; ++kt) {
        const int k = kw + kt * 16;
        const int sk = k >= S ? 1 : 0, kk = k - sk * S + (lane >> 4) * 8;   // stream, element of the slice
        uint32_t b6[6];
        if constexpr (PRE) {
#pragma unroll
          for (int i = 0; i < 6; ++i) b6[i] = wb[kt][i];
        } else {
          split3_bf(wf[kt], b6);
        }
        const uint32_t bh[2] = {b6[0], b6[1]}, bm[2] = {b6[2], b6[3]}, bl[2] = {b6[4], b6[5]};
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          uint32_t af[4];
          const int r = m * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
          ldsm_x4(af, reinterpret_cast<const bf*>(Xb + swz(P::XBOX, 2 * r + sk, kk)));
          mma16816(acc[m], af, bl);
          mma16816(acm[m], af, bm);
          mma16816(ach[m], af, bh);
          const uint32_t xt0[2] = {af[0], af[2]}, xt1[2] = {af[1], af[3]};
          mma16816(g0[m], af, xt0);
          mma16816(g1[m], af, xt1);
        }
      }
#pragma unroll
      for (int m = 0; m < MT; ++m) {
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[m][i] = (acc[m][i] + acm[m][i]) + ach[m][i];
        const int t = m * 16 + n;
        float* rw = red + (warp * TB + t) * 9 + 2 * q;
        rw[0] = acc[m][0];
        rw[1] = acc[m][1];
        rw[8 * 9] = acc[m][2];                 // token t + 8
        rw[8 * 9 + 1] = acc[m][3];
        if (q == (n >> 1)) {                   // this lane holds the diagonal entries (t, t), (t + 8, t + 8)
          red[(warp * TB + t) * 9 + 8] = (n & 1) ? g0[m][1] : g0[m][0];
          red[(warp * TB + t + 8) * 9 + 8] = (n & 1) ? g1[m][3] : g1[m][2];
        }
      }
    }
    __syncthreads();
    // every CTA of the cluster is done with the previous block's exchange: its sums have
    // landed everywhere (so `part` is free) and nobody reads `gath` any more
    cluster_wait();
    // ---- 3. this slice's 9 sums per token, copied into slot [rank] of every CTA of the cluster
    for (int i = tid; i < TB * 9; i += 256) {
      float v = 0.f;
#pragma unroll
      for (int w = 0; w < 8; ++w) v += red[w * TB * 9 + i];
      part[i] = v;
    }
    tc::fence_proxy_async();                   // the copies read `part` through the async proxy
    __syncthreads();
    if (tid < CL) {                            // lane r sends to CTA r
      const uint32_t src = su32(part), dst = su32(gath + (int)rank * TB * 9);
      bulk_s2peer(peer_addr(dst, (uint32_t)tid), src, (uint32_t)P::PART_B, peer_addr(bar_x, (uint32_t)tid));
    }
    sinkhorn_pending();                        // the previous block's, while the sums travel
    tc::mbar_wait(bar_x, (uint32_t)(it & 1), abort_flag);   // all CL slices' sums have landed here
    if (tid == 0) tc::mbar_expect_tx(bar_x, (uint32_t)(CL * P::PART_B));   // the next block's exchange

    // ---- 4. full sums in rank order (bit-identical in every CTA), coefficients: eight lanes
    //         per token, lane o owns logit o; token t's coefficients are written by CTA t mod CL
    if (tid < TB * 8) {
      const int t = tid >> 3, o = tid & 7;
      const long tok = t0 + t;
      float v = 0.f, sq = 0.f;
      for (int r = 0; r < CL; ++r) {
        v += gath[(r * TB + t) * 9 + o];
        sq += gath[(r * TB + t) * 9 + 8];
      }
      const float inv = rsqrtf(sq / (float)(2 * d) + eps);
      const float lt = v * inv + brs[o];
      const float cv = o < 2 ? sigmoidf_acc(lt) : 2.f * sigmoidf_acc(lt);   // H_pre, H_post (o < 4)
      if (o < 2) coef[2 * t + o] = cv;
      float l4[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) l4[j] = __shfl_sync(0xffffffffu, lt, (lane & ~7) + 4 + j);
      if (t % CL == (int)rank && tok < N) {
        if (o < 4) coeffs_out[tok * 8 + o] = cv;
        if (o == 4) {
#pragma unroll
          for (int j = 0; j < 4; ++j) sk_l[j] = l4[j];
          sk_tok = tok;
        }
      }
    }
    __syncthreads();

    // ---- 5. layer input for this slice from the mixed streams, into the row-slice boxes
#pragma unroll
    for (int i = 0; i < TB / 8; ++i) {
      const int t = warp + 8 * i;
      const float a0 = coef[2 * t], a1 = coef[2 * t + 1];
#pragma unroll
      for (int c = 0; c < NCH; ++c) {
        const int e = c * 256 + lane * 8;
        float y0[8], y1[8], o[8];
        load8(reinterpret_cast<const bf*>(Xb + swz(P::XBOX, 2 * t, e)), y0);
        load8(reinterpret_cast<const bf*>(Xb + swz(P::XBOX, 2 * t + 1, e)), y1);
#pragma unroll
        for (int k = 0; k < 8; ++k) o[k] = a0 * y0[k] + a1 * y1[k];
        store8(reinterpret_cast<bf*>(Fb + swz(P::FBOX, t, e)), o);
      }
    }
    cluster_arrive_relaxed();                  // this CTA's sums have landed and its `gath` is read
    tc::fence_proxy_async();
    __syncthreads();
    if (tid == 0) {
      tc::tma_store_3d(&mXi, su32(Fb), 0, (int)t0, j0 / 64);
      tc::bulk_commit();
    }
  }
  sinkhorn_pending();                          // the last block's
  if (tid == 0) tc::bulk_wait<0>();            // the last stores have landed
  cluster_wait();                              // no CTA leaves while a copy out of or into its shared memory may run
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
// spreads the work over more SMs).  A 64-token decode batch is four 16-token blocks:
// 32 CTAs each with one slice run faster than 64 CTAs each with a whole token
// (0.92 -> 0.62 ms of mHC per decode step at B = 64).
constexpr int kClusterMinTokens = 64;

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

// How many clusters of the kernel are resident at once on this device (cached per kernel,
// device and cluster size).
static cudaError_t resident_clusters(const void* kern, const cudaLaunchConfig_t& cfg, int CL, int& n) {
  static std::mutex mu;
  static std::map<std::tuple<const void*, int, int>, int> cache;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const auto key = std::make_tuple(kern, dev, CL);
  std::lock_guard<std::mutex> lock(mu);
  auto it = cache.find(key);
  if (it != cache.end()) {
    n = it->second;
    return cudaSuccess;
  }
  e = cudaOccupancyMaxActiveClusters(&n, kern, &cfg);
  if (e != cudaSuccess) return e;
  if (n < 1) return cudaErrorInvalidConfiguration;
  cache[key] = n;
  return cudaSuccess;
}

template <int TB, int NCH, int MODE>
static cudaError_t launch_cluster(const void* X_in, const void* F, const float* coeffs_in, const float* w_r,
                                  const float* b_r, void* X_out, void* x_in, float* coeffs_out, int N, int d, int CL,
                                  float eps, int iters, cudaStream_t s) {
  auto kern = mhc_cluster_kernel<TB, NCH, MODE>;
  const size_t bytes = MhcCl<TB, NCH>::BYTES;
  cudaError_t e = set_smem_limit(kern, (int)bytes);
  if (e != cudaSuccess) return e;
  // TMA maps with the 64-column chunk as the outermost dimension (stride 128 bytes), so one
  // box covers a CTA's whole slice of a token block: streams [N][2][d] as (64, 2, N, d/64)
  // with boxes (64, 2, TB, S/64), rows [N][d] as (64, N, d/64) with boxes (64, TB, S/64),
  // both 128-byte swizzled; coefficients [N][8] fp32 as (8, N) with boxes (8, TB).  Maps a
  // mode does not use still describe valid memory.
  constexpr int NB = MhcCl<TB, NCH>::S / 64;
  const auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const cuuint64_t dr[3] = {64, (cuuint64_t)N, (cuuint64_t)d / 64}, sr[2] = {(cuuint64_t)d * 2, 128};
  const cuuint64_t ds[4] = {64, 2, (cuuint64_t)N, (cuuint64_t)d / 64};
  const cuuint64_t ss[3] = {(cuuint64_t)d * 2, (cuuint64_t)d * 4, 128};
  const cuuint64_t dc[2] = {8, (cuuint64_t)N}, sc[1] = {32};
  const cuuint32_t br[3] = {64, TB, NB}, bs[4] = {64, 2, TB, NB}, bc[2] = {8, TB};
  CUtensorMap mX, mF, mXo, mXi, mC;
  const bool ok = (MODE == MHC_OPEN ? tc::make_map_nd(&mX, BF, 3, X_in, dr, sr, br, true)
                                    : tc::make_map_nd(&mX, BF, 4, X_in, ds, ss, bs, true)) &&
                  tc::make_map_nd(&mF, BF, 3, MODE == MHC_MIX ? F : x_in, dr, sr, br, true) &&
                  tc::make_map_nd(&mXo, BF, 4, MODE == MHC_ROUTE ? X_in : X_out, ds, ss, bs, true) &&
                  tc::make_map_nd(&mXi, BF, 3, x_in, dr, sr, br, true) &&
                  tc::make_map_nd(&mC, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2,
                                  MODE == MHC_MIX ? (const void*)coeffs_in : (const void*)coeffs_out, dc, sc, bc,
                                  false);
  if (!ok) return cudaErrorInvalidValue;
  const long n_blk = ((long)N + TB - 1) / TB;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)CL);
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
  int n_cl = 0;
  e = resident_clusters(reinterpret_cast<const void*>(kern), cfg, CL, n_cl);
  if (e != cudaSuccess) return e;
  cfg.gridDim = dim3((unsigned)(std::min((long)n_cl, n_blk) * CL));   // persistent: one wave of clusters
  return cudaLaunchKernelEx(&cfg, kern, mX, mF, mXo, mXi, mC, w_r, b_r, coeffs_out, N, d, CL, eps, iters);
}

template <int NCH>
static cudaError_t cluster_mode(int mode, const void* X_in, const void* F, const float* coeffs_in, const float* w_r,
                                const float* b_r, void* X_out, void* x_in, float* coeffs_out, int N, int d, int CL,
                                float eps, int iters, cudaStream_t s) {
  constexpr int TB = NCH >= 2 ? 16 : 32;       // two token-block buffers per CTA, two CTAs per SM for NCH <= 2
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
  const bool al16 = ((uintptr_t)X_in | (uintptr_t)F | (uintptr_t)X_out | (uintptr_t)x_in) % 16 == 0;
  if (dtype == BF16 && mode != MHC_MERGE && N >= kClusterMinTokens && al16 && cluster_shape(d, CL, nch)) {
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
