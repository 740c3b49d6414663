// Full-attention execution ("Loop-9B engineering teardown" §三): GQA 16 q / 4 KV heads,
// head dim 256, QK-norm, interleaved rotary on 0.25 of the head dims, sigmoid
// output gate; §四: each execution writes its own KV slab.
//
// fa_prep_kernel : QK-norm + rotary for q (to a compact buffer) and k (into the
//                  slab), v copied into the slab.  One warp per (token, head).
// attn_rows_kernel: softmax attention for a block of query rows of one KV group.
//                  One warp per (query row, q head); the Hq/Hkv heads of a group
//                  share each K/V row through L1.  Lanes split the head dim;
//                  scores of 8 keys are reduced together (reduce-scatter), so a
//                  key costs ~2 shuffles.  Keys may be split across CTAs
//                  (flash-decode); attn_combine_kernel merges the splits.
#include "common.cuh"
#include "internal.h"

namespace lk {

// ------------------------------------------------------------------ QK-norm + rotary + KV write
// cos/sin of pos * base^(-2j/rot) for positions pos0 .. pos0+T-1 and pairs j < rot/2,
// evaluated in fp64 (angles reach 1e5 rad at long context) and stored as fp32 pairs.
__global__ void rope_table_kernel(float2* __restrict__ tab, int T_len, int pos0, int rot, float base) {
  const long i = (long)blockIdx.x * blockDim.x + threadIdx.x;
  const int half = rot / 2;
  if (i >= (long)T_len * half) return;
  const int t = (int)(i / half), j = (int)(i % half);
  const double theta = pow((double)base, -2.0 * (double)j / (double)rot);
  double ang = (double)(pos0 + t) * theta;
  ang -= 6.283185307179586 * floor(ang / 6.283185307179586);
  double sn, cs;
  sincos(ang, &sn, &cs);
  tab[i] = make_float2((float)cs, (float)sn);
}

cudaError_t rope_table(float2* tab, int T, int pos0, int rot, float base, cudaStream_t s) {
  const long n = (long)T * (rot / 2);
  if (n == 0) return cudaSuccess;
  rope_table_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(tab, T, pos0, rot, base);
  return cudaGetLastError();
}

// One warp per R heads of one token (all query heads or all key heads: R divides Hq and
// Hkv), so R rows' loads are in flight together and the norm gain and the rotary table
// entries are read once for them.
template <typename T, int DH, bool VEC, int R>
__global__ void __launch_bounds__(256) fa_prep_kernel(const T* __restrict__ P, int ld_p, const T* __restrict__ q_norm,
                                                      const T* __restrict__ k_norm, T* __restrict__ q_out,
                                                      T* __restrict__ k_cache, T* __restrict__ v_cache, int kv_cap,
                                                      int T_len, int pos0, int Hq, int Hkv, int rot, float base,
                                                      float eps, const float2* __restrict__ tab) {
  constexpr int PER = DH / 32;         // contiguous elements per lane (even: rotary pairs stay local)
  const int lane = threadIdx.x & 31;
  const int hq = q_out ? Hq : 0;       // no q_out: keys and values only
  const int groups = (hq + Hkv) / R;
  const long w = (long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int b = blockIdx.y;
  if (w >= (long)T_len * groups) return;
  const int t = (int)(w / groups), hh0 = (int)(w % groups) * R + (Hq - hq);
  const long m = (long)b * T_len + t;
  const int pos = pos0 + t;
  const T* row = P + m * ld_p;
  const bool is_q = hh0 < Hq;
  const int kvh0 = hh0 - Hq;
  const T* src = is_q ? row + hh0 * DH : row + 2 * Hq * DH + kvh0 * DH;
  const T* gain = is_q ? q_norm : k_norm;
  // VEC: rows 16-byte aligned, so each lane moves its PER elements as 8-element vectors
  constexpr bool V8 = VEC && PER % 8 == 0;
  float x[R][PER], gn[PER];
  // key rows: their values' 16-byte pieces are loaded together with the keys (one round trip)
  constexpr int VP = V8 ? PER * (int)sizeof(T) / 16 : 1;
  uint4 vv[R][VP];
  const T* vsrc = row + 2 * Hq * DH + Hkv * DH + kvh0 * DH;
  if constexpr (V8) {
    if (!is_q) {
#pragma unroll
      for (int r = 0; r < R; ++r)
#pragma unroll
        for (int i = 0; i < VP; ++i)
          vv[r][i] = *reinterpret_cast<const uint4*>(vsrc + r * DH + lane * PER + i * (16 / (int)sizeof(T)));
    }
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int u = 0; u < PER; u += 8) load8(src + r * DH + lane * PER + u, x[r] + u);
#pragma unroll
    for (int u = 0; u < PER; u += 8) load8(gain + lane * PER + u, gn + u);
  } else {
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int u = 0; u < PER; ++u) x[r][u] = ldf(src + r * DH + lane * PER + u);
#pragma unroll
    for (int u = 0; u < PER; ++u) gn[u] = ldf(gain + lane * PER + u);
  }
  float inv[R];
#pragma unroll
  for (int r = 0; r < R; ++r) {
    float ss = 0.f;
#pragma unroll
    for (int u = 0; u < PER; ++u) ss += x[r][u] * x[r][u];
    inv[r] = ss;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1)
#pragma unroll
    for (int r = 0; r < R; ++r) inv[r] += __shfl_xor_sync(0xffffffffu, inv[r], o);
#pragma unroll
  for (int r = 0; r < R; ++r) {
    inv[r] = rsqrtf(inv[r] / (float)DH + eps);
#pragma unroll
    for (int u = 0; u < PER; ++u) x[r][u] = x[r][u] * inv[r] * gn[u];
  }
  // rotary on dims [0, rot): pair (2j, 2j+1), angle pos * base^(-2j/rot), evaluated in fp64
#pragma unroll
  for (int u = 0; u < PER; u += 2) {
    const int e = lane * PER + u;
    if (e < rot) {
      const int j = e >> 1;
      float c, s;
      if (tab) {
        const float2 cs2 = tab[(long)t * (rot / 2) + j];
        c = cs2.x;
        s = cs2.y;
      } else {
        const double theta = pow((double)base, -2.0 * (double)j / (double)rot);
        double ang = (double)pos * theta;
        ang -= 6.283185307179586 * floor(ang / 6.283185307179586);
        double sn, cs;
        sincos(ang, &sn, &cs);
        c = (float)cs;
        s = (float)sn;
      }
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const float a0 = x[r][u], a1 = x[r][u + 1];
        x[r][u] = a0 * c - a1 * s;
        x[r][u + 1] = a0 * s + a1 * c;
      }
    }
  }
#pragma unroll
  for (int r = 0; r < R; ++r) {
    T* dst;
    if (is_q) {
      dst = q_out + (m * Hq + hh0 + r) * DH;
    } else {
      const long slot = (((long)b * Hkv + kvh0 + r) * kv_cap + pos) * DH;
      dst = k_cache + slot;
      const T* vs = vsrc + r * DH;
      T* vd = v_cache + slot;
      if constexpr (V8) {
#pragma unroll
        for (int i = 0; i < VP; ++i)
          *reinterpret_cast<uint4*>(vd + lane * PER + i * (16 / (int)sizeof(T))) = vv[r][i];
      } else {
#pragma unroll
        for (int u = 0; u < PER; ++u) vd[lane * PER + u] = vs[lane * PER + u];
      }
    }
    if constexpr (V8) {
#pragma unroll
      for (int u = 0; u < PER; u += 8) store8(dst + lane * PER + u, x[r] + u);
    } else {
#pragma unroll
      for (int u = 0; u < PER; ++u) stf(dst + lane * PER + u, x[r][u]);
    }
  }
}

cudaError_t fa_prep(const void* P, int ld_p, const void* q_norm, const void* k_norm, void* q_out,
                    void* k_cache, void* v_cache, int kv_cap, int B, int T, int pos0, int Hq,
                    int Hkv, int dh, int rotary_dims, float rope_base, float eps, int dtype,
                    cudaStream_t s, const float2* rope_tab) {
  if (T == 0 || B == 0) return cudaSuccess;
  const int warps = 8;
  auto al16 = [](const void* p) { return ((uintptr_t)p % 16) == 0; };
  const int es = dtype == BF16 ? 2 : 4;
  const bool vec = al16(P) && al16(q_norm) && al16(k_norm) && al16(q_out) && al16(k_cache) && al16(v_cache) &&
                   ((long)ld_p * es) % 16 == 0;
  const int hq = q_out ? Hq : 0;                                // no q_out: keys and values only
  const int R = (vec && hq % 4 == 0 && Hkv % 4 == 0) ? 4 : 1;   // heads per warp
  dim3 grid((unsigned)(((long)T * ((hq + Hkv) / R) + warps - 1) / warps), B);
#define FA_PREP(TT, DHV)                                                                                   \
  do {                                                                                                     \
    if (R == 4) FA_PREP_V(TT, DHV, true, 4);                                                               \
    else if (vec) FA_PREP_V(TT, DHV, true, 1);                                                             \
    else FA_PREP_V(TT, DHV, false, 1);                                                                     \
  } while (0)
#define FA_PREP_V(TT, DHV, V, RR)                                                                          \
  fa_prep_kernel<TT, DHV, V, RR><<<grid, warps * 32, 0, s>>>((const TT*)P, ld_p, (const TT*)q_norm,            \
                                                      (const TT*)k_norm, (TT*)q_out, (TT*)k_cache,         \
                                                      (TT*)v_cache, kv_cap, T, pos0, Hq, Hkv, rotary_dims, \
                                                      rope_base, eps, rope_tab)
  if (dtype == BF16) {
    if (dh == 256) FA_PREP(__nv_bfloat16, 256); else if (dh == 128) FA_PREP(__nv_bfloat16, 128);
    else if (dh == 64) FA_PREP(__nv_bfloat16, 64); else return cudaErrorNotSupported;
  } else {
    if (dh == 256) FA_PREP(float, 256); else if (dh == 128) FA_PREP(float, 128);
    else if (dh == 64) FA_PREP(float, 64); else return cudaErrorNotSupported;
  }
#undef FA_PREP
#undef FA_PREP_V
  return cudaGetLastError();
}

// ------------------------------------------------------------------ attention over rows
// Reduce-scatter of 8 per-lane partial sums: afterwards lane L holds the full sum
// of value index (L >> 2) & 7.
__device__ __forceinline__ float reduce_scatter8(const float v[8], int lane) {
  float a[4], b2[2];
  const bool h4 = lane & 16, h3 = lane & 8, h2 = lane & 4;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float send = h4 ? v[i] : v[i + 4];
    float keep = h4 ? v[i + 4] : v[i];
    a[i] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
  }
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    float send = h3 ? a[i] : a[i + 2];
    float keep = h3 ? a[i + 2] : a[i];
    b2[i] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
  }
  float send = h2 ? b2[0] : b2[1];
  float s = (h2 ? b2[1] : b2[0]) + __shfl_xor_sync(0xffffffffu, send, 4);
  s += __shfl_xor_sync(0xffffffffu, s, 2);
  s += __shfl_xor_sync(0xffffffffu, s, 1);
  return s;
}

template <typename T, int DH>
__global__ void attn_rows_kernel(const T* __restrict__ q, int ld_q, const T* __restrict__ kc,
                                 const T* __restrict__ vc, int kv_cap, const T* __restrict__ gate,
                                 int ld_gate, T* __restrict__ out, float* __restrict__ ws, int Tq, int Tkv,
                                 int q_off, int Hq, int Hkv, int causal, int n_split, int split_len,
                                 float scale) {
  constexpr int PER = DH / 32;
  const int lane = threadIdx.x & 31, hw = threadIdx.x >> 5;    // warp = q head within the group
  const int rep = Hq / Hkv;
  const int t = blockIdx.x;
  const int kvh = blockIdx.y / n_split, split = blockIdx.y % n_split;
  const int b = blockIdx.z;
  const int h = kvh * rep + hw;
  const long m = (long)b * Tq + t;
  float qq[PER], o[PER];
  const T* qp = q + m * ld_q + (long)h * DH + lane * PER;
#pragma unroll
  for (int u = 0; u < PER; ++u) { qq[u] = ldf(qp + u) * scale; o[u] = 0.f; }
  int k_end = Tkv;
  if (causal) k_end = min(k_end, q_off + t + 1);
  const int k_begin = split * split_len;
  k_end = min(k_end, k_begin + split_len);
  const T* Kb = kc + ((long)b * Hkv + kvh) * kv_cap * DH + lane * PER;
  const T* Vb = vc + ((long)b * Hkv + kvh) * kv_cap * DH + lane * PER;
  float mx = -INFINITY, l = 0.f;
  for (int p0 = k_begin; p0 < k_end; p0 += 8) {
    float part[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      part[c] = 0.f;
      const int p = p0 + c;
      if (p < k_end) {
        const T* kr = Kb + (long)p * DH;
#pragma unroll
        for (int u = 0; u < PER; ++u) part[c] = fmaf(qq[u], ldf(kr + u), part[c]);
      }
    }
    const float mine = reduce_scatter8(part, lane);
    float s8[8];
    float tmax = -INFINITY;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      s8[c] = __shfl_sync(0xffffffffu, mine, c << 2);
      if (p0 + c >= k_end) s8[c] = -INFINITY;
      tmax = fmaxf(tmax, s8[c]);
    }
    const float mnew = fmaxf(mx, tmax);
    const float corr = expf(mx - mnew);     // mx = -inf on the first tile -> 0
    l *= corr;
#pragma unroll
    for (int u = 0; u < PER; ++u) o[u] *= corr;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const int p = p0 + c;
      if (p < k_end) {
        const float pc = expf(s8[c] - mnew);
        l += pc;
        const T* vr = Vb + (long)p * DH;
#pragma unroll
        for (int u = 0; u < PER; ++u) o[u] = fmaf(pc, ldf(vr + u), o[u]);
      }
    }
    mx = mnew;
  }
  if (n_split == 1) {
    const float inv = l > 0.f ? 1.f / l : 0.f;
    const T* gp = gate ? gate + m * ld_gate + (long)h * DH + lane * PER : nullptr;
    T* op = out + (m * Hq + h) * DH + lane * PER;
#pragma unroll
    for (int u = 0; u < PER; ++u) {
      float r = o[u] * inv;
      if (gp) r *= sigmoidf_acc(ldf(gp + u));
      stf(op + u, r);
    }
  } else {
    // partials: [m, h, split] -> (max, sum, o[DH])
    float* w = ws + ((m * Hq + h) * n_split + split) * (DH + 2);
    if (lane == 0) { w[0] = mx; w[1] = l; }
#pragma unroll
    for (int u = 0; u < PER; ++u) w[2 + lane * PER + u] = o[u];
  }
}

template <typename T, int DH>
__global__ void attn_combine_kernel(const float* __restrict__ ws, const T* __restrict__ gate, int ld_gate,
                                    T* __restrict__ out, long rows, int Hq, int n_split) {
  pdl_trigger();
  constexpr int PER = DH / 32;
  const int lane = threadIdx.x & 31;
  const long r = (long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);   // r = m * Hq + h
  if (r >= rows) return;
  const float* w = ws + r * n_split * (DH + 2);
  float M = -INFINITY;
  for (int s = 0; s < n_split; ++s) M = fmaxf(M, w[s * (DH + 2)]);
  float L = 0.f, o[PER];
#pragma unroll
  for (int u = 0; u < PER; ++u) o[u] = 0.f;
  for (int s = 0; s < n_split; ++s) {
    const float* ws_s = w + s * (DH + 2);
    const float f = ws_s[0] == -INFINITY ? 0.f : expf(ws_s[0] - M);
    L += f * ws_s[1];
#pragma unroll
    for (int u = 0; u < PER; ++u) o[u] = fmaf(f, ws_s[2 + lane * PER + u], o[u]);
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
  const long m = r / Hq;
  const int h = (int)(r % Hq);
  const T* gp = gate ? gate + m * ld_gate + (long)h * DH + lane * PER : nullptr;
  T* op = out + r * DH + lane * PER;
#pragma unroll
  for (int u = 0; u < PER; ++u) {
    float v = o[u] * inv;
    if (gp) v *= sigmoidf_acc(ldf(gp + u));
    stf(op + u, v);
  }
}

static int attn_splits(int B, int Tq, int Tkv, int Hkv) {
  const long blocks = (long)B * Tq * Hkv;
  int want = (int)((8L * 148 + blocks - 1) / blocks);
  int cap = (Tkv + 255) / 256;
  int s = want < cap ? want : cap;
  if (s > 32) s = 32;
  return s < 1 ? 1 : s;
}


// ------------------------------------------------------------------ single-token decode
// One CTA per (sequence, KV head, key split); warp w = q head w of the group, so every
// K/V tile is read from HBM once for the 4 heads that share it.  Tiles of 32 keys stream
// through a 3-stage cp.async ring.  Scores: lane = key (K rows padded by 16 B so the
// 32 lanes hit distinct banks); P.V: lanes over the head dim.
constexpr int DEC_KT = 32, DEC_STAGES = 3;

template <int DH>
struct DecSmem {
  static constexpr int KROW = DH * 2 + 16;            // padded K row (bytes)
  static constexpr int VROW = DH * 2;
  static constexpr int STAGE = DEC_KT * (KROW + VROW);
  static constexpr int Q = 4 * DH * 4;                // 4 heads, fp32
  static constexpr size_t BYTES = (size_t)DEC_STAGES * STAGE + Q;
};

__device__ __forceinline__ void cpa16(void* smem, const void* gmem, bool valid) {
  const uint32_t d = (uint32_t)__cvta_generic_to_shared(smem);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(gmem), "r"(valid ? 16 : 0) : "memory");
}

template <int DH>
__global__ void __launch_bounds__(128) attn_decode_kernel(const __nv_bfloat16* __restrict__ q, int ld_q,
                                                          const __nv_bfloat16* __restrict__ kc,
                                                          const __nv_bfloat16* __restrict__ vc, int kv_cap,
                                                          const __nv_bfloat16* __restrict__ gate, int ld_gate,
                                                          __nv_bfloat16* __restrict__ out, float* __restrict__ ws,
                                                          int Tkv, int q_off, int Hq, int Hkv, int causal,
                                                          int n_split, int split_len, float scale) {
  pdl_trigger();
  using L = DecSmem<DH>;
  constexpr int PER = DH / 32;                          // dims per lane in P.V
  constexpr int CH = DH / 8;                            // 16-byte chunks per row
  extern __shared__ __align__(16) uint8_t sm[];
  float* qs = (float*)(sm + DEC_STAGES * L::STAGE);     // [4][DH]
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int rep = Hq / Hkv;
  const int h = kvh * rep + w;
  const bool head_ok = w < rep;
  for (int i = threadIdx.x; i < 4 * DH; i += 128) {
    const int hh = i / DH, j = i % DH;
    qs[i] = hh < rep ? __bfloat162float(q[(long)b * ld_q + (long)(kvh * rep + hh) * DH + j]) * scale : 0.f;
  }
  int k_end = Tkv;
  if (causal) k_end = min(k_end, q_off + 1);
  const int k_begin = split * split_len;
  k_end = min(k_end, k_begin + split_len);
  const int n_tiles = k_end > k_begin ? (k_end - k_begin + DEC_KT - 1) / DEC_KT : 0;
  const __nv_bfloat16* Kb = kc + ((long)b * Hkv + kvh) * kv_cap * DH;
  const __nv_bfloat16* Vb = vc + ((long)b * Hkv + kvh) * kv_cap * DH;

  auto issue = [&](int t) {
    uint8_t* st = sm + (t % DEC_STAGES) * L::STAGE;
    const int key0 = k_begin + t * DEC_KT;
    for (int i = threadIdx.x; i < DEC_KT * CH; i += 128) {
      const int r = i / CH, c = i % CH;
      const int key = key0 + r;
      const bool ok = key < k_end;
      const long off = (long)(ok ? key : k_begin) * DH + c * 8;
      cpa16(st + r * L::KROW + c * 16, Kb + off, ok);
      cpa16(st + DEC_KT * L::KROW + r * L::VROW + c * 16, Vb + off, ok);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
#pragma unroll
  for (int t = 0; t < DEC_STAGES - 1; ++t) {
    if (t < n_tiles) issue(t);
    else asm volatile("cp.async.commit_group;" ::: "memory");
  }
  float mx = -INFINITY, l = 0.f, o[PER];
#pragma unroll
  for (int u = 0; u < PER; ++u) o[u] = 0.f;
  const float* qh = qs + w * DH;
  for (int t = 0; t < n_tiles; ++t) {
    asm volatile("cp.async.wait_group %0;" ::"n"(DEC_STAGES - 2) : "memory");
    __syncthreads();
    const uint8_t* st = sm + (t % DEC_STAGES) * L::STAGE;
    // scores: lane = key
    const uint8_t* krow = st + lane * L::KROW;
    float sc = 0.f;
#pragma unroll 8
    for (int c = 0; c < CH; ++c) {
      float kf[8];
      load8(reinterpret_cast<const __nv_bfloat16*>(krow + c * 16), kf);
      const float4 q0 = *reinterpret_cast<const float4*>(qh + c * 8);
      const float4 q1 = *reinterpret_cast<const float4*>(qh + c * 8 + 4);
      sc = fmaf(kf[0], q0.x, sc); sc = fmaf(kf[1], q0.y, sc); sc = fmaf(kf[2], q0.z, sc); sc = fmaf(kf[3], q0.w, sc);
      sc = fmaf(kf[4], q1.x, sc); sc = fmaf(kf[5], q1.y, sc); sc = fmaf(kf[6], q1.z, sc); sc = fmaf(kf[7], q1.w, sc);
    }
    const int key = k_begin + t * DEC_KT + lane;
    if (key >= k_end) sc = -INFINITY;
    const float mnew = fmaxf(mx, warp_max(sc));
    const float p = expf(sc - mnew);
    const float corr = expf(mx - mnew);
    l = l * corr + warp_sum(p);
    mx = mnew;
    // P.V: lanes over the head dim
    const uint8_t* vt = st + DEC_KT * L::KROW;
#pragma unroll
    for (int u = 0; u < PER; ++u) o[u] *= corr;
#pragma unroll 4
    for (int r = 0; r < DEC_KT; ++r) {
      const float pr = __shfl_sync(0xffffffffu, p, r);
      float vf[PER];
      const __nv_bfloat16* vrow = reinterpret_cast<const __nv_bfloat16*>(vt + r * L::VROW) + lane * PER;
      if (PER == 8) {
        load8(vrow, vf);
      } else {
#pragma unroll
        for (int u = 0; u < PER; ++u) vf[u] = __bfloat162float(vrow[u]);
      }
#pragma unroll
      for (int u = 0; u < PER; ++u) o[u] = fmaf(pr, vf[u], o[u]);
    }
    __syncthreads();
    if (t + DEC_STAGES - 1 < n_tiles) issue(t + DEC_STAGES - 1);
    else asm volatile("cp.async.commit_group;" ::: "memory");
  }
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  if (!head_ok) return;
  if (n_split == 1) {
    const float inv = l > 0.f ? 1.f / l : 0.f;
    const __nv_bfloat16* gp = gate ? gate + (long)b * ld_gate + (long)h * DH + lane * PER : nullptr;
    __nv_bfloat16* op = out + ((long)b * Hq + h) * DH + lane * PER;
#pragma unroll
    for (int u = 0; u < PER; ++u) {
      float r = o[u] * inv;
      if (gp) r *= sigmoidf_acc(__bfloat162float(gp[u]));
      op[u] = __float2bfloat16(r);
    }
  } else {
    float* wp = ws + (((long)b * Hq + h) * n_split + split) * (DH + 2);
    if (lane == 0) { wp[0] = mx; wp[1] = l; }
#pragma unroll
    for (int u = 0; u < PER; ++u) wp[2 + lane * PER + u] = o[u];
  }
}

template <int DH>
static cudaError_t launch_decode(const void* q, int ld_q, const void* k, const void* v, int kv_cap, const void* gate,
                                 int ld_gate, void* out, int B, int Tkv, int q_off, int Hq, int Hkv, int causal,
                                 void* workspace, cudaStream_t s) {
  using L = DecSmem<DH>;
  const int n_split = workspace ? attn_splits(B, 1, Tkv, Hkv) : 1;
  const int split_len = (((Tkv + n_split - 1) / n_split) + DEC_KT - 1) / DEC_KT * DEC_KT;
  {
    cudaError_t e = set_smem_limit(attn_decode_kernel<DH>,
                                         (int)L::BYTES);
    if (e != cudaSuccess) return e;
  }
  dim3 grid(n_split, Hkv, B);
  attn_decode_kernel<DH><<<grid, 128, L::BYTES, s>>>(
      (const __nv_bfloat16*)q, ld_q, (const __nv_bfloat16*)k, (const __nv_bfloat16*)v, kv_cap,
      (const __nv_bfloat16*)gate, ld_gate, (__nv_bfloat16*)out, (float*)workspace, Tkv, q_off, Hq, Hkv, causal,
      n_split, split_len, 1.f / sqrtf((float)DH));
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || n_split == 1) return e;
  const long rows = (long)B * Hq;
  attn_combine_kernel<__nv_bfloat16, DH><<<(unsigned)((rows + 7) / 8), 256, 0, s>>>(
      (const float*)workspace, (const __nv_bfloat16*)gate, ld_gate, (__nv_bfloat16*)out, rows, Hq, n_split);
  return cudaGetLastError();
}


// ------------------------------------------------------------------ single-token decode on tensor cores
// The same flash-decode with the products on mma.sync (m16n8k16, bf16 -> fp32): the
// q heads of one KV group are the rows of a 16-row A tile (rows >= Hq/Hkv are zero).
// Per 64-key tile: warp w computes S for keys [16w, 16w+16) (Q fragments stay in
// registers), the tile's row max and sum are combined through shared memory, then warp
// w accumulates O for head dims [w*DH/4, (w+1)*DH/4) with P from shared memory.
constexpr int DTC_KT = 64, DTC_STAGES = 3;

template <int DH>
struct DecTc {
  static constexpr int ROW = DH * 2 + 16;                   // padded K / V row (bytes)
  static constexpr int STAGE = 2 * DTC_KT * ROW;
  static constexpr int QROW = DH * 2 + 16;
  static constexpr int PROW = DTC_KT * 2 + 16;
  static constexpr size_t BYTES = (size_t)DTC_STAGES * STAGE + 16 * QROW + 16 * PROW + 2 * 4 * 16 * 4;
};

__device__ __forceinline__ uint32_t sa32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }
__device__ __forceinline__ void lds_x4(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(sa32(p)));
}
__device__ __forceinline__ void lds_x4_t(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(sa32(p)));
}
__device__ __forceinline__ void hmma(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

template <int DH>
__global__ void __launch_bounds__(128) attn_decode_tc_kernel(const __nv_bfloat16* __restrict__ q, int ld_q,
                                                             const __nv_bfloat16* __restrict__ kc,
                                                             const __nv_bfloat16* __restrict__ vc, int kv_cap,
                                                             const __nv_bfloat16* __restrict__ gate, int ld_gate,
                                                             __nv_bfloat16* __restrict__ out, float* __restrict__ ws,
                                                             int Tkv, int q_off, int Hq, int Hkv, int causal,
                                                             int n_split, int split_len, float scale_log2) {
  pdl_trigger();
  using L = DecTc<DH>;
  constexpr int CH = DH / 8;                                 // 16-byte chunks per K/V row
  constexpr int WD = DH / 4;                                 // head dims per warp in P.V
  constexpr int NTO = WD / 8;                                // 8-wide output tiles per warp
  extern __shared__ __align__(16) uint8_t sm[];
  uint8_t* sQ = sm + DTC_STAGES * L::STAGE;                  // [16][QROW] bf16
  uint8_t* sP = sQ + 16 * L::QROW;                           // [16][PROW] bf16
  float* sMax = (float*)(sP + 16 * L::PROW);                 // [4 warps][16 rows]
  float* sSum = sMax + 4 * 16;
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5, gq = lane >> 2, tq = lane & 3;
  const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int rep = Hq / Hkv;
  for (int i = tid; i < 16 * CH; i += 128) {
    const int r = i / CH, c = i % CH;
    uint4 val = make_uint4(0, 0, 0, 0);
    if (r < rep) val = *reinterpret_cast<const uint4*>(q + (long)b * ld_q + (long)(kvh * rep + r) * DH + c * 8);
    *reinterpret_cast<uint4*>(sQ + r * L::QROW + c * 16) = val;
  }
  int k_end = Tkv;
  if (causal) k_end = min(k_end, q_off + 1);
  const int k_begin = split * split_len;
  k_end = min(k_end, k_begin + split_len);
  const int n_tiles = k_end > k_begin ? (k_end - k_begin + DTC_KT - 1) / DTC_KT : 0;
  const __nv_bfloat16* Kb = kc + ((long)b * Hkv + kvh) * kv_cap * DH;
  const __nv_bfloat16* Vb = vc + ((long)b * Hkv + kvh) * kv_cap * DH;
  auto issue = [&](int t) {
    uint8_t* st = sm + (t % DTC_STAGES) * L::STAGE;
    const int key0 = k_begin + t * DTC_KT;
    for (int i = tid; i < DTC_KT * CH; i += 128) {
      const int r = i / CH, c = i % CH;
      const int key = key0 + r;
      const bool ok = key < k_end;
      const long off = (long)(ok ? key : k_begin) * DH + c * 8;
      cpa16(st + r * L::ROW + c * 16, Kb + off, ok);
      cpa16(st + DTC_KT * L::ROW + r * L::ROW + c * 16, Vb + off, ok);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
#pragma unroll
  for (int t = 0; t < DTC_STAGES - 1; ++t) {
    if (t < n_tiles) issue(t);
    else asm volatile("cp.async.commit_group;" ::: "memory");
  }
  __syncthreads();
  uint32_t qa[DH / 16][4];                                   // Q fragments for every 16-dim step
#pragma unroll
  for (int ks = 0; ks < DH / 16; ++ks) lds_x4(qa[ks], sQ + (lane & 15) * L::QROW + (ks * 16 + (lane >> 4) * 8) * 2);
  float o[NTO][4];
#pragma unroll
  for (int j = 0; j < NTO; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
  float m_run = -INFINITY, l_run = 0.f;                      // row gq (rows gq+8 are padding)
  for (int t = 0; t < n_tiles; ++t) {
    asm volatile("cp.async.wait_group %0;" ::"n"(DTC_STAGES - 2) : "memory");
    __syncthreads();
    const uint8_t* st = sm + (t % DTC_STAGES) * L::STAGE;
    const uint8_t* vt = st + DTC_KT * L::ROW;
    // S for keys [16w, 16w + 16): two 8-key tiles
    float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
    for (int ks = 0; ks < DH / 16; ks += 2) {
      uint32_t kb0[4], kb1[4];
      // keys 16w + (lane & 7) (+8 for the second tile), dims ks*16 .. ks*16 + 32
      lds_x4(kb0, st + (w * 16 + (lane & 7)) * L::ROW + (ks * 16 + (lane >> 3) * 8) * 2);
      lds_x4(kb1, st + (w * 16 + 8 + (lane & 7)) * L::ROW + (ks * 16 + (lane >> 3) * 8) * 2);
      hmma(sc[0], qa[ks], kb0[0], kb0[1]);
      hmma(sc[1], qa[ks], kb1[0], kb1[1]);
      hmma(sc[0], qa[ks + 1], kb0[2], kb0[3]);
      hmma(sc[1], qa[ks + 1], kb1[2], kb1[3]);
    }
    const int kbase = k_begin + t * DTC_KT + w * 16 + 2 * tq;
    float mx = -INFINITY;
#pragma unroll
    for (int j = 0; j < 2; ++j)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int key = kbase + j * 8 + e;
        sc[j][e] = key < k_end ? sc[j][e] * scale_log2 : -INFINITY;
        mx = fmaxf(mx, sc[j][e]);
      }
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    if (tq == 0) sMax[w * 16 + gq] = mx;
    __syncthreads();
    const float tmax = fmaxf(fmaxf(sMax[gq], sMax[16 + gq]), fmaxf(sMax[32 + gq], sMax[48 + gq]));
    const float m_new = fmaxf(m_run, tmax);
    const float corr = exp2f(m_run - m_new);
    float ps = 0.f;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const float p0 = exp2f(sc[j][0] - m_new), p1 = exp2f(sc[j][1] - m_new);
      const __nv_bfloat162 pb = __floats2bfloat162_rn(p0, p1);
      const float2 pf = __bfloat1622float2(pb);
      ps += pf.x + pf.y;
      *reinterpret_cast<__nv_bfloat162*>(sP + gq * L::PROW + (w * 16 + j * 8 + 2 * tq) * 2) = pb;
      *reinterpret_cast<__nv_bfloat162*>(sP + (gq + 8) * L::PROW + (w * 16 + j * 8 + 2 * tq) * 2) =
          __floats2bfloat162_rn(0.f, 0.f);
    }
    ps += __shfl_xor_sync(0xffffffffu, ps, 1);
    ps += __shfl_xor_sync(0xffffffffu, ps, 2);
    if (tq == 0) sSum[w * 16 + gq] = ps;
    __syncthreads();
    l_run = l_run * corr + (sSum[gq] + sSum[16 + gq] + sSum[32 + gq] + sSum[48 + gq]);
    m_run = m_new;
#pragma unroll
    for (int j = 0; j < NTO; ++j) {
      o[j][0] *= corr;
      o[j][1] *= corr;
    }
    // O[:, w*WD .. +WD) += P V
#pragma unroll
    for (int ks = 0; ks < DTC_KT / 16; ++ks) {
      uint32_t pa[4];
      lds_x4(pa, sP + (lane & 15) * L::PROW + (ks * 16 + (lane >> 4) * 8) * 2);
#pragma unroll
      for (int j = 0; j < NTO; j += 2) {
        uint32_t vb[4];
        // rows ks*16 + (lane & 15) of V, dims w*WD + j*8 (+8 for lanes 16..31)
        lds_x4_t(vb, vt + (ks * 16 + (lane & 15)) * L::ROW + (w * WD + j * 8 + (lane >> 4) * 8) * 2);
        hmma(o[j], pa, vb[0], vb[1]);
        hmma(o[j + 1], pa, vb[2], vb[3]);
      }
    }
    __syncthreads();
    if (t + DTC_STAGES - 1 < n_tiles) issue(t + DTC_STAGES - 1);
    else asm volatile("cp.async.commit_group;" ::: "memory");
  }
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  if (gq >= rep) return;
  const int h = kvh * rep + gq;
  if (n_split == 1) {
    const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
#pragma unroll
    for (int j = 0; j < NTO; ++j) {
      const int dcol = w * WD + j * 8 + 2 * tq;
      float v0 = o[j][0] * inv, v1 = o[j][1] * inv;
      if (gate) {
        const __nv_bfloat16* gp = gate + (long)b * ld_gate + (long)h * DH + dcol;
        v0 *= sigmoidf_acc(__bfloat162float(gp[0]));
        v1 *= sigmoidf_acc(__bfloat162float(gp[1]));
      }
      *reinterpret_cast<__nv_bfloat162*>(out + ((long)b * Hq + h) * DH + dcol) = __floats2bfloat162_rn(v0, v1);
    }
  } else {
    // partials in the split-K layout: (max in natural-log units, sum, o[DH])
    float* wp = ws + (((long)b * Hq + h) * n_split + split) * (DH + 2);
    if (w == 0 && tq == 0) {
      wp[0] = m_run / 1.4426950408889634f;
      wp[1] = l_run;
    }
#pragma unroll
    for (int j = 0; j < NTO; ++j) {
      const int dcol = w * WD + j * 8 + 2 * tq;
      wp[2 + dcol] = o[j][0];
      wp[3 + dcol] = o[j][1];
    }
  }
}

template <int DH>
static cudaError_t launch_decode_tc(const void* q, int ld_q, const void* k, const void* v, int kv_cap,
                                   const void* gate, int ld_gate, void* out, int B, int Tkv, int q_off, int Hq, int Hkv,
                                   int causal, void* workspace, cudaStream_t s) {
  using L = DecTc<DH>;
  const int n_split = workspace ? attn_splits(B, 1, Tkv, Hkv) : 1;
  const int split_len = (((Tkv + n_split - 1) / n_split) + DTC_KT - 1) / DTC_KT * DTC_KT;
  {
    cudaError_t e = set_smem_limit(attn_decode_tc_kernel<DH>,
                                         (int)L::BYTES);
    if (e != cudaSuccess) return e;
  }
  dim3 grid(n_split, Hkv, B);
  attn_decode_tc_kernel<DH><<<grid, 128, L::BYTES, s>>>(
      (const __nv_bfloat16*)q, ld_q, (const __nv_bfloat16*)k, (const __nv_bfloat16*)v, kv_cap,
      (const __nv_bfloat16*)gate, ld_gate, (__nv_bfloat16*)out, (float*)workspace, Tkv, q_off, Hq, Hkv, causal,
      n_split, split_len, 1.4426950408889634f / sqrtf((float)DH));
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || n_split == 1) return e;
  const long rows = (long)B * Hq;
  attn_combine_kernel<__nv_bfloat16, DH><<<(unsigned)((rows + 7) / 8), 256, 0, s>>>(
      (const float*)workspace, (const __nv_bfloat16*)gate, ld_gate, (__nv_bfloat16*)out, rows, Hq, n_split);
  return cudaGetLastError();
}

size_t gqa_workspace_bytes(int B, int Tq, int Tkv, int Hq, int dh) {
  const int Hkv = 1;   // upper bound: splits computed with Hkv = 1 are never fewer
  const int s = attn_splits(B, Tq, Tkv, Hkv);
  return (size_t)B * Tq * Hq * s * (dh + 2) * sizeof(float);
}

// Which kernel a call runs, from its shape alone:
//   ATT_TC      multi-token queries, bf16, head dim 256, 128 % (Hq/Hkv) == 0: attn_tc.cu
//   ATT_DEC_TC  one query token, bf16, head dim 128/256, <= 16 q heads per KV head: tensor-core flash-decode
//   ATT_DEC     one query token, bf16, head dim 64, <= 4 q heads per KV head: flash-decode
//   ATT_ROWS    everything else (fp32 models; bf16 prefill segments of 2..15 tokens, head dims without
//               a tiled kernel): one warp per query row
enum AttnPath { ATT_TC, ATT_DEC_TC, ATT_DEC, ATT_ROWS };

static AttnPath attn_path(int Tq, int dtype, int dh, int Hq, int Hkv) {
  const int rep = Hq / Hkv;
  if (dtype == BF16 && Tq >= 16 && dh == 256 && 128 % rep == 0) return ATT_TC;   // 128 MMA rows = rep heads x positions
  if (dtype == BF16 && Tq == 1 && (dh == 256 || dh == 128) && rep <= 16) return ATT_DEC_TC;
  if (dtype == BF16 && Tq == 1 && dh == 64 && rep <= 4) return ATT_DEC;
  return ATT_ROWS;
}

// Key splits (> 1 means a second, combining launch and scratch partials) of a call given a workspace.
static int attn_path_splits(AttnPath p, int B, int Tq, int Tkv, int Hkv) {
  if (p == ATT_TC) return 1;
  return attn_splits(B, p == ATT_ROWS ? Tq : 1, Tkv, Hkv);
}

size_t gqa_scratch_bytes(int B, int Tq, int Tkv, int Hq, int Hkv, int dh, int dtype) {
  if (B <= 0 || Tq <= 0 || Tkv <= 0) return 0;
  const int n = attn_path_splits(attn_path(Tq, dtype, dh, Hq, Hkv), B, Tq, Tkv, Hkv);
  return n > 1 ? (size_t)B * Tq * Hq * n * (dh + 2) * sizeof(float) : 0;
}

int gqa_launches(int B, int Tq, int Tkv, int Hq, int Hkv, int dh, int dtype, bool has_workspace) {
  const AttnPath p = attn_path(Tq, dtype, dh, Hq, Hkv);
  return has_workspace && attn_path_splits(p, B, Tq, Tkv, Hkv) > 1 ? 2 : 1;
}

bool gqa_supported(int dh, int Hq, int Hkv) {
  return (dh == 64 || dh == 128 || dh == 256) && Hkv > 0 && Hq % Hkv == 0 && Hq / Hkv <= 32;
}

template <typename T, int DH>
static cudaError_t launch_attn(const void* q, int ld_q, const void* k, const void* v, int kv_cap,
                               const void* gate, int ld_gate, void* out, int B, int Tq, int Tkv, int q_off,
                               int Hq, int Hkv, int causal, void* workspace, cudaStream_t s) {
  int n_split = workspace ? attn_splits(B, Tq, Tkv, Hkv) : 1;
  const int split_len = (Tkv + n_split - 1) / n_split;
  dim3 grid(Tq, Hkv * n_split, B);
  const int threads = 32 * (Hq / Hkv);
  const float scale = 1.f / sqrtf((float)DH);
  attn_rows_kernel<T, DH><<<grid, threads, 0, s>>>((const T*)q, ld_q, (const T*)k, (const T*)v, kv_cap,
                                                   (const T*)gate, ld_gate, (T*)out, (float*)workspace, Tq,
                                                   Tkv, q_off, Hq, Hkv, causal, n_split, split_len, scale);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || n_split == 1) return e;
  const long rows = (long)B * Tq * Hq;
  attn_combine_kernel<T, DH><<<(unsigned)((rows + 7) / 8), 256, 0, s>>>((const float*)workspace, (const T*)gate,
                                                                         ld_gate, (T*)out, rows, Hq, n_split);
  return cudaGetLastError();
}

cudaError_t gqa_attn(const void* q, int ld_q, const void* k, const void* v, int kv_cap,
                     const void* gate, int ld_gate, void* out, int B, int Tq, int Tkv, int q_off,
                     int Hq, int Hkv, int dh, int causal, void* workspace, int dtype,
                     cudaStream_t s, const QNorm* qn) {
  if (B == 0 || Tq == 0) return cudaSuccess;
  auto al16 = [](const void* p) { return ((uintptr_t)p % 16) == 0; };
  const AttnPath path = attn_path(Tq, dtype, dh, Hq, Hkv);
  // raw queries (normalised and rotated while staged) only on the tensor-core kernel
  if (qn) {
    if (path != ATT_TC || !al16(qn->gain)) return cudaErrorNotSupported;
    if (Tkv == 0) return cudaSuccess;
    if (!gqa_tc_supported(dh, dtype, q, ld_q, gate, ld_gate, k, v, kv_cap)) return cudaErrorNotSupported;
    return gqa_attn_tc(q, ld_q, k, v, kv_cap, gate, ld_gate, out, B, Tq, Tkv, q_off, Hq, Hkv, causal, s, qn);
  }
  // The tiled kernels move 16-byte pieces (TMA boxes, cp.async); a call whose shape selects one of
  // them but whose buffers are not 16-byte aligned is refused rather than run on a slower kernel.
  if (path == ATT_TC) {
    if (Tkv == 0) return cudaSuccess;
    if (!gqa_tc_supported(dh, dtype, q, ld_q, gate, ld_gate, k, v, kv_cap)) return cudaErrorNotSupported;
    return gqa_attn_tc(q, ld_q, k, v, kv_cap, gate, ld_gate, out, B, Tq, Tkv, q_off, Hq, Hkv, causal, s);
  }
  if (path == ATT_DEC_TC) {
    if (!(al16(k) && al16(v) && al16(q) && ld_q % 8 == 0)) return cudaErrorNotSupported;
    if (dh == 256)
      return launch_decode_tc<256>(q, ld_q, k, v, kv_cap, gate, ld_gate, out, B, Tkv, q_off, Hq, Hkv, causal, workspace, s);
    return launch_decode_tc<128>(q, ld_q, k, v, kv_cap, gate, ld_gate, out, B, Tkv, q_off, Hq, Hkv, causal, workspace, s);
  }
  if (path == ATT_DEC) {
    if (!(al16(k) && al16(v))) return cudaErrorNotSupported;
    return launch_decode<64>(q, ld_q, k, v, kv_cap, gate, ld_gate, out, B, Tkv, q_off, Hq, Hkv, causal, workspace, s);
  }
#define ATTN(TT, DHV) \
  return launch_attn<TT, DHV>(q, ld_q, k, v, kv_cap, gate, ld_gate, out, B, Tq, Tkv, q_off, Hq, Hkv, causal, workspace, s)
  if (dtype == BF16) {
    if (dh == 256) ATTN(__nv_bfloat16, 256);
    if (dh == 128) ATTN(__nv_bfloat16, 128);
    if (dh == 64) ATTN(__nv_bfloat16, 64);
  } else {
    if (dh == 256) ATTN(float, 256);
    if (dh == 128) ATTN(float, 128);
    if (dh == 64) ATTN(float, 64);
  }
#undef ATTN
  return cudaErrorNotSupported;
}

}  // namespace lk
