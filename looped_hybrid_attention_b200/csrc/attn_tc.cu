// Causal GQA flash attention on the 5th-generation tensor cores, head dim 256, bf16
// ("Loop-9B engineering teardown" §三: GQA 16 q / 4 KV heads, head dim 256, output gate).
//
// One CTA = 128 MMA rows = the Hq/Hkv q heads of one KV group x 128/(Hq/Hkv) query
// positions (row r: head r / QT, position q0 + r % QT), so every K/V tile loaded serves
// all heads that share it.  Key tiles are 128 wide, so S = Q K^T runs as M128 x N128
// MMAs (the tensor pipe's cost per MMA instruction is fixed, and at N64 it dominated).
// Warps:
//   0     TMA: K and V stream through one ring of 16 KiB slots in the order the MMAs use
//         them (K_0, then K_{j+1}, V_j for j = 0, 1, ...): a K slot is a 64-dim quarter of
//         a 128-key tile, a V slot 32 keys x 256 dims.  3-D maps over the per-execution
//         slab, so keys past Tkv read as zeros;
//   1     MMA: S_j = Q K_j^T (M 128, N 128, K 256; Q and K from shared memory) into one of
//         two 128-column TMEM buffers, and O += P_j V_j (M 128, N 256, K 128) into TMEM,
//         with P_j read from TMEM as the A operand and V an MN-major shared-memory operand;
//   2..9  softmax in two warpgroups, two threads per query row (TMEM lane = row): each
//         takes 64 of the tile's keys, the two exchange their half-row maxima through
//         shared memory (one mbarrier round per tile, which also tells each that the
//         other has finished reading S), then write bf16 P, two keys per column, over
//         the first 64 columns of S_j's own buffer.  O is rescaled in TMEM only when
//         the running max grows by more than 2^8 (the stale max cancels in the final
//         O / l); finally O / l * sigmoid(gate) is stored.  Each thread first writes
//         its half of its row of Q into shared memory (128-byte swizzled quarters).
//         With a query-norm gain the rows are read raw from the input projection and
//         normalised and rotated on the way ("Loop-9B engineering teardown" §三: QK
//         normalisation, then interleaved rotary on the first dims): the two threads of a
//         row add their halves' sums of squares, scale by rsqrt(mean + eps) and the gain,
//         and rotate the pairs (2j, 2j+1) of dims [0, rot) by the position's angle.
// Q K^T of tile j+1 overlaps the softmax of tile j.  The tensor pipe runs its MMAs in
// issue order (Q K^T j+1, P V j, Q K^T j+2, ...), so P V j has read P_j before
// Q K^T j+2 overwrites that buffer: no barrier is needed for the reuse.  TMEM: the two
// S buffers and O fill all 512 columns.  All waits are bounded.
#include "internal.h"
#include "tc_common.cuh"

namespace lk {
namespace tc {

constexpr int AT_M = 128, AT_N = 128, AT_D = 256;
constexpr int Q_BYTES = AT_M * AT_D * 2;            // 64 KiB: four [128 rows][64 dims] quarters
constexpr int SLOT = 16384;                         // K quarter [128 keys][64 dims] or V [4][32 keys][64 dims]
constexpr int N_SLOTS = 9;
constexpr int XCH_BYTES = 2 * AT_M * 4 + 4 * AT_M * 4;   // row sums [2][128]; half-row maxima [2][2][128]
// query staging with QK-norm and rotary: the norm gain [256] bf16, and the cos/sin rows of
// the CTA's query positions ([QT <= 32][RT_MAX + 1] float2: one pad entry per row keeps the
// rows' same entries in different banks) when rot <= 2 * RT_MAX
constexpr int RT_MAX = 32, STAB_ROWS = 32;
constexpr int GAIN_BYTES = AT_D * 2, STAB_BYTES = STAB_ROWS * (RT_MAX + 1) * 8;
constexpr int AT_SMEM = Q_BYTES + N_SLOTS * SLOT + 1024 + 256 + XCH_BYTES + GAIN_BYTES + STAB_BYTES;
constexpr int AT_THREADS = 320;                  // TMA, MMA, two softmax warpgroups
// mbarrier slots
constexpr int B_Q = 0, B_F = 1, B_E = B_F + N_SLOTS, B_SF = B_E + N_SLOTS, B_PF = B_SF + 2, B_PV = B_PF + 2,
              B_X = B_PV + 2, B_L = B_X + 2, N_BARS = B_L + 1;
static_assert(N_BARS * 8 + 8 <= 256, "barrier region");
static_assert(AT_SMEM <= 232448, "shared memory per CTA");
// TMEM columns: S buffers 0..127 and 128..255 (P over the first 64 of each), O 256..511
constexpr uint32_t T_O = 256;
constexpr float RESCALE_THRESHOLD = 8.0f;        // log2 units

// 2^x as one MUFU op (x <= 0 here after the row-max shift; denormal results flush to 0).
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 8 bf16 (one 16-byte piece) -> 8 floats.
__device__ __forceinline__ void unpack8_bf16(const uint4& u, float* f) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 t = __bfloat1622float2(h[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}

// Two fp32 FMAs / adds as one packed instruction (each lane rounds exactly as fmaf / +).
__device__ __forceinline__ void fma_x2(float& d0, float& d1, float a0, float a1, float b0, float b1, float c0,
                                       float c1) {
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1), "f"(c0), "f"(c1));
}
__device__ __forceinline__ void add_x2(float& d0, float& d1, float a0, float a1, float b0, float b1) {
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

__global__ void __launch_bounds__(AT_THREADS, 1)
    attn_tc_kernel(const __nv_bfloat16* __restrict__ q, int ld_q, const __grid_constant__ CUtensorMap tK,
                   const __grid_constant__ CUtensorMap tV, const __nv_bfloat16* __restrict__ gate, int ld_gate,
                   __nv_bfloat16* __restrict__ out, int Tq, int Tkv, int q_off, int Hq, int Hkv, int causal,
                   float scale_log2, int QT, const __nv_bfloat16* __restrict__ q_norm, float eps, int rot,
                   float rope_base, const float2* __restrict__ rope_tab, int tab_pos0) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sQ = smem;                                 // Q quarters: dims [64c, 64c + 64) at c * Q_BYTES / 4
  uint8_t* sR = sQ + Q_BYTES;                         // K/V ring: slot i at i * SLOT
  uint64_t* bars = (uint64_t*)(sR + N_SLOTS * SLOT);
  uint32_t* tmem_slot = (uint32_t*)(bars + N_BARS);
  float* xsum = (float*)((uint8_t*)bars + 256);        // row-sum exchange [2 halves][AT_M]
  float* xmax = xsum + 2 * AT_M;                       // half-row maxima [tile parity][half][AT_M]
  uint4* sgain = reinterpret_cast<uint4*>(xmax + 4 * AT_M);   // query norm gain (fused query staging)
  float2* stab = reinterpret_cast<float2*>(sgain + AT_D / 8);  // cos/sin rows of the CTA's positions
  volatile int* abort_flag = (volatile int*)(tmem_slot + 1);
  const uint32_t bar0 = smem_u32(bars);
  const uint32_t q_full = bar0 + 8u * B_Q;
  auto full_bar = [&](int i) { return bar0 + 8u * (B_F + i); };
  auto empty_bar = [&](int i) { return bar0 + 8u * (B_E + i); };
  auto s_full = [&](int b) { return bar0 + 8u * (B_SF + b); };
  // one p_full / pv_done per S buffer, so no barrier runs two phases ahead of its waiter
  auto p_full = [&](int s) { return bar0 + 8u * (B_PF + s); };
  auto pv_done = [&](int s) { return bar0 + 8u * (B_PV + s); };
  auto x_bar = [&](int s) { return bar0 + 8u * (B_X + s); };     // both halves' maxima written (tile parity s)
  const uint32_t l_bar = bar0 + 8u * B_L;                         // row-sum exchange

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_qt = gridDim.x;
  const int qt = n_qt - 1 - blockIdx.x;               // longest causal rows first
  const int kvh = blockIdx.y, b = blockIdx.z;
  const int rep = Hq / Hkv;
  const int q0 = qt * QT;
  int k_end = Tkv;
  if (causal) k_end = min(k_end, q_off + q0 + QT);
  const int n_kv = (k_end + AT_N - 1) / AT_N;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 256);                           // the softmax threads' halves of the Q rows
    for (int i = 0; i < N_SLOTS; ++i) {
      mbar_init(full_bar(i), 1);
      mbar_init(empty_bar(i), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(s_full(s), 1);
      mbar_init(p_full(s), 256);
      mbar_init(x_bar(s), 256);
      mbar_init(pv_done(s), 1);
    }
    mbar_init(l_bar, 256);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) tmem_alloc(smem_u32(tmem_slot), 512);
  if (warp == 0 && lane == 0) {
    asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&tK) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&tV) : "memory");
  }
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tO = tmem + T_O;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int cnt = 0;                                    // ring slots filled so far
      auto slot_begin = [&](uint32_t& dst, uint32_t& fb) -> bool {
        const int i = cnt % N_SLOTS;
        if (!mbar_wait(empty_bar(i), (uint32_t)(((cnt / N_SLOTS) & 1) ^ 1), abort_flag)) return false;
        dst = smem_u32(sR + i * SLOT);
        fb = full_bar(i);
        mbar_expect_tx(fb, SLOT);
        ++cnt;
        return true;
      };
      auto load_k = [&](int j) -> bool {
        for (int c = 0; c < 4; ++c) {                 // dims [64c, 64c + 64) of keys [128j, 128j + 128)
          uint32_t dst, fb;
          if (!slot_begin(dst, fb)) return false;
          tma_load_3d(dst, &tK, fb, c * 64, j * AT_N, b * Hkv + kvh);
        }
        return true;
      };
      auto load_v = [&](int j) -> bool {
        for (int p = 0; p < 4; ++p) {                 // keys [128j + 32p, +32), all dims
          uint32_t dst, fb;
          if (!slot_begin(dst, fb)) return false;
#pragma unroll
          for (int c = 0; c < 4; ++c) tma_load_3d(dst + c * 4096, &tV, fb, c * 64, j * AT_N + p * 32, b * Hkv + kvh);
        }
        return true;
      };
      if (n_kv > 0 && !load_k(0)) goto done;
      for (int j = 0; j < n_kv; ++j) {
        if (j + 1 < n_kv && !load_k(j + 1)) goto done;
        if (!load_v(j)) goto done;
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t id_qk = idesc_bf16(AT_M, AT_N);
      constexpr uint32_t id_pv = idesc_bf16(AT_M, AT_D, 1);
      if (!mbar_wait(q_full, 0, abort_flag)) goto done;
      fence_after();
      const uint32_t qa = smem_u32(sQ);
      int cnt = 0;                                    // ring slots consumed so far (same order as filled)
      auto slot_wait = [&](uint32_t& a) -> bool {
        const int i = cnt % N_SLOTS;
        if (!mbar_wait(full_bar(i), (uint32_t)((cnt / N_SLOTS) & 1), abort_flag)) return false;
        fence_after();
        a = smem_u32(sR + i * SLOT);
        return true;
      };
      auto slot_release = [&]() {
        mma_commit(empty_bar(cnt % N_SLOTS));         // free once the MMAs issued so far have read it
        ++cnt;
      };
      auto issue_qk = [&](int j) -> bool {
        const uint32_t d = tmem + (uint32_t)((j & 1) * AT_N);
        for (int c = 0; c < 4; ++c) {
          uint32_t ka;
          if (!slot_wait(ka)) return false;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)              // 16-dim steps inside the 128-byte swizzled rows
            mma_bf16(d, sw128_desc(qa + c * (Q_BYTES / 4) + kk * 32), sw128_desc(ka + kk * 32), id_qk,
                     (c | kk) ? 1u : 0u);
          slot_release();
        }
        mma_commit(s_full(j & 1));
        return true;
      };
      auto issue_pv = [&](int j) -> bool {
        if (!mbar_wait(p_full(j & 1), (uint32_t)((j >> 1) & 1), abort_flag)) return false;
        fence_after();
        const uint32_t pa = tmem + (uint32_t)((j & 1) * AT_N);     // P_j: bf16 pairs over 64 columns
        for (int p = 0; p < 4; ++p) {
          uint32_t va;
          if (!slot_wait(va)) return false;
#pragma unroll
          for (int kk = 0; kk < 2; ++kk)              // 16-key steps; V dim blocks 4 KiB apart
            mma_bf16_ts(tO, pa + (uint32_t)((2 * p + kk) * 8), sw128_desc_mn(va + kk * 2048, 4096), id_pv,
                        (j | p | kk) ? 1u : 0u);
          slot_release();
        }
        mma_commit(pv_done(j & 1));
        return true;
      };
      if (n_kv > 0 && !issue_qk(0)) goto done;
      for (int j = 0; j < n_kv; ++j) {
        if (j + 1 < n_kv && !issue_qk(j + 1)) goto done;
        if (!issue_pv(j)) goto done;
      }
    }
  } else {
    // ------------------------------------------------------------------ softmax: two warpgroups
    // Warps 2-5 and 6-9 reach the same TMEM lanes (lane quarter = warp % 4), so every
    // row has two threads: `half` 0 takes keys 0-63 of each tile and O columns 0-127,
    // half 1 keys 64-127 and O columns 128-255.  They exchange their half-row maxima,
    // so both take the same lazy-rescale decision; half h writes its 32 columns of P
    // at [32 h, 32 h + 32) of the buffer, over scores that both have finished reading
    // by then (they passed the same exchange).
    const int quarter = warp & 3, half = (warp - 2) >> 2;
    const int r = quarter * 32 + lane;                // MMA row: head r / QT, query q0 + r % QT
    const int qi = r % QT;
    const int h = kvh * rep + r / QT;
    const int qpos = q_off + q0 + qi;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    // this thread's half of row r of Q, dims [128 half, 128 half + 128), into quarters
    // 2 half and 2 half + 1: 128-byte rows, 16-byte chunk c of row r at chunk c ^ (r & 7)
    {
      const bool ok = q0 + qi < Tq;
      const uint4* src = reinterpret_cast<const uint4*>(q + ((long)b * Tq + (ok ? q0 + qi : 0)) * ld_q + (long)h * AT_D);
      auto put = [&](int dim, uint4 v4) {
        *reinterpret_cast<uint4*>(sQ + (dim >> 6) * (Q_BYTES / 4) + r * 128 + ((((dim & 63) >> 3) ^ (r & 7)) << 4)) = v4;
      };
      if (!q_norm) {
#pragma unroll 4
        for (int c = 0; c < 16; ++c) {
          const int dim = 128 * half + 8 * c;
          put(dim, ok ? src[dim >> 3] : make_uint4(0, 0, 0, 0));
        }
      } else if (rot / 2 <= RT_MAX && QT <= STAB_ROWS) {
        // Every global load of the staging in one round trip: this thread's raw half-row
        // (kept in registers), and, shared by the CTA, the norm gain and the cos/sin rows of
        // its QT positions (from the forward's table, coalesced, or evaluated here in fp64)
        // into shared memory.  Then the row's sum of squares is exchanged with the other
        // half's thread, and the rows are normalised and rotated from registers and shared
        // memory.
        const int tid_s = threadIdx.x - 64;             // 0..255
        const int rt = rot / 2;
        uint4 raw[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) raw[c] = ok ? src[16 * half + c] : make_uint4(0, 0, 0, 0);
        if (tid_s < AT_D / 8) sgain[tid_s] = reinterpret_cast<const uint4*>(q_norm)[tid_s];
        for (int i = tid_s; i < QT * rt; i += 256) {
          const int qr = i / rt, jp = i - qr * rt;
          float2 t2 = make_float2(1.f, 0.f);
          if (q0 + qr < Tq) {
            const int p = q_off + q0 + qr;
            if (rope_tab) {
              t2 = rope_tab[(long)(p - tab_pos0) * rt + jp];
            } else {
              const double theta = pow((double)rope_base, -2.0 * (double)jp / (double)rot);
              double ang = (double)p * theta;
              ang -= 6.283185307179586 * floor(ang / 6.283185307179586);
              double sd, cd;
              sincos(ang, &sd, &cd);
              t2 = make_float2((float)cd, (float)sd);
            }
          }
          stab[qr * (RT_MAX + 1) + jp] = t2;
        }
        float ss = 0.f;
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          float x8[8];
          unpack8_bf16(raw[c], x8);
#pragma unroll
          for (int e = 0; e < 8; ++e) ss = fmaf(x8[e], x8[e], ss);
        }
        xsum[half * AT_M + r] = ss;
        asm volatile("bar.sync 1, 256;" ::: "memory");     // the 256 softmax threads: sums, gain, table
        const float inv = rsqrtf((xsum[r] + xsum[AT_M + r]) * (1.f / AT_D) + eps);
        asm volatile("bar.sync 1, 256;" ::: "memory");     // both read before xsum is reused
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const int dim = 128 * half + 8 * c;
          float x8[8], g8[8];
          unpack8_bf16(raw[c], x8);
          unpack8_bf16(sgain[dim >> 3], g8);
#pragma unroll
          for (int e = 0; e < 8; ++e) x8[e] = x8[e] * inv * g8[e];
          if (dim < rot) {
#pragma unroll
            for (int e = 0; e < 8; e += 2) {
              const float2 t2 = stab[qi * (RT_MAX + 1) + ((dim + e) >> 1)];
              const float a0 = x8[e], a1 = x8[e + 1];
              x8[e] = a0 * t2.x - a1 * t2.y;
              x8[e + 1] = a0 * t2.y + a1 * t2.x;
            }
          }
          uint4 v4;
          uint32_t* pw = reinterpret_cast<uint32_t*>(&v4);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const __nv_bfloat162 pr = __floats2bfloat162_rn(x8[2 * e], x8[2 * e + 1]);
            pw[e] = *reinterpret_cast<const uint32_t*>(&pr);
          }
          put(dim, v4);
        }
      } else {
        // other head groupings or rotary widths: two passes over the raw row (sum of
        // squares, then scale and rotate), the angles from the table or in fp64
        float ss = 0.f;
#pragma unroll 4
        for (int c = 0; c < 16; ++c) {
          float x8[8];
          load8(reinterpret_cast<const __nv_bfloat16*>(src) + 128 * half + 8 * c, x8);
#pragma unroll
          for (int e = 0; e < 8; ++e) ss = fmaf(x8[e], x8[e], ss);
        }
        xsum[half * AT_M + r] = ok ? ss : 0.f;
        asm volatile("bar.sync 1, 256;" ::: "memory");     // the 256 softmax threads
        const float inv = rsqrtf((xsum[r] + xsum[AT_M + r]) * (1.f / AT_D) + eps);
        asm volatile("bar.sync 1, 256;" ::: "memory");     // both read before xsum is reused
        const int pos = qpos;
#pragma unroll 2
        for (int c = 0; c < 16; ++c) {
          const int dim = 128 * half + 8 * c;
          float x8[8], g8[8];
          load8(reinterpret_cast<const __nv_bfloat16*>(src) + dim, x8);
          load8(q_norm + dim, g8);
#pragma unroll
          for (int e = 0; e < 8; ++e) x8[e] = ok ? x8[e] * inv * g8[e] : 0.f;
          if (dim < rot) {
#pragma unroll
            for (int e = 0; e < 8; e += 2) {
              const int jp = (dim + e) >> 1;
              float cs, sn;
              if (rope_tab) {
                const float2 t2 = rope_tab[(long)(ok ? pos - tab_pos0 : 0) * (rot / 2) + jp];
                cs = t2.x;
                sn = t2.y;
              } else {
                const double theta = pow((double)rope_base, -2.0 * (double)jp / (double)rot);
                double ang = (double)pos * theta;
                ang -= 6.283185307179586 * floor(ang / 6.283185307179586);
                double sd, cd;
                sincos(ang, &sd, &cd);
                cs = (float)cd;
                sn = (float)sd;
              }
              const float a0 = x8[e], a1 = x8[e + 1];
              x8[e] = a0 * cs - a1 * sn;
              x8[e + 1] = a0 * sn + a1 * cs;
            }
          }
          uint4 v4;
          uint32_t* pw = reinterpret_cast<uint32_t*>(&v4);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const __nv_bfloat162 pr = __floats2bfloat162_rn(x8[2 * e], x8[2 * e + 1]);
            pw[e] = *reinterpret_cast<const uint32_t*>(&pr);
          }
          put(dim, v4);
        }
      }
      fence_proxy_async();                            // generic stores -> tensor-core reads
      mbar_arrive(q_full);
    }
    float m_used = -INFINITY, l = 0.f;
    for (int j = 0; j < n_kv; ++j) {
      const int s = j & 1;
      if (!mbar_wait(s_full(s), (j >> 1) & 1, abort_flag)) goto done;
      fence_after();
      uint32_t sa[32], sb[32];
      tmem_ld32(tmem + lane_off + s * AT_N + half * 64, sa);         // this half's 64 keys
      tmem_ld32(tmem + lane_off + s * AT_N + half * 64 + 32, sb);
      tmem_wait_ld();
      // raw scores; the max is taken before scaling (scale > 0).  Only tiles that reach
      // the causal diagonal or the end of the keys need the per-element mask.
      float t[64];
      float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
      const int kbase = j * AT_N + half * 64;
      const bool all_visible = j * AT_N + AT_N <= Tkv && (!causal || j * AT_N + AT_N - 1 <= q_off + q0);
      if (all_visible) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          t[i] = __uint_as_float(sa[i]);
          t[32 + i] = __uint_as_float(sb[i]);
        }
      } else {
#pragma unroll
        for (int i = 0; i < 64; ++i) {
          const int key = kbase + i;
          const bool ok = key < Tkv && (!causal || key <= qpos);
          t[i] = ok ? __uint_as_float(i < 32 ? sa[i] : sb[i - 32]) : -INFINITY;
        }
      }
#pragma unroll
      for (int i = 0; i < 64; ++i) m4[i & 3] = fmaxf(m4[i & 3], t[i]);
      const float mh = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
      // exchange the half-row maxima (slot by tile parity: the partner reads it before
      // either thread can reach the tile two ahead)
      xmax[(s * 2 + half) * AT_M + r] = mh;
      mbar_arrive(x_bar(s));
      if (!mbar_wait(x_bar(s), (j >> 1) & 1, abort_flag)) goto done;
      // the row maximum of the tile (every processed tile but a last partial one has a
      // visible key per row; a row without one gets P = 0 there)
      const float mt = fmaxf(mh, xmax[(s * 2 + (half ^ 1)) * AT_M + r]) * scale_log2;
      const bool grow = mt > m_used + RESCALE_THRESHOLD;
      // O holds tiles < j scaled by 2^-m_used.  The TMEM loads and stores are warp-wide
      // instructions, so the whole warp rescales when any of its rows must (the others
      // with factor 1, which leaves O unchanged); the two threads of a row decide alike.
      if (j > 0 && __any_sync(0xffffffffu, grow)) {
        if (!mbar_wait(pv_done((j - 1) & 1), ((j - 1) >> 1) & 1, abort_flag)) goto done;
        const float corr = grow ? exp2f(m_used - mt) : 1.f;
        l *= corr;
        fence_after();
#pragma unroll 1
        for (int c = 0; c < AT_D / 64; ++c) {
          uint32_t o[32];
          tmem_ld32(tO + lane_off + half * (AT_D / 2) + c * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * corr);
          tmem_st32(tO + lane_off + half * (AT_D / 2) + c * 32, o);
        }
        tmem_wait_st();
      }
      if (grow) m_used = mt;
      // this half's 64 keys of P as bf16 pairs (key 2i in the low half of column i) into
      // columns [32 half, 32 half + 32) of this tile's S buffer, the A operand of P V
      // (packed f32x2 FMAs and adds: two scores per instruction)
      float ps0 = 0.f, ps1 = 0.f;
      uint32_t w[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        float x0, x1;
        fma_x2(x0, x1, t[2 * i], t[2 * i + 1], scale_log2, scale_log2, -m_used, -m_used);
        const float p0 = ex2(x0), p1 = ex2(x1);
        add_x2(ps0, ps1, ps0, ps1, p0, p1);
        const __nv_bfloat162 pr = __floats2bfloat162_rn(p0, p1);
        w[i] = *reinterpret_cast<const uint32_t*>(&pr);
      }
      const float psum = ps0 + ps1;
      tmem_st32(tmem + lane_off + s * AT_N + half * 32, w);
      tmem_wait_st();
      l += psum;
      fence_before();
      mbar_arrive(p_full(s));
    }
    if (n_kv > 0 && !mbar_wait(pv_done((n_kv - 1) & 1), ((n_kv - 1) >> 1) & 1, abort_flag)) goto done;
    fence_after();
    // the row sum over both halves
    xsum[half * AT_M + r] = l;
    mbar_arrive(l_bar);
    if (!mbar_wait(l_bar, 0, abort_flag)) goto done;
    const float lt = l + xsum[(half ^ 1) * AT_M + r];
    const int row = q0 + qi;
    const float inv = lt > 0.f ? 1.f / lt : 0.f;
#pragma unroll 1
    for (int c = 0; c < AT_D / 64; ++c) {
      const int col = half * (AT_D / 2) + c * 32;
      uint32_t o[32];
      tmem_ld32(tO + lane_off + col, o);
      tmem_wait_ld();
      if (row < Tq) {
        const long m = (long)b * Tq + row;
        float v[32];
        const __nv_bfloat16* gp = gate ? gate + m * ld_gate + (long)h * AT_D + col : nullptr;
#pragma unroll
        for (int i = 0; i < 32; i += 8) {
          float g8[8];
          if (gp) load8(gp + i, g8);
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float x = __uint_as_float(o[i + e]) * inv;
            v[i + e] = gp ? x / (1.f + __expf(-g8[e])) : x;
          }
        }
        __nv_bfloat16* op = out + (m * Hq + h) * AT_D + col;
#pragma unroll
        for (int i = 0; i < 32; i += 8) store8(op + i, v + i);
      }
    }
  }
done:
  __syncthreads();
  if (warp == 1) {
    fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace tc

bool gqa_tc_supported(int dh, int dtype, const void* q, int ld_q, const void* gate, int ld_gate, const void* k,
                      const void* v, int kv_cap) {
  auto al16 = [](const void* p) { return ((uintptr_t)p % 16) == 0; };
  return dtype == BF16 && dh == tc::AT_D && al16(q) && al16(k) && al16(v) && (ld_q % 8 == 0) &&
         (!gate || (al16(gate) && ld_gate % 8 == 0)) && kv_cap > 0;
}

cudaError_t gqa_attn_tc(const void* q, int ld_q, const void* k, const void* v, int kv_cap, const void* gate,
                        int ld_gate, void* out, int B, int Tq, int Tkv, int q_off, int Hq, int Hkv, int causal,
                        cudaStream_t s, const QNorm* qn) {
  using namespace tc;
  const int rep = Hq / Hkv;
  if (rep < 1 || AT_M % rep != 0) return cudaErrorNotSupported;
  const int QT = AT_M / rep;                              // query positions per CTA
  CUtensorMap mK, mV;
  if (!make_map_3d(&mK, k, AT_D, Tkv, (long)B * Hkv, AT_D, (long)kv_cap * AT_D, 64, AT_N)) return cudaErrorNotSupported;
  if (!make_map_3d(&mV, v, AT_D, Tkv, (long)B * Hkv, AT_D, (long)kv_cap * AT_D, 64, 32)) return cudaErrorNotSupported;
  {
    cudaError_t e = set_smem_limit(attn_tc_kernel, AT_SMEM);
    if (e != cudaSuccess) return e;
  }
  dim3 grid((Tq + QT - 1) / QT, Hkv, B);
  const float scale_log2 = 1.4426950408889634f / sqrtf((float)AT_D);
  if (qn && qn->rot > AT_D / 2) return cudaErrorNotSupported;   // rotary dims must lie in the first half
  attn_tc_kernel<<<grid, AT_THREADS, AT_SMEM, s>>>(
      (const __nv_bfloat16*)q, ld_q, mK, mV, (const __nv_bfloat16*)gate, ld_gate, (__nv_bfloat16*)out, Tq, Tkv, q_off,
      Hq, Hkv, causal, scale_log2, QT, qn ? (const __nv_bfloat16*)qn->gain : nullptr, qn ? qn->eps : 0.f,
      qn ? qn->rot : 0, qn ? qn->base : 1.f, qn ? qn->tab : nullptr, qn ? qn->tab_pos0 : 0);
  return cudaGetLastError();
}

}  // namespace lk
