// Causal GQA flash attention on the 5th-generation tensor cores, head dim 256, bf16
// ("Loop-9B engineering teardown" §三: GQA 16 q / 4 KV heads, head dim 256, output gate).
//
// One CTA = 128 MMA rows = the Hq/Hkv q heads of one KV group x 128/(Hq/Hkv) query
// positions (row r: head r / QT, position q0 + r % QT), so every K/V tile loaded serves
// all heads that share it.  Warps:
//   0     TMA: K and V tiles of 64 keys into two separate rings (3-D maps over the per-execution slab, so keys
//         past Tkv read as zeros).  A K slot is free as soon as Q K^T has read it, a V
//         slot once P V has, so K tiles stream in ahead of their use;
//   1     MMA: S_j = Q K_j^T (M 128, N 64, K 256) into one of two TMEM buffers, and
//         O += P_j V_j (M 128, N 256, K 64) into TMEM, with P_j read from TMEM as the
//         A operand and V an MN-major shared-memory operand;
//   2..9  softmax in two warpgroups, two threads per query row (TMEM lane = row): both
//         read the tile's 64 scores for the row max, each computes P for half of the
//         keys and rescales / writes half of O's columns.  Scores -> exp2 ->
//         bf16 P, packed two per column and stored over the first 32 columns of S_j's
//         own buffer; O is rescaled in TMEM only when the running max grows by more
//         than 2^8 (the stale max cancels in the final O / l); finally
//         O / l * sigmoid(gate) is stored.  Each thread first writes its half of its
//         row of Q into TMEM, where Q K^T reads it as the A operand.
// Q K^T of tile j+1 overlaps the softmax of tile j.  The tensor pipe runs its MMAs in
// issue order (Q K^T j+1, P V j, Q K^T j+2, ...), so P V j has read P_j before
// Q K^T j+2 overwrites that buffer: no barrier is needed for the reuse.  The K ring
// has four stages, the V ring two.  TMEM: S buffers, Q and O fill all 512 columns.
// All waits are bounded.
#include "internal.h"
#include "tc_common.cuh"

namespace lk {
namespace tc {

constexpr int AT_M = 128, AT_N = 64, AT_D = 256;
constexpr int KV_TILE = AT_N * AT_D * 2;         // 32 KiB each for K and V
constexpr int K_STAGES = 4, V_STAGES = 2;
constexpr int XCH_BYTES = 2 * AT_M * 4;             // row sums of the two halves [2][128]
constexpr int AT_SMEM = (K_STAGES + V_STAGES) * KV_TILE + 1024 + 256 + XCH_BYTES;
constexpr int AT_THREADS = 320;                  // TMA, MMA, two softmax warpgroups
// mbarrier slots
constexpr int B_Q = 0, B_KF = 1, B_KE = B_KF + K_STAGES, B_VF = B_KE + K_STAGES, B_VE = B_VF + V_STAGES,
              B_SF = B_VE + V_STAGES, B_PF = B_SF + 2, B_PV = B_PF + 2, B_X = B_PV + 2, B_L = B_X + 2,
              N_BARS = B_L + 1;
static_assert(N_BARS * 8 + 8 <= 256, "barrier region");
// TMEM columns: S buffers 0..63 and 64..127 (P over the first 32 of each), Q 128..255
// (bf16 pairs: the A operand of Q K^T), O 256..511
constexpr uint32_t T_Q = 128, T_O = 256;
constexpr float RESCALE_THRESHOLD = 8.0f;        // log2 units

// 2^x as one MUFU op (x <= 0 here after the row-max shift; denormal results flush to 0).
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

__global__ void __launch_bounds__(AT_THREADS, 1)
    attn_tc_kernel(const __nv_bfloat16* __restrict__ q, int ld_q, const __grid_constant__ CUtensorMap tK,
                   const __grid_constant__ CUtensorMap tV, const __nv_bfloat16* __restrict__ gate, int ld_gate,
                   __nv_bfloat16* __restrict__ out, int Tq, int Tkv, int q_off, int Hq, int Hkv, int causal,
                   float scale_log2, int QT) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sK = smem;                                 // K ring: stage s at s * KV_TILE
  uint8_t* sV = sK + K_STAGES * KV_TILE;              // V ring
  uint64_t* bars = (uint64_t*)(sV + V_STAGES * KV_TILE);
  uint32_t* tmem_slot = (uint32_t*)(bars + N_BARS);
  float* xsum = (float*)((uint8_t*)bars + 256);        // row-sum exchange [2 halves][AT_M]
  volatile int* abort_flag = (volatile int*)(tmem_slot + 1);
  const uint32_t bar0 = smem_u32(bars);
  const uint32_t q_full = bar0 + 8u * B_Q;
  auto k_full = [&](int s) { return bar0 + 8u * (B_KF + s); };
  auto k_empty = [&](int s) { return bar0 + 8u * (B_KE + s); };
  auto v_full = [&](int s) { return bar0 + 8u * (B_VF + s); };
  auto v_empty = [&](int s) { return bar0 + 8u * (B_VE + s); };
  auto s_full = [&](int b) { return bar0 + 8u * (B_SF + b); };
  // one p_full / pv_done per S buffer, so no barrier runs two phases ahead of its waiter
  auto p_full = [&](int s) { return bar0 + 8u * (B_PF + s); };
  auto pv_done = [&](int s) { return bar0 + 8u * (B_PV + s); };
  auto x_bar = [&](int s) { return bar0 + 8u * (B_X + s); };     // both halves done reading S (tile parity s)
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
    for (int s = 0; s < K_STAGES; ++s) {
      mbar_init(k_full(s), 1);
      mbar_init(k_empty(s), 1);
    }
    for (int s = 0; s < V_STAGES; ++s) {
      mbar_init(v_full(s), 1);
      mbar_init(v_empty(s), 1);
    }
    for (int s = 0; s < 2; ++s) mbar_init(s_full(s), 1);
    for (int s = 0; s < 2; ++s) {
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
  const uint32_t tO = tmem + T_O, tQ = tmem + T_Q;

  if (warp == 0) {
    if (lane == 0) {
      for (int j = 0; j < n_kv; ++j) {
        const int sk = j % K_STAGES, sv = j % V_STAGES;
        if (!mbar_wait(k_empty(sk), ((j / K_STAGES) & 1) ^ 1, abort_flag)) goto done;
        mbar_expect_tx(k_full(sk), KV_TILE);
        const uint32_t kd = smem_u32(sK + sk * KV_TILE), vd = smem_u32(sV + sv * KV_TILE);
#pragma unroll
        for (int c = 0; c < 4; ++c) tma_load_3d(kd + c * (KV_TILE / 4), &tK, k_full(sk), c * 64, j * AT_N, b * Hkv + kvh);
        if (!mbar_wait(v_empty(sv), ((j / V_STAGES) & 1) ^ 1, abort_flag)) goto done;
        mbar_expect_tx(v_full(sv), KV_TILE);
#pragma unroll
        for (int c = 0; c < 4; ++c) tma_load_3d(vd + c * (KV_TILE / 4), &tV, v_full(sv), c * 64, j * AT_N, b * Hkv + kvh);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t id_qk = idesc_bf16(AT_M, AT_N);
      constexpr uint32_t id_pv = idesc_bf16(AT_M, AT_D, 1);
      if (!mbar_wait(q_full, 0, abort_flag)) goto done;
      fence_after();
      auto issue_qk = [&](int j) -> bool {
        const int s = j & 1, sk = j % K_STAGES;
        if (!mbar_wait(k_full(sk), (j / K_STAGES) & 1, abort_flag)) return false;
        fence_after();
        const uint32_t ka = smem_u32(sK + sk * KV_TILE);
#pragma unroll
        for (int ks = 0; ks < AT_D / 16; ++ks) {
          const uint32_t sub = ks >> 2, in = (ks & 3) * 32;   // 64-wide sub-tile of K, 16-element step
          mma_bf16_ts(tmem + s * AT_N, tQ + ks * 8, sw128_desc(ka + sub * (KV_TILE / 4) + in), id_qk, ks > 0 ? 1u : 0u);
        }
        mma_commit(s_full(s));
        mma_commit(k_empty(sk));           // K slot free once these MMAs have read it
        return true;
      };
      if (n_kv > 0 && !issue_qk(0)) goto done;
      for (int j = 0; j < n_kv; ++j) {
        if (j + 1 < n_kv && !issue_qk(j + 1)) goto done;
        const int sv = j % V_STAGES;
        if (!mbar_wait(p_full(j & 1), (j >> 1) & 1, abort_flag)) goto done;
        if (!mbar_wait(v_full(sv), (j / V_STAGES) & 1, abort_flag)) goto done;
        fence_after();
        const uint32_t pa = tmem + (uint32_t)((j & 1) * AT_N);     // P_j: bf16 pairs over 32 columns
        const uint32_t va = smem_u32(sV + sv * KV_TILE);
#pragma unroll
        for (int ks = 0; ks < AT_N / 16; ++ks)
          mma_bf16_ts(tO, pa + ks * 8, sw128_desc_mn(va + ks * 2048, KV_TILE / 4), id_pv, (j > 0 || ks > 0) ? 1u : 0u);
        mma_commit(pv_done(j & 1));
        mma_commit(v_empty(sv));
      }
    }
  } else {
    // ------------------------------------------------------------------ softmax: two warpgroups
    // Warps 2-5 and 6-9 reach the same TMEM lanes (lane quarter = warp % 4), so every
    // row has two threads: `half` 0 takes keys 0-31 of each tile and O columns 0-127,
    // half 1 keys 32-63 and O columns 128-255.  Both read all 64 scores, so they take
    // the same lazy-rescale decision without a hand-off; each writes its 16 columns of
    // P once both have finished reading S (one mbarrier round per tile).
    const int quarter = warp & 3, half = (warp - 2) >> 2;
    const int r = quarter * 32 + lane;                // MMA row: head r / QT, query q0 + r % QT
    const int qi = r % QT;
    const int h = kvh * rep + r / QT;
    const int qpos = q_off + q0 + qi;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    // this thread's half of the row of Q into TMEM lane r as bf16 pairs (dims 2c, 2c + 1
    // in column c): dims [128 half, 128 half + 128) -> columns [64 half, 64 half + 64)
    {
      const bool ok = q0 + qi < Tq;
      const uint4* src = reinterpret_cast<const uint4*>(q + ((long)b * Tq + (ok ? q0 + qi : 0)) * ld_q + (long)h * AT_D);
#pragma unroll 1
      for (int c = 2 * half; c < 2 * half + 2; ++c) {  // 32 columns = 64 dims per store
        uint32_t w[32];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint4 v4 = ok ? src[c * 8 + i] : make_uint4(0, 0, 0, 0);
          w[4 * i] = v4.x, w[4 * i + 1] = v4.y, w[4 * i + 2] = v4.z, w[4 * i + 3] = v4.w;
        }
        tmem_st32(tQ + lane_off + c * 32, w);
      }
      tmem_wait_st();
      fence_before();
      mbar_arrive(q_full);
    }
    float m_used = -INFINITY, l = 0.f;
    for (int j = 0; j < n_kv; ++j) {
      const int s = j & 1;
      if (!mbar_wait(s_full(s), (j >> 1) & 1, abort_flag)) goto done;
      fence_after();
      // both threads of a row read all 64 scores (the row max needs them all; reading
      // twice from TMEM is cheaper than a hand-off between the two threads)
      uint32_t sa[32], sb[32];
      tmem_ld32(tmem + lane_off + s * AT_N + half * 32, sa);          // this half's keys
      tmem_ld32(tmem + lane_off + s * AT_N + (half ^ 1) * 32, sb);    // the other half's
      tmem_wait_ld();
      // raw scores; the max is taken before scaling (scale > 0).  Only tiles that reach
      // the causal diagonal or the end of the keys need the per-element mask.
      float t[32];
      float mh = -INFINITY;
      const int kbase = j * AT_N + half * 32, kother = j * AT_N + (half ^ 1) * 32;
      const bool all_visible = j * AT_N + AT_N <= Tkv && (!causal || j * AT_N + AT_N - 1 <= q_off + q0);
      if (all_visible) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          t[i] = __uint_as_float(sa[i]);
          mh = fmaxf(mh, fmaxf(t[i], __uint_as_float(sb[i])));
        }
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int key = kbase + i, key2 = kother + i;
          const bool ok = key < Tkv && (!causal || key <= qpos);
          const bool ok2 = key2 < Tkv && (!causal || key2 <= qpos);
          t[i] = ok ? __uint_as_float(sa[i]) : -INFINITY;
          mh = fmaxf(mh, fmaxf(t[i], ok2 ? __uint_as_float(sb[i]) : -INFINITY));
        }
      }
      // the row maximum of the tile (every processed tile has a visible key per row)
      const float mt = mh * scale_log2;
      if (mt > m_used + RESCALE_THRESHOLD) {
        if (j > 0) {                                  // O holds tiles < j scaled by 2^-m_used
          if (!mbar_wait(pv_done((j - 1) & 1), ((j - 1) >> 1) & 1, abort_flag)) goto done;
          const float corr = exp2f(m_used - mt);
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
        m_used = mt;
      }
      // this half's 32 keys of P as bf16 pairs (key 2i in the low half of column i) into
      // columns [16 half, 16 half + 16) of this tile's S buffer, the A operand of P V
      float psum = 0.f;
      uint32_t w[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float p0 = ex2(fmaf(t[2 * i], scale_log2, -m_used));
        const float p1 = ex2(fmaf(t[2 * i + 1], scale_log2, -m_used));
        psum += p0 + p1;
        const __nv_bfloat162 pr = __floats2bfloat162_rn(p0, p1);
        w[i] = *reinterpret_cast<const uint32_t*>(&pr);
      }
      // the partner may still be reading S columns 16-31 (which P overwrites): both
      // threads pass this barrier after their S loads have completed
      mbar_arrive(x_bar(s));
      if (!mbar_wait(x_bar(s), (j >> 1) & 1, abort_flag)) goto done;
      tmem_st16(tmem + lane_off + s * AT_N + half * 16, w);
      tmem_wait_st();
      l += psum;
      fence_before();
      mbar_arrive(p_full(j & 1));
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
                        cudaStream_t s) {
  using namespace tc;
  const int rep = Hq / Hkv;
  if (rep < 1 || AT_M % rep != 0) return cudaErrorNotSupported;
  const int QT = AT_M / rep;                              // query positions per CTA
  if (QT % 8 != 0) return cudaErrorNotSupported;          // whole 8-row swizzle atoms per head
  CUtensorMap mK, mV;
  if (!make_map_3d(&mK, k, AT_D, Tkv, (long)B * Hkv, AT_D, (long)kv_cap * AT_D, 64, AT_N)) return cudaErrorNotSupported;
  if (!make_map_3d(&mV, v, AT_D, Tkv, (long)B * Hkv, AT_D, (long)kv_cap * AT_D, 64, AT_N)) return cudaErrorNotSupported;
  {
    cudaError_t e = set_smem_limit(attn_tc_kernel, AT_SMEM);
    if (e != cudaSuccess) return e;
  }
  dim3 grid((Tq + QT - 1) / QT, Hkv, B);
  const float scale_log2 = 1.4426950408889634f / sqrtf((float)AT_D);
  attn_tc_kernel<<<grid, AT_THREADS, AT_SMEM, s>>>((const __nv_bfloat16*)q, ld_q, mK, mV, (const __nv_bfloat16*)gate, ld_gate,
                                            (__nv_bfloat16*)out, Tq, Tkv, q_off, Hq, Hkv, causal, scale_log2, QT);
  return cudaGetLastError();
}

}  // namespace lk
