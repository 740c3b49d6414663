// bf16 projection Y = X W^T for many rows (M > 128) on CTA pairs (tcgen05 cta_group::2).
//
// The prefill projections and the SwiGLU FFN of the decoder layer ("Loop-9B engineering
// teardown" §二).  Two CTAs of a cluster form a pair that computes a 256 x 256 tile of
// X W^T with one stream of M = 256 MMAs:
//   - each CTA stages its own 128 rows of X and one half of the tile's 256 weight rows
//     (the MMA splits B by N across the pair), so a 256 x 256 x 64 step moves 32 KB per
//     CTA through shared memory instead of 48 KB for a 128 x 256 tile on one CTA;
//   - the even CTA of the pair (the leader) owns the full / tempty barriers and issues
//     the MMAs; both CTAs' TMA loads complete on the leader's full barrier, and the
//     leader's commits are multicast to the empty / tfull barriers of both CTAs;
//   - each CTA's epilogue drains its own TMEM (its 128 rows x 256 columns), then arrives
//     on the leader's tempty barrier (remotely from the odd CTA);
//   - SwiGLU: the leader stages 128 rows of W_gate and the odd CTA the same rows of W_up,
//     so TMEM columns [0, 128) hold the gate and [128, 256) the up projection.
// Persistent: one pair per two SMs, tiles in groups of 8 row-pairs (2,048 rows) so a
// wave's activation rows stay in L2.  Every mbarrier wait is bounded; cluster barriers
// order the barrier set-up before any peer traffic and keep both CTAs resident until
// the last remote arrival.
#include "internal.h"
#include "tc_common.cuh"

namespace lk {
namespace tc {
namespace p2 {

constexpr int BM = 128;          // rows of X per CTA (256 per pair)
constexpr int BN = 256;          // MMA N: weight rows per pair tile (128 per CTA)
constexpr int BK = 64;
constexpr int A_BYTES = BM * BK * 2;                 // 16 KB
constexpr int B_BYTES = (BN / 2) * BK * 2;           // 16 KB (this CTA's half)
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int STAGES = 6;
constexpr int TMEM_COLS = 2 * BN;                    // two accumulators
constexpr size_t SMEM = (size_t)STAGES * STAGE_BYTES + 1024 + 256;
constexpr int GROUP_M = 8;                           // row-pairs per raster group

__device__ __forceinline__ uint32_t cta_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t map_to(uint32_t a, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(rank));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// TMA tile load into this CTA's shared memory that completes on the pair leader's
// mbarrier (bar: a shared::cluster address, possibly the peer's).
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map, uint32_t bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], "
      "[%2];" ::"r"(dst),
      "l"((uint64_t)map), "r"(bar), "r"(x), "r"(y)
      : "memory");
}
__device__ __forceinline__ void mma_bf16_pair(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}
// Arrive (once each) on the barrier at this shared offset in every CTA of `mask`, when
// the leader's MMAs issued so far have completed.
__device__ __forceinline__ void commit_pair(uint32_t bar, uint16_t mask) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
                   bar),
               "h"(mask)
               : "memory");
}
__device__ __forceinline__ void arrive_remote(uint32_t bar_cluster) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster) : "memory");
}

// EPI_GDN: one row's 128 columns of a q or k head from TMEM (4 loads of 32), L2-normalised
// and stored; v heads copied; the gate tile turned into g and beta.  The TMEM loads are
// warp-collective: every lane issues them, and only the stores are guarded by the row.
__device__ __forceinline__ void gdn_epilogue(uint32_t t_row, int row, int n0, int M, const GdnEpi& ep) {
  const int H = ep.H, qk = 2 * H * 128, vend = qk + H * 128;
  const bool ok = row < M;
  if (n0 < vend) {
#pragma unroll 1
    for (int hh = 0; hh < 2; ++hh) {                  // the tile's two heads
      const int col = n0 + hh * 128;
      const uint32_t th = t_row + hh * 128;
      float inv = 1.f;
      if (col < qk) {
        float ss = 0.f;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t r[32];
          tmem_ld32(th + c * 32, r);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) ss = fmaf(__uint_as_float(r[i]), __uint_as_float(r[i]), ss);
        }
        inv = rsqrtf(ss + ep.eps);
      }
      __nv_bfloat16* dst;
      if (col < H * 128) dst = (__nv_bfloat16*)ep.q + ((long)row * H + col / 128) * 128;
      else if (col < qk) dst = (__nv_bfloat16*)ep.k + ((long)row * H + (col - H * 128) / 128) * 128;
      else dst = (__nv_bfloat16*)ep.v + ((long)row * H + (col - qk) / 128) * 128;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t r[32];
        tmem_ld32(th + c * 32, r);
        tmem_wait_ld();
        float v[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]) * inv;
        if (ok) {
#pragma unroll
          for (int i = 0; i < 32; i += 8) store8(dst + c * 32 + i, v + i);
        }
      }
    }
  } else {                                            // gates: a (H columns) then b (H columns)
    uint32_t r[32];
    tmem_ld32(t_row, r);
    tmem_wait_ld();
    for (int j = 0; ok && j < H && j < 16; ++j) {
      const float a = __uint_as_float(r[j]) + ep.a_bias[j];
      const float b = __uint_as_float(r[H + j]) + ep.b_bias[j];
      ep.g[(long)row * H + j] = -(a > 20.f ? a : log1pf(expf(a)));
      ep.beta[(long)row * H + j] = 1.f / (1.f + expf(-b));
    }
  }
}

// EPI_FA: one row's 256 columns (one head or a 256-column piece of the gate / v block) from
// TMEM (8 loads of 32).  q and k heads: sum of squares, then scaled by rsqrt(mean + eps)
// and the gain, the first `rot` dims rotated in adjacent pairs, stored (k into the slab);
// gate and v pieces copied.  The TMEM loads are warp-collective: every lane issues them,
// and only the stores are guarded by the row.
__device__ __forceinline__ void fa_epilogue(uint32_t t_row, int row, int n0, int M, const FaEpi& fe) {
  constexpr int D = 256;
  const bool ok = row < M;
  const int qe = fe.Hq * D, ge = 2 * qe, ke = ge + fe.Hkv * D;
  const int b = ok ? row / fe.T : 0, t = ok ? row % fe.T : 0;
  const long pos = (long)fe.pos0 + t;
  const bool norm = n0 < qe || (n0 >= ge && n0 < ke);
  __nv_bfloat16* dst;
  if (n0 < qe) dst = (__nv_bfloat16*)fe.q + ((long)row * fe.Hq + n0 / D) * D;
  else if (n0 < ge) dst = (__nv_bfloat16*)fe.gate + (long)row * fe.ld_gate + (n0 - qe);
  else if (n0 < ke) dst = (__nv_bfloat16*)fe.k_slab + (((long)b * fe.Hkv + (n0 - ge) / D) * fe.kv_cap + pos) * D;
  else dst = (__nv_bfloat16*)fe.v_slab + (((long)b * fe.Hkv + (n0 - ke) / D) * fe.kv_cap + pos) * D;
  float inv = 1.f;
  if (norm) {
    float ss = 0.f;
#pragma unroll 1
    for (int c = 0; c < D / 32; ++c) {
      uint32_t r[32];
      tmem_ld32(t_row + c * 32, r);
      tmem_wait_ld();
#pragma unroll
      for (int i = 0; i < 32; ++i) ss = fmaf(__uint_as_float(r[i]), __uint_as_float(r[i]), ss);
    }
    inv = rsqrtf(ss * (1.f / D) + fe.eps);
  }
  const __nv_bfloat16* gain = (const __nv_bfloat16*)(n0 < qe ? fe.q_gain : fe.k_gain);
  const int rh = fe.rot / 2;
#pragma unroll 1
  for (int c = 0; c < D / 32; ++c) {
    uint32_t r[32];
    tmem_ld32(t_row + c * 32, r);
    tmem_wait_ld();
    float v[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
    if (norm) {
#pragma unroll
      for (int i = 0; i < 32; i += 8) {
        float g8[8];
        load8(gain + c * 32 + i, g8);
#pragma unroll
        for (int e = 0; e < 8; ++e) v[i + e] = v[i + e] * inv * g8[e];
      }
      if (c * 32 < fe.rot) {
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          const int j = (c * 32 + i) >> 1;
          if (j < rh) {
            const float2 cs = fe.rope[(long)t * rh + j];
            const float a0 = v[i], a1 = v[i + 1];
            v[i] = a0 * cs.x - a1 * cs.y;
            v[i + 1] = a0 * cs.y + a1 * cs.x;
          }
        }
      }
    }
    if (ok) {
#pragma unroll
      for (int i = 0; i < 32; i += 8) store8(dst + c * 32 + i, v + i);
    }
  }
}

template <int EPI>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(192, 1)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap tA, const __grid_constant__ CUtensorMap tB,
                     const __grid_constant__ CUtensorMap tB2, void* __restrict__ Y, int ldy,
                     const __nv_bfloat16* R, int ldr, int M, int N, int K, int vec_ok, const GdnEpi ep,
                     const FaEpi fe) {
  constexpr int OUT_COLS = (EPI == EPI_SWIGLU) ? BN / 2 : BN;   // output columns per pair tile
  extern __shared__ uint8_t smem_raw[];
  // the same offsets in both CTAs: descriptors and barriers are addressed by offset
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint64_t* bars = (uint64_t*)(smem + (size_t)STAGES * STAGE_BYTES);
  // bars: full[STAGES] (leader's used), empty[STAGES], tfull[2], tempty[2] (leader's used)
  uint32_t* tmem_slot = (uint32_t*)(bars + 2 * STAGES + 4);
  volatile int* abort_flag = (volatile int*)(tmem_slot + 1);

  const uint32_t rank = cta_rank();                    // 0 = leader, 1 = peer
  const bool leader = rank == 0;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pair = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;
  const int mb = (M + 2 * BM - 1) / (2 * BM);
  const int nb = (N + OUT_COLS - 1) / OUT_COLS;
  const int n_tiles = mb * nb;
  const int kb_n = (K + BK - 1) / BK;
  auto tile_mn = [&](int t, int& m0, int& n0) {
    const int per_group = GROUP_M * nb;
    const int grp = t / per_group, first_m = grp * GROUP_M;
    const int gm = min(GROUP_M, mb - first_m);
    const int in = t % per_group;
    m0 = (first_m + in % gm) * 2 * BM;
    n0 = (in / gm) * OUT_COLS;
  };
  const uint32_t bar0 = smem_u32(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
  auto tfull_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + a); };
  auto tempty_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + 2 + a); };

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);                       // the leader's expect_tx arrival
      mbar_init(empty_bar(s), 1);                      // one multicast commit
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar(a), 1);
      mbar_init(tempty_bar(a), 2 * 128);               // the epilogue threads of both CTAs
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"((uint32_t)TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  if (warp == 0 && lane == 0) {
    asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&tA) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&tB) : "memory");
    if (EPI == EPI_SWIGLU) asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&tB2) : "memory");
  }
  fence_before();
  __syncthreads();
  cluster_sync_all();                                  // both CTAs' barriers exist before any peer traffic
  fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer (both CTAs)
    if (lane == 0) {
      int it = 0;
      for (int t = pair; t < n_tiles; t += n_pairs) {
        int m0, n0;
        tile_mn(t, m0, n0);
        for (int kb = 0; kb < kb_n; ++kb, ++it) {
          const int s = it % STAGES;
          if (!mbar_wait(empty_bar(s), ((it / STAGES) & 1) ^ 1, abort_flag)) goto done;
          // the leader's full barrier counts the bytes of both CTAs' copies
          if (leader) mbar_expect_tx(full_bar(s), 2 * STAGE_BYTES);
          const uint32_t fb = map_to(full_bar(s), 0);
          const uint32_t a_dst = smem_u32(smem + (size_t)s * STAGE_BYTES);
          const uint32_t b_dst = a_dst + A_BYTES;
          tma_load_2d_pair(a_dst, &tA, fb, kb * BK, m0 + (int)rank * BM);
          if (EPI == EPI_SWIGLU)
            tma_load_2d_pair(b_dst, rank ? &tB2 : &tB, fb, kb * BK, n0);
          else
            tma_load_2d_pair(b_dst, &tB, fb, kb * BK, n0 + (int)rank * (BN / 2));
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer (leader only)
    if (leader && lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(2 * BM, BN);
      int it = 0, local = 0;
      for (int t = pair; t < n_tiles; t += n_pairs, ++local) {
        const int acc = local & 1;
        if (!mbar_wait(tempty_bar(acc), ((local >> 1) & 1) ^ 1, abort_flag)) goto done;
        fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
        for (int kb = 0; kb < kb_n; ++kb, ++it) {
          const int s = it % STAGES;
          if (!mbar_wait(full_bar(s), (it / STAGES) & 1, abort_flag)) goto done;
          fence_after();
          const uint32_t a_addr = smem_u32(smem + (size_t)s * STAGE_BYTES);
          const uint32_t b_addr = a_addr + A_BYTES;
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)
            mma_bf16_pair(d_tmem, sw128_desc(a_addr + k * 32), sw128_desc(b_addr + k * 32), idesc,
                          (kb > 0 || k > 0) ? 1u : 0u);
          commit_pair(empty_bar(s), 0x3);     // both CTAs' ring slots are free once read
        }
        commit_pair(tfull_bar(acc), 0x3);     // both CTAs' accumulators are ready
      }
    }
  } else {
    // ---------------------------------------------------------------- epilogue (warps 2..5, both CTAs)
    const int quarter = warp & 3;                 // TMEM lanes 32*quarter .. +31
    int local = 0;
    for (int t = pair; t < n_tiles; t += n_pairs, ++local) {
      const int acc = local & 1;
      int m0, n0;
      tile_mn(t, m0, n0);
      if (!mbar_wait(tfull_bar(acc), (local >> 1) & 1, abort_flag)) goto done;
      fence_after();
      const int row = m0 + (int)rank * BM + quarter * 32 + lane;
      const uint32_t t_row = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * BN);
      if (EPI == EPI_GDN) gdn_epilogue(t_row, row, n0, M, ep);
      if (EPI == EPI_FA) fa_epilogue(t_row, row, n0, M, fe);
#pragma unroll 1
      for (int c = 0; c < ((EPI == EPI_GDN || EPI == EPI_FA) ? 0 : OUT_COLS / 32); ++c) {
        uint32_t r[32];
        tmem_ld32(t_row + c * 32, r);
        float v[32];
        if (EPI == EPI_SWIGLU) {
          uint32_t u[32];
          tmem_ld32(t_row + BN / 2 + c * 32, u);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float gt = __uint_as_float(r[i]);
            v[i] = gt / (1.f + expf(-gt)) * __uint_as_float(u[i]);
          }
        } else {
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
        }
        const int col0 = n0 + c * 32;
        if (row >= M || col0 >= N) continue;
        const bool full = vec_ok && (col0 + 32 <= N);
        if (EPI == EPI_F32) {
          float* yp = reinterpret_cast<float*>(Y) + (long)row * ldy + col0;
          if (full) {
#pragma unroll
            for (int i = 0; i < 32; i += 4)
              *reinterpret_cast<float4*>(yp + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
          } else {
            for (int i = 0; i < 32 && col0 + i < N; ++i) yp[i] = v[i];
          }
        } else {
          __nv_bfloat16* yp = reinterpret_cast<__nv_bfloat16*>(Y) + (long)row * ldy + col0;
          if (EPI == EPI_ADD) {
            const __nv_bfloat16* rp = R + (long)row * ldr + col0;
            if (full) {
#pragma unroll
              for (int i = 0; i < 32; i += 8) {
                float rr[8];
                load8(rp + i, rr);
#pragma unroll
                for (int j = 0; j < 8; ++j) v[i + j] += rr[j];
              }
            } else {
              for (int i = 0; i < 32 && col0 + i < N; ++i) v[i] += __bfloat162float(rp[i]);
            }
          }
          if (full) {
#pragma unroll
            for (int i = 0; i < 32; i += 8) store8(yp + i, v + i);
          } else {
            for (int i = 0; i < 32 && col0 + i < N; ++i) yp[i] = __float2bfloat16(v[i]);
          }
        }
      }
      fence_before();
      if (leader) mbar_arrive(tempty_bar(acc));
      else arrive_remote(map_to(tempty_bar(acc), 0));
    }
  }
done:
  __syncthreads();
  cluster_sync_all();            // the peer's remote arrivals and copies have landed before either CTA leaves
  if (warp == 1) {
    fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"((uint32_t)TMEM_COLS)
                 : "memory");
  }
}

template <int EPI>
static cudaError_t launch(const void* X, int ldx, const void* W, const void* W2, const void* R, int ldr, void* Y,
                          int ldy, int M, int N, int K, cudaStream_t s, const GdnEpi& ep = GdnEpi{},
                          const FaEpi& fe = FaEpi{}) {
  constexpr int OUT_COLS = (EPI == EPI_SWIGLU) ? BN / 2 : BN;
  CUtensorMap tA, tB, tB2;
  if (!make_map(&tA, X, M, K, ldx, BM)) return cudaErrorNotSupported;
  if (!make_map(&tB, W, N, K, K, BN / 2)) return cudaErrorNotSupported;
  if (EPI == EPI_SWIGLU) {
    if (!make_map(&tB2, W2, N, K, K, BN / 2)) return cudaErrorNotSupported;
  } else {
    tB2 = tB;
  }
  auto kern = gemm_pair_kernel<EPI>;
  {
    cudaError_t e = set_smem_limit(kern, (int)SMEM);
    if (e != cudaSuccess) return e;
  }
  const long tiles = (long)((M + 2 * BM - 1) / (2 * BM)) * ((N + OUT_COLS - 1) / OUT_COLS);
  const long pairs = tiles < num_sms() / 2 ? tiles : num_sms() / 2;
  const int esz = EPI == EPI_F32 ? 4 : 2;
  const int vec_ok = ((ldy * esz) % 16 == 0) && (((uintptr_t)Y) % 16 == 0) &&
                     (EPI != EPI_ADD || ((ldr * 2) % 16 == 0 && ((uintptr_t)R) % 16 == 0));
  kern<<<(unsigned)(2 * pairs), 192, SMEM, s>>>(tA, tB, tB2, Y, ldy, (const __nv_bfloat16*)R, ldr, M, N, K, vec_ok,
                                                 ep, fe);
  return cudaGetLastError();
}

}  // namespace p2
}  // namespace tc

cudaError_t linear_pair(const void* X, int ldx, const void* W, const void* W2, const void* R, int ldr, void* Y,
                        int ldy, int M, int N, int K, int epi, cudaStream_t s) {
  switch (epi) {
    case EPI_STORE: return tc::p2::launch<EPI_STORE>(X, ldx, W, W2, R, ldr, Y, ldy, M, N, K, s);
    case EPI_ADD: return tc::p2::launch<EPI_ADD>(X, ldx, W, W2, R, ldr, Y, ldy, M, N, K, s);
    case EPI_SWIGLU: return tc::p2::launch<EPI_SWIGLU>(X, ldx, W, W2, R, ldr, Y, ldy, M, N, K, s);
    case EPI_F32: return tc::p2::launch<EPI_F32>(X, ldx, W, W2, R, ldr, Y, ldy, M, N, K, s);
  }
  return cudaErrorNotSupported;
}

cudaError_t linear_gdn(const void* X, int ldx, const void* W, int M, int K, const GdnEpi& ep, cudaStream_t s) {
  auto al16 = [](const void* p) { return ((uintptr_t)p % 16) == 0; };
  if (M <= 128 || ep.H % 2 != 0 || ep.H > 16 || !al16(X) || !al16(W) || (ldx * 2) % 16 || (K * 2) % 16 ||
      !al16(ep.q) || !al16(ep.k) || !al16(ep.v))
    return cudaErrorNotSupported;
  const int N = 3 * ep.H * 128 + 2 * ep.H;
  return tc::p2::launch<EPI_GDN>(X, ldx, W, nullptr, nullptr, 0, nullptr, 0, M, N, K, s, ep);
}

cudaError_t linear_fa(const void* X, int ldx, const void* W, int M, int K, const FaEpi& fe, cudaStream_t s) {
  auto al16 = [](const void* p) { return ((uintptr_t)p % 16) == 0; };
  if (M <= 128 || fe.T <= 0 || fe.rot < 0 || fe.rot > 64 || fe.rot % 2 || (fe.rot > 0 && !fe.rope) || !al16(X) ||
      !al16(W) || (ldx * 2) % 16 || (K * 2) % 16 || !al16(fe.q) || !al16(fe.gate) || (fe.ld_gate * 2) % 16 ||
      !al16(fe.k_slab) || !al16(fe.v_slab) || !al16(fe.q_gain) || !al16(fe.k_gain))
    return cudaErrorNotSupported;
  const int N = (2 * fe.Hq + 2 * fe.Hkv) * 256;
  return tc::p2::launch<EPI_FA>(X, ldx, W, nullptr, nullptr, 0, nullptr, 0, M, N, K, s, GdnEpi{}, fe);
}

}  // namespace lk
