// bf16 projection Y = X W^T on the 5th-generation tensor cores (sm_100a).
//
// The dense contractions of the decoder layer (GDN / FA input and output maps and the
// SwiGLU FFN, "Loop-9B engineering teardown" §二) run here.  Design:
//   - persistent kernel, one CTA per SM, tiles of 128 x BN outputs, K in 64-wide slices;
//   - warp 0 issues TMA loads (128-byte swizzle) into a STAGES-deep shared-memory ring;
//   - warp 1 issues tcgen05.mma (M = 128, N = BN, K = 16 per instruction) into one of
//     two TMEM accumulators and frees ring slots with tcgen05.commit;
//   - warps 2-5 drain the other accumulator with tcgen05.ld (one TMEM lane = one output
//     row per thread) and apply the epilogue (store / + residual / SwiGLU / fp32),
//     so the epilogue of tile i overlaps the MMAs of tile i+1;
//   - SwiGLU loads BN/2 rows of W_gate and BN/2 rows of W_up into one BN-row operand,
//     so a single N = BN MMA yields both halves side by side in TMEM.
// Every mbarrier wait is bounded (clock64); a timeout records a device error and the
// kernel unwinds instead of spinning forever.
#include "internal.h"
#include "tc_common.cuh"

namespace lk {
namespace tc {

constexpr int BM = 128, BK = 64;

template <int BN>
struct Cfg {
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES = (192 * 1024) / STAGE_BYTES;
  static constexpr int TMEM_COLS = 2 * BN;           // two accumulators
  static constexpr size_t SMEM = (size_t)STAGES * STAGE_BYTES + 1024 + 256;
};

template <int BN, int EPI>
__global__ void __launch_bounds__(192, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tA, const __grid_constant__ CUtensorMap tB,
                   const __grid_constant__ CUtensorMap tB2, void* __restrict__ Y, int ldy,
                   const __nv_bfloat16* __restrict__ R, int ldr, int M, int N, int K, int vec_ok) {
  using C = Cfg<BN>;
  constexpr int STAGES = C::STAGES;
  constexpr int OUT_COLS = (EPI == EPI_SWIGLU) ? BN / 2 : BN;   // output columns per tile
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint64_t* bars = (uint64_t*)(smem + (size_t)STAGES * C::STAGE_BYTES);
  // bars: full[STAGES], empty[STAGES], tfull[2], tempty[2]
  uint32_t* tmem_slot = (uint32_t*)(bars + 2 * STAGES + 4);
  volatile int* abort_flag = (volatile int*)(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int mb = (M + BM - 1) / BM;
  const int nb = (N + OUT_COLS - 1) / OUT_COLS;
  const int n_tiles = mb * nb;
  const int kb_n = (K + BK - 1) / BK;
  // Tile t -> (m-block, n-block), grouped GROUP_M m-blocks at a time: a wave of CTAs
  // covers a compact block of outputs, so the activation rows of a group stay in L2
  // while every weight column streams past them once per group.
  constexpr int GROUP_M = 16;
  auto tile_mn = [&](int t, int& m0, int& n0) {
    const int per_group = GROUP_M * nb;
    const int grp = t / per_group, first_m = grp * GROUP_M;
    const int gm = min(GROUP_M, mb - first_m);
    const int in = t % per_group;
    m0 = (first_m + in % gm) * BM;
    n0 = (in / gm) * OUT_COLS;
  };
  const uint32_t bar0 = smem_u32(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
  auto tfull_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + a); };
  auto tempty_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + 2 + a); };

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar(a), 1);
      mbar_init(tempty_bar(a), 128);
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"((uint32_t)C::TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (warp == 0 && lane == 0) {
    asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&tA) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&tB) : "memory");
    if (EPI == EPI_SWIGLU) asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&tB2) : "memory");
  }
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      int it = 0;
      for (int t = blockIdx.x; t < n_tiles; t += gridDim.x) {
        int m0, n0;
        tile_mn(t, m0, n0);
        for (int kb = 0; kb < kb_n; ++kb, ++it) {
          const int s = it % STAGES;
          if (!mbar_wait(empty_bar(s), ((it / STAGES) & 1) ^ 1, abort_flag)) goto done;
          const uint32_t a_dst = smem_u32(smem + (size_t)s * C::STAGE_BYTES);
          const uint32_t b_dst = a_dst + C::A_BYTES;
          mbar_expect_tx(full_bar(s), C::STAGE_BYTES);
          tma_load_2d(a_dst, &tA, full_bar(s), kb * BK, m0);
          if (EPI == EPI_SWIGLU) {
            tma_load_2d(b_dst, &tB, full_bar(s), kb * BK, n0);
            tma_load_2d(b_dst + (BN / 2) * BK * 2, &tB2, full_bar(s), kb * BK, n0);
          } else {
            tma_load_2d(b_dst, &tB, full_bar(s), kb * BK, n0);
          }
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(BM, BN);
      int it = 0, local = 0;
      for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, ++local) {
        const int acc = local & 1;
        if (!mbar_wait(tempty_bar(acc), ((local >> 1) & 1) ^ 1, abort_flag)) goto done;
        fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
        for (int kb = 0; kb < kb_n; ++kb, ++it) {
          const int s = it % STAGES;
          if (!mbar_wait(full_bar(s), (it / STAGES) & 1, abort_flag)) goto done;
          fence_after();
          const uint32_t a_addr = smem_u32(smem + (size_t)s * C::STAGE_BYTES);
          const uint32_t b_addr = a_addr + C::A_BYTES;
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)
            mma_bf16(d_tmem, sw128_desc(a_addr + k * 32), sw128_desc(b_addr + k * 32), idesc,
                     (kb > 0 || k > 0) ? 1u : 0u);
          mma_commit(empty_bar(s));          // ring slot is free once these MMAs have read it
        }
        mma_commit(tfull_bar(acc));          // accumulator ready for the epilogue
      }
    }
  } else {
    // ---------------------------------------------------------------- epilogue (warps 2..5)
    const int quarter = warp & 3;                 // TMEM lanes 32*quarter .. +31
    int local = 0;
    for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, ++local) {
      const int acc = local & 1;
      int m0, n0;
      tile_mn(t, m0, n0);
      if (!mbar_wait(tfull_bar(acc), (local >> 1) & 1, abort_flag)) goto done;
      fence_after();
      const int row = m0 + quarter * 32 + lane;
      const uint32_t t_row = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * BN);
#pragma unroll 1
      for (int c = 0; c < OUT_COLS / 32; ++c) {
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
      mbar_arrive(tempty_bar(acc));
    }
  }
done:
  __syncthreads();
  if (warp == 1) {
    fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"((uint32_t)C::TMEM_COLS)
                 : "memory");
  }
}

template <int BN, int EPI>
static cudaError_t launch(const void* X, int ldx, const void* W, const void* W2, const void* R, int ldr, void* Y,
                          int ldy, int M, int N, int K, cudaStream_t s) {
  using C = Cfg<BN>;
  constexpr int OUT_COLS = (EPI == EPI_SWIGLU) ? BN / 2 : BN;
  constexpr int B_ROWS = (EPI == EPI_SWIGLU) ? BN / 2 : BN;
  CUtensorMap tA, tB, tB2;
  if (!make_map(&tA, X, M, K, ldx, BM)) return cudaErrorNotSupported;
  if (!make_map(&tB, W, N, K, K, B_ROWS)) return cudaErrorNotSupported;
  if (EPI == EPI_SWIGLU) {
    if (!make_map(&tB2, W2, N, K, K, B_ROWS)) return cudaErrorNotSupported;
  } else {
    tB2 = tB;
  }
  auto kern = gemm_tc_kernel<BN, EPI>;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::SMEM);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  const long tiles = (long)((M + BM - 1) / BM) * ((N + OUT_COLS - 1) / OUT_COLS);
  const int esz = EPI == EPI_F32 ? 4 : 2;
  const int vec_ok = ((ldy * esz) % 16 == 0) && (((uintptr_t)Y) % 16 == 0) &&
                     (EPI != EPI_ADD || ((ldr * 2) % 16 == 0 && ((uintptr_t)R) % 16 == 0));
  const int grid = (int)(tiles < num_sms() ? tiles : num_sms());
  kern<<<grid, 192, C::SMEM, s>>>(tA, tB, tB2, Y, ldy, (const __nv_bfloat16*)R, ldr, M, N, K, vec_ok);
  return cudaGetLastError();
}

}  // namespace tc

size_t linear_workspace_bytes(int M, int N, int K, int epi) {
  (void)K;
  if (M > tc::BM || M <= 0 || N <= 0) return 0;
  return linear_skinny_workspace_bytes(M, N, epi);
}

cudaError_t linear_tc(const void* X, int ldx, const void* W, const void* W2, const void* R, int ldr, void* Y, int ldy,
                      int M, int N, int K, int epi, cudaStream_t s, void* ws, size_t ws_bytes) {
  if (M == 0 || N == 0) return cudaSuccess;
  // TMA needs 16-byte aligned bases and row strides
  if (((uintptr_t)X) % 16 || ((uintptr_t)W) % 16 || (ldx * 2) % 16 || (K * 2) % 16) return cudaErrorNotSupported;
  if (epi == EPI_SWIGLU && ((uintptr_t)W2) % 16) return cudaErrorNotSupported;
  if (M <= tc::BM) return linear_skinny(X, ldx, W, W2, R, ldr, Y, ldy, M, N, K, epi, s, ws, ws_bytes);
  switch (epi) {
    case EPI_STORE: return tc::launch<256, EPI_STORE>(X, ldx, W, W2, R, ldr, Y, ldy, M, N, K, s);
    case EPI_ADD: return tc::launch<256, EPI_ADD>(X, ldx, W, W2, R, ldr, Y, ldy, M, N, K, s);
    case EPI_SWIGLU: return tc::launch<256, EPI_SWIGLU>(X, ldx, W, W2, R, ldr, Y, ldy, M, N, K, s);
    case EPI_F32: return tc::launch<256, EPI_F32>(X, ldx, W, W2, R, ldr, Y, ldy, M, N, K, s);
  }
  return cudaErrorNotSupported;
}

}  // namespace lk
