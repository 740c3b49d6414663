// Projections with few rows, Y[M, N] = X[M, K] W[N, K]^T with M <= 128, on tcgen05.
//
// These are the decode-time projections of the decoder layer ("Loop-9B engineering
// teardown" §二: the 56 executions stream every projection weight once per decode step,
// §四) and the LM head on the last prefill position.  With M <= 128 the work is a
// stream of the weight matrix through the SMs, so the kernel is built around that:
//   - swap-AB: a tile is 128 weight rows (the MMA's M) x NB batch rows (the MMA's N,
//     NB in {16, 32, 64, 128} >= M), so no MMA row is spent on padding tokens;
//   - the k-block iterations of all tiles, n_tiles x ceil(K/64), are divided evenly
//     over <= one CTA per SM; a CTA's range may start and end inside a tile;
//   - a tile that one CTA covers whole gets its epilogue straight from TMEM; a tile
//     split between CTAs is summed with red.global.add.f32 into a zero-filled fp32
//     buffer, and the CTA whose part completes the tile (per-tile counter) applies the
//     epilogue and re-zeros its slice of the buffer: one launch, and no CTA ever waits
//     on another;
//   - SwiGLU tiles carry the same 128 rows of W_gate and W_up as two MMAs into two
//     TMEM accumulators, so a thread holds the gate and up value of its output column;
//   - programmatic dependent launch: the weight tiles of the first ring stages are
//     requested before griddepcontrol.wait, so they stream in while the kernel that
//     produces X is still finishing.
// Warp roles as in the large-M kernel: warp 0 TMA, warp 1 MMA issue, warps 2-5 the
// epilogue.  Every mbarrier wait is bounded (clock64).
#include "internal.h"
#include "tc_common.cuh"

namespace lk {
namespace tc {
namespace sk {

constexpr int BW = 128;     // weight rows per tile (MMA M)
constexpr int BK = 64;      // K per stage (one 128-byte swizzle row of bf16)
constexpr int MIN_KB = 8;   // fewest k-blocks a CTA is given (fewer only adds partial sums)

template <int NB, int NMAT>
struct Cfg {
  static constexpr int A_BYTES = BW * BK * 2;                     // one weight matrix
  static constexpr int B_BYTES = NB * BK * 2;                     // the activations
  static constexpr int STAGE_BYTES = NMAT * A_BYTES + B_BYTES;
  static constexpr int ACC_COLS = NMAT * NB;                      // one accumulator
  static constexpr int TMEM_COLS = 2 * ACC_COLS;                  // double-buffered (power of two >= 32)
  // two CTAs per SM when their accumulators fit TMEM together: one CTA's ramp and
  // split-tile tail then overlap the other's streaming
  static constexpr int PER_SM = TMEM_COLS <= 256 ? 2 : 1;
  static constexpr int STAGES_FIT = (200 * 1024 / PER_SM) / STAGE_BYTES;
  static constexpr int STAGES = STAGES_FIT > 10 ? 10 : STAGES_FIT;
  static constexpr size_t SMEM = (size_t)STAGES * STAGE_BYTES + 1024 + 256;
  static_assert(STAGE_BYTES % 1024 == 0, "stages must keep 1024-byte swizzle alignment");
  static_assert(TMEM_COLS >= 32 && TMEM_COLS <= 512 && (TMEM_COLS & (TMEM_COLS - 1)) == 0, "TMEM allocation");
};

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void red_add4(float* p, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a), "f"(b), "f"(c), "f"(d) : "memory");
}
__device__ __forceinline__ void epi_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Outputs (b0 + j, n), j < CW and b0 + j < M, from their fp32 sums g (and u for SwiGLU).
// All residual loads are issued before the first store: R may be Y itself.
template <int EPI, int CW>
__device__ __forceinline__ void put_chunk(void* Y, int ldy, const __nv_bfloat16* R, int ldr, int b0, int M, int n,
                                          const float* g, const float* u) {
  float v[CW];
#pragma unroll
  for (int j = 0; j < CW; ++j) {
    v[j] = g[j];
    if (EPI == EPI_SWIGLU) v[j] = g[j] / (1.f + expf(-g[j])) * u[j];
  }
  if (EPI == EPI_ADD) {
    float r[CW];
#pragma unroll
    for (int j = 0; j < CW; ++j) r[j] = b0 + j < M ? __bfloat162float(R[(long)(b0 + j) * ldr + n]) : 0.f;
#pragma unroll
    for (int j = 0; j < CW; ++j) v[j] += r[j];
  }
#pragma unroll
  for (int j = 0; j < CW; ++j) {
    if (b0 + j >= M) break;
    if (EPI == EPI_F32)
      reinterpret_cast<float*>(Y)[(long)(b0 + j) * ldy + n] = v[j];
    else
      reinterpret_cast<__nv_bfloat16*>(Y)[(long)(b0 + j) * ldy + n] = __float2bfloat16(v[j]);
  }
}

template <int NB, int NMAT, int EPI>
__global__ void __launch_bounds__(192, Cfg<NB, NMAT>::PER_SM)
    gemm_skinny_kernel(const __grid_constant__ CUtensorMap tW, const __grid_constant__ CUtensorMap tW2,
                       const __grid_constant__ CUtensorMap tX, void* __restrict__ Y, int ldy,
                       const __nv_bfloat16* R, int ldr, int M, int N, int K, int whole_tiles,
                       float* __restrict__ acc_ws, int* __restrict__ cnt_ws) {
  using C = Cfg<NB, NMAT>;
  constexpr int STAGES = C::STAGES;
  constexpr int CW = NB < 32 ? NB : 32;            // TMEM columns per tcgen05.ld
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint64_t* bars = (uint64_t*)(smem + (size_t)STAGES * C::STAGE_BYTES);
  // bars: full[STAGES], empty[STAGES], tfull[2], tempty[2]
  uint32_t* tmem_slot = (uint32_t*)(bars + 2 * STAGES + 4);
  volatile int* abort_flag = (volatile int*)(tmem_slot + 1);
  volatile int* last_flag = (volatile int*)(tmem_slot + 2);

  griddep_launch();   // the next kernel may start its own prologue on SMs this grid frees
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_tiles = (N + BW - 1) / BW;
  const int kb_n = (K + BK - 1) / BK;
  // this CTA's range of (tile, k-block) iterations; whole_tiles != 0 keeps ranges on
  // whole tiles (no partial-sum buffer)
  long lo, hi;
  if (whole_tiles) {
    lo = (long)blockIdx.x * n_tiles / gridDim.x * kb_n;
    hi = (long)(blockIdx.x + 1) * n_tiles / gridDim.x * kb_n;
  } else {
    const long I = (long)n_tiles * kb_n;
    lo = (long)blockIdx.x * I / gridDim.x;
    hi = (long)(blockIdx.x + 1) * I / gridDim.x;
  }
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
  if (warp == 1) tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
  if (warp == 0 && lane == 0) {
    asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&tW) : "memory");
    if (NMAT == 2) asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&tW2) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&tX) : "memory");
  }
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      // weights of the first stages first: they do not depend on the previous kernel
      const long pre = min((long)STAGES, hi - lo);
      for (long q = 0; q < pre; ++q) {
        const long it = lo + q;
        const int t = (int)(it / kb_n), kb = (int)(it % kb_n);
        const uint32_t a_dst = smem_u32(smem + (size_t)q * C::STAGE_BYTES);
        mbar_expect_tx(full_bar((int)q), C::STAGE_BYTES);
        tma_load_2d(a_dst, &tW, full_bar((int)q), kb * BK, t * BW);
        if (NMAT == 2) tma_load_2d(a_dst + C::A_BYTES, &tW2, full_bar((int)q), kb * BK, t * BW);
      }
      griddep_wait();     // X (and R, Y) belong to the previous kernels from here on
      for (long q = 0; q < pre; ++q) {
        const int kb = (int)((lo + q) % kb_n);
        const uint32_t b_dst = smem_u32(smem + (size_t)q * C::STAGE_BYTES) + NMAT * C::A_BYTES;
        tma_load_2d(b_dst, &tX, full_bar((int)q), kb * BK, 0);
      }
      for (long q = pre; q < hi - lo; ++q) {
        const long it = lo + q;
        const int t = (int)(it / kb_n), kb = (int)(it % kb_n);
        const int s = (int)(q % STAGES);
        if (!mbar_wait(empty_bar(s), (uint32_t)(((q / STAGES) & 1) ^ 1), abort_flag)) goto done;
        const uint32_t a_dst = smem_u32(smem + (size_t)s * C::STAGE_BYTES);
        mbar_expect_tx(full_bar(s), C::STAGE_BYTES);
        tma_load_2d(a_dst, &tW, full_bar(s), kb * BK, t * BW);
        if (NMAT == 2) tma_load_2d(a_dst + C::A_BYTES, &tW2, full_bar(s), kb * BK, t * BW);
        tma_load_2d(a_dst + NMAT * C::A_BYTES, &tX, full_bar(s), kb * BK, 0);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(BW, NB);
      long q = 0;
      int seg = 0;
      for (long it = lo; it < hi; ++seg) {
        const int kb0 = (int)(it % kb_n);
        const int kb1 = (int)min((long)kb_n, kb0 + (hi - it));
        const int acc = seg & 1;
        if (!mbar_wait(tempty_bar(acc), (uint32_t)(((seg >> 1) & 1) ^ 1), abort_flag)) goto done;
        fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * C::ACC_COLS);
        for (int kb = kb0; kb < kb1; ++kb, ++q) {
          const int s = (int)(q % STAGES);
          if (!mbar_wait(full_bar(s), (uint32_t)((q / STAGES) & 1), abort_flag)) goto done;
          fence_after();
          const uint32_t a_addr = smem_u32(smem + (size_t)s * C::STAGE_BYTES);
          const uint32_t b_addr = a_addr + NMAT * C::A_BYTES;
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)
#pragma unroll
            for (int mat = 0; mat < NMAT; ++mat)
              mma_bf16(d_tmem + mat * NB, sw128_desc(a_addr + mat * C::A_BYTES + k * 32), sw128_desc(b_addr + k * 32),
                       idesc, (kb > kb0 || k > 0) ? 1u : 0u);
          mma_commit(empty_bar(s));
        }
        mma_commit(tfull_bar(acc));
        it += kb1 - kb0;
      }
    }
  } else {
    // ---------------------------------------------------------------- epilogue (warps 2..5)
    const int quarter = warp & 3;                       // TMEM lanes 32*quarter .. +31
    const int et = threadIdx.x - 64;                    // 0..127
    griddep_wait();                                     // R, Y and the sums belong to earlier kernels
    int seg = 0;
    for (long it = lo; it < hi; ++seg) {
      const int t = (int)(it / kb_n);
      const int kb0 = (int)(it % kb_n);
      const int kb1 = (int)min((long)kb_n, kb0 + (hi - it));
      it += kb1 - kb0;
      const bool whole = kb0 == 0 && kb1 == kb_n;
      const int acc = seg & 1;
      if (!mbar_wait(tfull_bar(acc), (uint32_t)((seg >> 1) & 1), abort_flag)) goto done;
      fence_after();
      const int n = t * BW + quarter * 32 + lane;       // this thread's output column
      const uint32_t t_row = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * C::ACC_COLS);
      // partial sums: [M4 / 4][N][4] fp32 per matrix (4 batch rows of a column are one
      // 16-byte vector, so a warp's vector reductions cover 512 contiguous bytes)
      const int M4 = (M + 3) & ~3;
      float* ws_g = acc_ws;
      float* ws_u = acc_ws + (long)M4 * N;
#pragma unroll 1
      for (int c = 0; c < NB / CW; ++c) {
        uint32_t g[CW], u[CW];
        if constexpr (CW == 32) {
          tmem_ld32(t_row + c * CW, g);
          if (NMAT == 2) tmem_ld32(t_row + NB + c * CW, u);
        } else {
          tmem_ld16(t_row + c * CW, g);
          if (NMAT == 2) tmem_ld16(t_row + NB + c * CW, u);
        }
        tmem_wait_ld();
        if (n >= N || c * CW >= M) continue;
        float gf[CW], uf[CW];
#pragma unroll
        for (int j = 0; j < CW; ++j) {
          gf[j] = __uint_as_float(g[j]);
          uf[j] = NMAT == 2 ? __uint_as_float(u[j]) : 0.f;
        }
        if (whole) {
#pragma unroll
          for (int h = 0; h < CW; h += 16) put_chunk<EPI, 16>(Y, ldy, R, ldr, c * CW + h, M, n, gf + h, uf + h);
        } else {
#pragma unroll
          for (int j = 0; j < CW; j += 4) {
            const int b = c * CW + j;
            if (b >= M) break;
            const long o = ((long)(b >> 2) * N + n) * 4;
            red_add4(ws_g + o, gf[j], gf[j + 1], gf[j + 2], gf[j + 3]);
            if (NMAT == 2) red_add4(ws_u + o, uf[j], uf[j + 1], uf[j + 2], uf[j + 3]);
          }
        }
      }
      fence_before();
      mbar_arrive(tempty_bar(acc));                     // accumulator free for the MMA warp
      if (whole) continue;
      // partial tile: the CTA that completes the tile's k-range applies the epilogue
      __threadfence();
      epi_bar();
      if (et == 0) {
        const int add = kb1 - kb0;
        const int old = atomicAdd(cnt_ws + t, add);
        *last_flag = (old + add == kb_n) ? 1 : 0;
      }
      epi_bar();
      if (*last_flag) {
        __threadfence();
        if (n < N) {
          // 32 batch rows per round: their sums (and residuals) are all loaded before
          // anything is stored, so M = 64 costs two round trips to L2
#pragma unroll 1
          for (int b0 = 0; b0 < M; b0 += 32) {
            float gf[32], uf[32], rf[32];
#pragma unroll
            for (int j = 0; j < 32; j += 4) {
              float4 a = make_float4(0.f, 0.f, 0.f, 0.f), c4 = a;
              if (b0 + j < M) {
                const long o = ((long)((b0 + j) >> 2) * N + n) * 4;
                a = __ldcg(reinterpret_cast<const float4*>(ws_g + o));
                if (NMAT == 2) c4 = __ldcg(reinterpret_cast<const float4*>(ws_u + o));
              }
              gf[j] = a.x, gf[j + 1] = a.y, gf[j + 2] = a.z, gf[j + 3] = a.w;
              uf[j] = c4.x, uf[j + 1] = c4.y, uf[j + 2] = c4.z, uf[j + 3] = c4.w;
            }
            if (EPI == EPI_ADD) {
#pragma unroll
              for (int j = 0; j < 32; ++j) rf[j] = b0 + j < M ? __bfloat162float(R[(long)(b0 + j) * ldr + n]) : 0.f;
#pragma unroll
              for (int j = 0; j < 32; ++j) gf[j] += rf[j];
            }
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              if (b0 + j >= M) break;
              float v = gf[j];
              if (EPI == EPI_SWIGLU) v = v / (1.f + expf(-v)) * uf[j];
              if (EPI == EPI_F32)
                reinterpret_cast<float*>(Y)[(long)(b0 + j) * ldy + n] = v;
              else
                reinterpret_cast<__nv_bfloat16*>(Y)[(long)(b0 + j) * ldy + n] = __float2bfloat16(v);
            }
#pragma unroll
            for (int j = 0; j < 32; j += 4) {
              if (b0 + j >= M) break;
              const long o = ((long)((b0 + j) >> 2) * N + n) * 4;
              __stcg(reinterpret_cast<float4*>(ws_g + o), make_float4(0.f, 0.f, 0.f, 0.f));
              if (NMAT == 2) __stcg(reinterpret_cast<float4*>(ws_u + o), make_float4(0.f, 0.f, 0.f, 0.f));
            }
          }
        }
        if (et == 0) cnt_ws[t] = 0;
      }
      epi_bar();                                        // everyone has read last_flag
    }
  }
done:
  __syncthreads();
  if (warp == 1) {
    fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

// Bytes of the partial-sum buffer: per-tile counters (padded to 256 B), then
// NMAT x [ceil(M/4), N, 4] fp32 sums.
static size_t ws_bytes_for(int M, int N, int epi) {
  const long n_tiles = (N + BW - 1) / BW;
  const long nmat = epi == EPI_SWIGLU ? 2 : 1;
  const long m4 = (M + 3) & ~3;
  return (size_t)((n_tiles * 4 + 255) / 256 * 256) + (size_t)nmat * m4 * N * 4;
}

template <int NB, int EPI>
static cudaError_t launch(const void* X, int ldx, const void* W, const void* W2, const void* R, int ldr, void* Y,
                          int ldy, int M, int N, int K, cudaStream_t s, void* ws, size_t ws_bytes) {
  constexpr int NMAT = EPI == EPI_SWIGLU ? 2 : 1;
  using C = Cfg<NB, NMAT>;
  CUtensorMap tW, tW2, tX;
  if (!make_map(&tW, W, N, K, K, BW)) return cudaErrorNotSupported;
  if (NMAT == 2) {
    if (!make_map(&tW2, W2, N, K, K, BW)) return cudaErrorNotSupported;
  } else {
    tW2 = tW;
  }
  if (!make_map(&tX, X, M, K, ldx, NB)) return cudaErrorNotSupported;
  auto kern = gemm_skinny_kernel<NB, NMAT, EPI>;
  {
    cudaError_t e = set_smem_limit(kern, (int)C::SMEM);
    if (e != cudaSuccess) return e;
  }
  const long n_tiles = (N + BW - 1) / BW, kb_n = (K + BK - 1) / BK;
  const bool split = ws != nullptr && ((uintptr_t)ws % 16) == 0 && ws_bytes >= ws_bytes_for(M, N, EPI);
  long grid;
  int whole_tiles = 0;
  if (split) {
    grid = (n_tiles * kb_n + MIN_KB - 1) / MIN_KB;
  } else {
    grid = n_tiles;
    whole_tiles = 1;
  }
  if (grid > (long)C::PER_SM * num_sms()) grid = (long)C::PER_SM * num_sms();
  int* cnt = split ? (int*)ws : nullptr;
  float* acc = split ? (float*)((char*)ws + (ws_bytes_for(M, N, EPI) - (size_t)NMAT * ((M + 3) & ~3) * N * 4))
                     : nullptr;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(192);
  cfg.dynamicSmemBytes = C::SMEM;
  cfg.stream = s;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, tW, tW2, tX, Y, ldy, (const __nv_bfloat16*)R, ldr, M, N, K, whole_tiles, acc,
                            cnt);
}

template <int EPI>
static cudaError_t dispatch(const void* X, int ldx, const void* W, const void* W2, const void* R, int ldr, void* Y,
                            int ldy, int M, int N, int K, cudaStream_t s, void* ws, size_t ws_bytes) {
  if (M <= 16) return launch<16, EPI>(X, ldx, W, W2, R, ldr, Y, ldy, M, N, K, s, ws, ws_bytes);
  if (M <= 32) return launch<32, EPI>(X, ldx, W, W2, R, ldr, Y, ldy, M, N, K, s, ws, ws_bytes);
  if (M <= 64) return launch<64, EPI>(X, ldx, W, W2, R, ldr, Y, ldy, M, N, K, s, ws, ws_bytes);
  return launch<128, EPI>(X, ldx, W, W2, R, ldr, Y, ldy, M, N, K, s, ws, ws_bytes);
}

}  // namespace sk
}  // namespace tc

size_t linear_skinny_workspace_bytes(int M, int N, int epi) { return tc::sk::ws_bytes_for(M, N, epi); }

cudaError_t linear_skinny(const void* X, int ldx, const void* W, const void* W2, const void* R, int ldr, void* Y,
                          int ldy, int M, int N, int K, int epi, cudaStream_t s, void* ws, size_t ws_bytes) {
  using namespace tc::sk;
  switch (epi) {
    case EPI_STORE: return dispatch<EPI_STORE>(X, ldx, W, W2, R, ldr, Y, ldy, M, N, K, s, ws, ws_bytes);
    case EPI_ADD: return dispatch<EPI_ADD>(X, ldx, W, W2, R, ldr, Y, ldy, M, N, K, s, ws, ws_bytes);
    case EPI_SWIGLU: return dispatch<EPI_SWIGLU>(X, ldx, W, W2, R, ldr, Y, ldy, M, N, K, s, ws, ws_bytes);
    case EPI_F32: return dispatch<EPI_F32>(X, ldx, W, W2, R, ldr, Y, ldy, M, N, K, s, ws, ws_bytes);
  }
  return cudaErrorNotSupported;
}

}  // namespace lk
