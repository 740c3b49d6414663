// FP32-arithmetic SIMT projection Y = X W^T with fused epilogues.  This is the
// precision path for fp32 models (tcgen05 has no fp32 MMA); bf16 projections go
// to the tcgen05 kernels (gemm_tc.cu dispatch).  64x64 output tile, 16-deep K slices
// staged transposed in shared memory, 4x4 outputs per thread.
#include "common.cuh"
#include "internal.h"

namespace lk {

template <typename T, int EPI>
__global__ void __launch_bounds__(256) gemm_simt_kernel(const T* __restrict__ X, int ldx, const T* __restrict__ W,
                                                        const T* __restrict__ W2, const T* R, int ldr, void* Y,
                                                        int ldy, int M, int N, int K) {
  constexpr int BM = 64, BN = 64, BK = 16, PAD = 4;
  __shared__ float Xs[BK][BM + PAD], Ws[BK][BN + PAD], W2s[EPI == EPI_SWIGLU ? BK : 1][BN + PAD];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
  float acc[4][4], acc2[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = acc2[i][j] = 0.f;
  for (int k0 = 0; k0 < K; k0 += BK) {
    for (int i = threadIdx.x; i < BM * BK; i += 256) {
      const int r = i / BK, kk = i % BK;
      const bool kin = k0 + kk < K;
      Xs[kk][r] = (m0 + r < M && kin) ? ldf(X + (long)(m0 + r) * ldx + k0 + kk) : 0.f;
      Ws[kk][r] = (n0 + r < N && kin) ? ldf(W + (long)(n0 + r) * K + k0 + kk) : 0.f;
      if (EPI == EPI_SWIGLU) W2s[kk][r] = (n0 + r < N && kin) ? ldf(W2 + (long)(n0 + r) * K + k0 + kk) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < BK; ++kk) {
      float a[4], b[4], b2[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) { a[i] = Xs[kk][ty * 4 + i]; b[i] = Ws[kk][tx * 4 + i]; }
      if (EPI == EPI_SWIGLU) {
#pragma unroll
        for (int i = 0; i < 4; ++i) b2[i] = W2s[kk][tx * 4 + i];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
          if (EPI == EPI_SWIGLU) acc2[i][j] = fmaf(a[i], b2[j], acc2[i][j]);
        }
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + ty * 4 + i;
    if (m >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n >= N) continue;
      const long o = (long)m * ldy + n;
      if (EPI == EPI_F32) {
        reinterpret_cast<float*>(Y)[o] = acc[i][j];
      } else {
        float v = acc[i][j];
        if (EPI == EPI_ADD) v += ldf(R + (long)m * ldr + n);
        if (EPI == EPI_SWIGLU) v = v * sigmoidf_acc(v) * acc2[i][j];
        stf(reinterpret_cast<T*>(Y) + o, v);
      }
    }
  }
}

cudaError_t linear_simt(const void* X, int ldx, const void* W, const void* W2, const void* R,
                        int ldr, void* Y, int ldy, int M, int N, int K, int epi, int dtype,
                        cudaStream_t s) {
  if (M == 0 || N == 0) return cudaSuccess;
  dim3 grid((N + 63) / 64, (M + 63) / 64);
#define G(TT, E) gemm_simt_kernel<TT, E><<<grid, 256, 0, s>>>((const TT*)X, ldx, (const TT*)W, (const TT*)W2, \
                                                              (const TT*)R, ldr, Y, ldy, M, N, K)
  if (dtype == BF16) {
    switch (epi) {
      case EPI_STORE: G(__nv_bfloat16, EPI_STORE); break;
      case EPI_ADD: G(__nv_bfloat16, EPI_ADD); break;
      case EPI_SWIGLU: G(__nv_bfloat16, EPI_SWIGLU); break;
      default: G(__nv_bfloat16, EPI_F32); break;
    }
  } else {
    switch (epi) {
      case EPI_STORE: G(float, EPI_STORE); break;
      case EPI_ADD: G(float, EPI_ADD); break;
      case EPI_SWIGLU: G(float, EPI_SWIGLU); break;
      default: G(float, EPI_F32); break;
    }
  }
#undef G
  return cudaGetLastError();
}

cudaError_t linear(const void* X, int ldx, const void* W, const void* W2, const void* R, int ldr,
                   void* Y, int ldy, int M, int N, int K, int epi, int dtype, cudaStream_t s, void* ws,
                   size_t ws_bytes) {
  // bf16 runs on the tensor cores only: a shape or alignment the tcgen05 kernels do not
  // take is an error (cudaErrorNotSupported), never a silent detour to the FP32 SIMT kernel.
  if (dtype == BF16) return linear_tc(X, ldx, W, W2, R, ldr, Y, ldy, M, N, K, epi, s, ws, ws_bytes);
  return linear_simt(X, ldx, W, W2, R, ldr, Y, ldy, M, N, K, epi, dtype, s);
}

}  // namespace lk
