// bf16 projections Y = X W^T on the 5th-generation tensor cores (sm_100a): dispatch.
//
// The dense contractions of the decoder layer (GDN / FA input and output maps and the
// SwiGLU FFN, "Loop-9B engineering teardown" §二) and the LM head:
//   - M <= 128 rows (decode batches, the last prefill position): gemm_skinny.cu, which
//     streams the weights with the batch as the MMA's N dimension;
//   - more rows (prefill): gemm_tc2.cu, CTA pairs on 256 x 256 tiles (cta_group::2).
// Epilogues: store / + residual / SwiGLU / fp32.
#include "internal.h"
#include "tc_common.cuh"

namespace lk {

constexpr int kSkinnyMaxRows = 128;   // rows up to which the weight-streaming kernel is used

size_t linear_workspace_bytes(int M, int N, int K, int epi) {
  (void)K;
  if (M > kSkinnyMaxRows || M <= 0 || N <= 0) return 0;
  return linear_skinny_workspace_bytes(M, N, epi);
}

cudaError_t linear_tc(const void* X, int ldx, const void* W, const void* W2, const void* R, int ldr, void* Y, int ldy,
                      int M, int N, int K, int epi, cudaStream_t s, void* ws, size_t ws_bytes) {
  if (M == 0 || N == 0) return cudaSuccess;
  // TMA needs 16-byte aligned bases and row strides
  if (((uintptr_t)X) % 16 || ((uintptr_t)W) % 16 || (ldx * 2) % 16 || (K * 2) % 16) return cudaErrorNotSupported;
  if (epi == EPI_SWIGLU && ((uintptr_t)W2) % 16) return cudaErrorNotSupported;
  if (M <= kSkinnyMaxRows) return linear_skinny(X, ldx, W, W2, R, ldr, Y, ldy, M, N, K, epi, s, ws, ws_bytes);
  return linear_pair(X, ldx, W, W2, R, ldr, Y, ldy, M, N, K, epi, s);
}

}  // namespace lk
