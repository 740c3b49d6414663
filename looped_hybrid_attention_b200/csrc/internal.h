// Internal launchers shared by the C-ABI layer and the model runtime.
#pragma once
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace lk {

enum Dtype { F32 = 0, BF16 = 1 };
enum Epilogue { EPI_STORE = 0, EPI_ADD = 1, EPI_SWIGLU = 2, EPI_F32 = 3, EPI_GDN = 4, EPI_FA = 5 };

// Outputs of the GDN input projection's fused epilogue (EPI_GDN): q, k L2-normalised per head,
// v, and the gates g = -softplus(a + a_bias), beta = sigmoid(b + b_bias), from the columns
// q | k | v | a | b of the product (what gdn_prep computes from the stored projection).
struct GdnEpi {
  void *q, *k, *v;          // [M, H, 128] bf16
  float *g, *beta;          // [M, H] fp32
  const float *a_bias, *b_bias;
  float eps;
  int H;
};
// The projection with the GDN preparation in its epilogue (bf16, M > 128, dk = dv = 128,
// H even); cudaErrorNotSupported otherwise.
cudaError_t linear_gdn(const void* X, int ldx, const void* W, int M, int K, const GdnEpi& ep, cudaStream_t s);

// Outputs of the FA input projection's fused epilogue (EPI_FA), from the columns
// q | gate | k | v of the product (head dim 256): each q and k head RMS-normalised over its
// 256 dims (eps inside the root), scaled by its gain and rotated on dims [0, rot) in
// adjacent pairs by the position's (cos, sin) -- what fa_prep computes; q goes to a compact
// buffer, k and v straight into the execution's slabs at their positions, the gate block
// to its place in `gate` (row stride ld_gate).
struct FaEpi {
  void* q;                       // [M, Hq, 256] bf16
  void* gate;                    // gate block of row m at gate + m * ld_gate
  int ld_gate;
  void *k_slab, *v_slab;         // [B, Hkv, kv_cap, 256] bf16
  int kv_cap;
  const void *q_gain, *k_gain;   // [256] bf16
  float eps;
  int Hq, Hkv, rot;              // rot <= 64
  const float2* rope;            // [T, rot / 2] (cos, sin) of positions pos0 .. pos0 + T - 1
  int T, pos0;                   // tokens per sequence (row m = b * T + t), position of t = 0
};
// The FA input projection with QK-norm, rotary and the KV write in its epilogue (bf16,
// M > 128, head dim 256); cudaErrorNotSupported otherwise.
cudaError_t linear_fa(const void* X, int ldx, const void* W, int M, int K, const FaEpi& fe, cudaStream_t s);
enum MhcMode { MHC_OPEN = 0, MHC_MIX = 1, MHC_ROUTE = 2, MHC_MERGE = 3 };

// ldx: row stride of x in elements (0 = d); r, sum_out and y are dense [M, d].
cudaError_t rmsnorm(const void* x, const void* r, void* sum_out, const void* w, void* y, int M,
                    int d, float eps, int dtype, cudaStream_t s, long ldx = 0);
cudaError_t embed(const int32_t* ids, const void* E, void* out, int M, int d, int vocab, int dtype,
                  cudaStream_t s);
cudaError_t argmax(const float* logits, int32_t* next, int B, int V, cudaStream_t s);

// ws / ws_bytes: optional zero-filled scratch for M <= 128 (linear_workspace_bytes): tiles
// split between CTAs are summed there; each call leaves it zero-filled again.
cudaError_t linear(const void* X, int ldx, const void* W, const void* W2, const void* R, int ldr,
                   void* Y, int ldy, int M, int N, int K, int epi, int dtype, cudaStream_t s, void* ws = nullptr,
                   size_t ws_bytes = 0);
// tcgen05 path (bf16); returns cudaErrorNotSupported for shapes it does not take.
cudaError_t linear_tc(const void* X, int ldx, const void* W, const void* W2, const void* R, int ldr,
                      void* Y, int ldy, int M, int N, int K, int epi, cudaStream_t s, void* ws = nullptr,
                      size_t ws_bytes = 0);
size_t linear_workspace_bytes(int M, int N, int K, int epi);
// M <= 128 (decode batches, the last prefill position): weight-streaming tcgen05 kernel.
cudaError_t linear_skinny(const void* X, int ldx, const void* W, const void* W2, const void* R, int ldr,
                          void* Y, int ldy, int M, int N, int K, int epi, cudaStream_t s, void* ws,
                          size_t ws_bytes);
size_t linear_skinny_workspace_bytes(int M, int N, int epi);
// M > 128 (prefill): CTA pairs, 256 x 256 tiles (tcgen05 cta_group::2).
cudaError_t linear_pair(const void* X, int ldx, const void* W, const void* W2, const void* R, int ldr, void* Y,
                        int ldy, int M, int N, int K, int epi, cudaStream_t s);
cudaError_t linear_simt(const void* X, int ldx, const void* W, const void* W2, const void* R,
                        int ldr, void* Y, int ldy, int M, int N, int K, int epi, int dtype,
                        cudaStream_t s);

cudaError_t gdn_prep(const void* P, int ld_p, const float* a_bias, const float* b_bias, void* q,
                     void* k, void* v, float* g, float* beta, int M, int H, int dk, int dv,
                     float eps, int dtype, cudaStream_t s);
// workspace: gdn_workspace_bytes(...) of device scratch for the two-pass scan, or NULL
// for the single-pass kernel (no scratch, slower).
cudaError_t gdn_chunk(const void* q, const void* k, const void* v, const float* g,
                      const float* beta, float* state, void* out, int B, int T, int H, int dk,
                      int dv, float scale, int dtype, cudaStream_t s, void* workspace = nullptr);
size_t gdn_workspace_bytes(int B, int T, int H, int dk, int dv);
cudaError_t gdn_step(const void* q, const void* k, const void* v, const float* g, const float* beta,
                     float* state, void* out, int B, int H, int dk, int dv, float scale, int dtype,
                     cudaStream_t s);
// Decode step from the stored input projection (q | k | v | a | b rows): the GDN preparation
// (L2 norms, gates) happens inside the step.
cudaError_t gdn_step_proj(const void* P, int ld_p, const float* a_bias, const float* b_bias, float eps, float* state,
                          void* out, int B, int H, int dk, int dv, float scale, int dtype, cudaStream_t s);
bool gdn_supported(int dk, int dv);
// GDN variant (short causal conv + gated output norm; Hv value heads reading Hk key heads)
bool gdn_variant_supported(int Hk, int Hv, int dk, int dv, int conv);
// conv + SiLU on the q|k|v channels of P (rows q | k | v | z | a | b), L2 norm of q and k
// (written once per value head that reads them), gates; then conv_state [B][conv-1][C]
// becomes the last conv-1 inputs.  q, k [B*T, Hv, dk], v [B*T, Hv, dv], g, beta [B*T, Hv].
cudaError_t gdn_conv_prep(const void* P, int ld_p, const void* conv_w, void* conv_state, const float* a_bias,
                          const float* b_bias, void* q, void* k, void* v, float* g, float* beta, int B, int T, int Hk,
                          int Hv, int dk, int dv, int conv, float eps, int dtype, cudaStream_t s);
// y [M, H, dv] = RMSNorm(o) * w * silu(z) per head (y may equal o); z rows of stride ld_z.
cudaError_t gdn_gated_norm(const void* o, const void* z, int ld_z, const void* w, void* y, long M, int H, int dv,
                           float eps, int dtype, cudaStream_t s);

// rope_tab: optional [T, rotary_dims/2] (cos, sin) table from rope_table (else fp64 in-kernel).
cudaError_t fa_prep(const void* P, int ld_p, const void* q_norm, const void* k_norm, void* q_out,
                    void* k_cache, void* v_cache, int kv_cap, int B, int T, int pos0, int Hq,
                    int Hkv, int dh, int rotary_dims, float rope_base, float eps, int dtype,
                    cudaStream_t s, const float2* rope_tab = nullptr);
cudaError_t rope_table(float2* tab, int T, int pos0, int rot, float base, cudaStream_t s);
struct QNorm;
// qn: queries arrive raw (the input projection) and are QK-normed and rotated by the
// tensor-core kernel as it stages them (bf16, head dim 256, Tq >= 16 only).
cudaError_t gqa_attn(const void* q, int ld_q, const void* k, const void* v, int kv_cap,
                     const void* gate, int ld_gate, void* out, int B, int Tq, int Tkv, int q_off,
                     int Hq, int Hkv, int dh, int causal, void* workspace, int dtype,
                     cudaStream_t s, const QNorm* qn = nullptr);
// Workspace bound for any Hkv and dtype (what loop_gqa_workspace_bytes promises).
size_t gqa_workspace_bytes(int B, int Tq, int Tkv, int Hq, int dh);
// Exact scratch bytes gqa_attn uses with a workspace for this call's shape (0: none).
size_t gqa_scratch_bytes(int B, int Tq, int Tkv, int Hq, int Hkv, int dh, int dtype);
bool gqa_supported(int dh, int Hq, int Hkv);
int gqa_launches(int B, int Tq, int Tkv, int Hq, int Hkv, int dh, int dtype, bool has_workspace);
// Query normalisation and rotary applied by the attention kernel as it stages Q (q then is
// the raw projection): gain [dh] (dtype), rotary dims (<= dh/2), base, eps, and an optional
// cos/sin table whose row p - tab_pos0 holds position p (else fp64 in-kernel).  Query t
// sits at position q_off + t.
struct QNorm {
  const void* gain;
  int rot;
  float base, eps;
  const float2* tab;
  int tab_pos0;
};
// tcgen05 flash attention (bf16, head dim 256); used for multi-token queries.
bool gqa_tc_supported(int dh, int dtype, const void* q, int ld_q, const void* gate, int ld_gate, const void* k,
                      const void* v, int kv_cap);
cudaError_t gqa_attn_tc(const void* q, int ld_q, const void* k, const void* v, int kv_cap, const void* gate,
                        int ld_gate, void* out, int B, int Tq, int Tkv, int q_off, int Hq, int Hkv, int causal,
                        cudaStream_t s, const QNorm* qn = nullptr);

// w_rt: optional [8, 2d] transposed copy of w_r (coalesced routing-map reads).
cudaError_t mhc(int mode, const void* X_in, const void* F, const float* coeffs_in, const float* w_r,
                const float* b_r, void* X_out, void* x_in, void* h_out, float* coeffs_out, int N,
                int d, float eps, int iters, int dtype, cudaStream_t s, const float* w_rt = nullptr);
cudaError_t transpose_wr(const float* w, float* wt, int two_d, cudaStream_t s);
cudaError_t sinkhorn(const float* logits, float* out, int N, int n, int iters, cudaStream_t s);

int read_and_clear_device_error();
// One bounded wait that runs out after `limit` SM clock cycles (the error path's self-test).
cudaError_t wait_selftest(long long limit, cudaStream_t s);

}  // namespace lk
