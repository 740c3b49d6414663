/*
 * loop.h -- C ABI of the B200 (sm_100a) looped hybrid decoder forward pass.
 *
 * The model is the looped hybrid decoder described for SenseNova-Loop-9B-Preview:
 *   - "Loop-9B engineering teardown" (hncyxsy.com/news/268323) §二: 32 stored layers
 *     run as 56 executions, layers 0-3, then the block 4-27 twice with the same
 *     weights (B(B(h))), then 28-31 and the head;
 *   - same page §三: groups of 3 Gated-DeltaNet layers + 1 GQA full-attention layer
 *     (16 query / 4 KV heads, head dim 256, QK-norm, output gate, interleaved
 *     rotary on 0.25 of the head dims);
 *   - same page §四: every execution keeps its own KV cache / GDN state;
 *   - same page §五 and "SenseNova-Loop-9B 是什么" (yuliuswiki.com) §二: a
 *     two-stream mHC residual in the loop block whose mixing matrix is made
 *     doubly stochastic by 20 Sinkhorn iterations in FP32;
 *   - same page §六: entering the loop copies h into both streams, leaving it
 *     averages them.
 *
 * Conventions (all entry points):
 *   - Every pointer named "device" is CUDA device memory owned by the caller unless
 *     stated otherwise; every pointer named "host" is host memory.  Tensors are
 *     dense row-major with the shapes given, innermost dimension last.
 *   - dtype selects the storage type of activations and weights: LOOP_F32 (float)
 *     or LOOP_BF16 (__nv_bfloat16).  Arithmetic is FP32 (accumulation, softmax,
 *     norms, GDN state, mHC routing) in both cases.
 *   - Work is enqueued asynchronously on `stream` (a cudaStream_t; NULL = default
 *     stream).  Argument errors are returned synchronously and nothing is launched.
 *     A launch failure is returned as LOOP_ERR_CUDA; faults inside kernels surface
 *     on the next synchronising call.  Kernels that detect bad data (a token id out
 *     of range, a wait that ran out) never trap: they record a code that
 *     loop_device_error() returns.
 *   - loop_last_error() gives a message for the last failing call of this thread.
 *   - A per-op call with an empty problem (a zero batch, length or row count) is a
 *     no-op that returns LOOP_OK; its pointers may then be NULL.
 *   - No entry point allocates device memory except loop_model_create (which keeps
 *     a grow-only activation workspace), loop_cache_create, and the first
 *     loop_prefill / loop_forward_hidden of a larger batch*length than before.
 *   - Functions are thread-compatible: one model/cache must not be used from two
 *     threads at once.
 */
#ifndef LOOP_B200_H
#define LOOP_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  LOOP_OK = 0,
  LOOP_ERR_INVALID_ARG = 1,   /* null pointer, negative size, unknown enum */
  LOOP_ERR_SHAPE = 2,         /* sizes the kernels do not support (see each entry) */
  LOOP_ERR_OOM = 3,           /* cudaMalloc failed */
  LOOP_ERR_CUDA = 4,          /* a CUDA runtime call or launch failed */
  LOOP_ERR_CAPACITY = 5,      /* a cache would overflow its max_tokens */
  LOOP_ERR_TIMEOUT = 6,       /* a device-side bounded wait gave up */
  LOOP_ERR_UNSUPPORTED = 7    /* valid but not built (e.g. a head size without a kernel) */
} loop_status;

typedef enum { LOOP_F32 = 0, LOOP_BF16 = 1 } loop_dtype;

/* Model dimensions.  Defaults for the 9B shape: d 4096, ffn 12288, vocab 248320,
 * n_layers 32, loop [4, 28) x 2 passes, group 4, GDN 16 heads x dk=dv=128,
 * FA 16 q / 4 kv heads x 256, rotary 64, 2 mHC streams, 20 Sinkhorn iterations,
 * GDN chunk 64, eps 1e-6, rope base 10000. */
typedef struct loop_config {
  int d, ffn, vocab;
  int n_layers, loop_start, loop_end, loop_passes, group;
  int gdn_heads, gdn_dk, gdn_dv;
  int fa_q_heads, fa_kv_heads, fa_head_dim, rotary_dims;
  int mhc_streams, sinkhorn_iters, gdn_chunk;
  float eps, rope_base;
  int dtype;             /* loop_dtype */
  int with_embedding;    /* 1: token ids in, logits out; 0: hidden states in/out */
  /* GDN variant ("原地套圈" investigation §01 declares the backbone qwen3_5_text):
   * 0 = plain GDN; 1 = causal depthwise conv (gdn_conv taps) + SiLU on the q | k | v
   * channels and a gated RMSNorm of each head's output, with gdn_v_heads value heads
   * (0 = gdn_heads; a multiple of gdn_heads) reading gdn_heads key heads. */
  int gdn_variant, gdn_v_heads, gdn_conv;
} loop_config;

/* Weights of one stored layer; device pointers, caller-owned, must outlive the model.
 * Projection weights are [out, in] row-major (y = x W^T).  Types: dtype unless
 * marked fp32. */
typedef struct loop_layer_weights {
  const void* attn_norm;      /* [d] pre-mixer RMSNorm gain */
  const void* w_in;           /* GDN: [2*H*dk + H*dv + 2*H, d], row blocks q | k | v | a | b
                                 GDN variant: [2*Hk*dk + 2*Hv*dv + 2*Hv, d], q | k | v | z | a | b
                                 FA:  [2*Hq*dh + 2*Hkv*dh, d],  row blocks q | gate | k | v */
  const float* gdn_a_bias;    /* GDN [H] fp32: decay gate g = -softplus(a + a_bias) */
  const float* gdn_b_bias;    /* GDN [H] fp32: beta = sigmoid(b + b_bias) */
  const void* q_norm;         /* FA [dh] QK-norm gain for queries */
  const void* k_norm;         /* FA [dh] QK-norm gain for keys */
  const void* w_out;          /* GDN [d, H*dv]; FA [d, Hq*dh] */
  const void* ffn_norm;       /* [d] */
  const void* w_gate;         /* [ffn, d] */
  const void* w_up;           /* [ffn, d] */
  const void* w_down;         /* [d, ffn] */
  const float* mhc_w_r;       /* looped layers: [streams*d, 8] fp32 routing map, else NULL */
  const float* mhc_b_r;       /* looped layers: [8] fp32 routing bias, else NULL */
  const void* gdn_conv_w;     /* GDN variant: [2*Hk*dk + Hv*dv, gdn_conv] conv taps (last = current token) */
  const void* gdn_o_norm;     /* GDN variant: [dv] gain of the gated output norm */
} loop_layer_weights;

typedef struct loop_weights {
  const void* embed;          /* [vocab, d] (with_embedding) */
  const void* final_norm;     /* [d]        (with_embedding) */
  const void* lm_head;        /* [vocab, d] (with_embedding; untied) */
  const loop_layer_weights* layers;   /* host array [n_layers], copied at create */
  int n_layers;
} loop_weights;

typedef struct loop_model loop_model;
typedef struct loop_cache loop_cache;

/* ---------------------------------------------------------------- library */
const char* loop_last_error(void);
/* Device error word (see Conventions); reads and clears it on the current device. */
loop_status loop_device_error(int* code_out /* host */);

/* Self-test of the bounded-wait error path: launches one CTA on `stream` in which a thread
 * waits on an mbarrier that nothing completes.  After `cycles` SM clock cycles (0 < cycles
 * <= 4e9; every wait inside the library's kernels gives up after 4e9, about 2 s) the wait
 * gives up, records the wait-timeout code in the device error word and the kernel returns
 * normally: the next loop_device_error() reports LOOP_ERR_TIMEOUT and clears it, and the
 * context stays usable.  Nothing else is touched.  Returns LOOP_ERR_INVALID_ARG for cycles
 * out of range, else the launch status. */
loop_status loop_wait_selftest(long long cycles, void* stream);
const char* loop_version(void);

/* ---------------------------------------------------------------- schedule
 * Execution table of a config ("Loop-9B engineering teardown" §二, §三, §四): one
 * row of 5 int32 per execution, written to host memory `table`:
 *   [execution, stored layer, kind (0 = GDN, 1 = full attention), cache slot, in_loop]
 * The slot is the ordinal among executions of the same kind (FA executions own KV
 * slabs 0..n_fa-1, GDN executions own states 0..n_gdn-1); in_loop = 1 for the
 * executions wrapped by the two-stream mHC residual.  capacity = rows available. */
loop_status loop_schedule(const loop_config* cfg, int32_t* table /* host [capacity*5] */,
                          int capacity, int* n_exec /* host */, int* n_fa /* host */,
                          int* n_gdn /* host */);

/* ---------------------------------------------------------------- model */
loop_status loop_model_create(const loop_config* cfg, const loop_weights* w, loop_model** out);
loop_status loop_model_destroy(loop_model* m);

/* ---------------------------------------------------------------- per-execution cache
 * Owns n_fa KV slabs, each K and V [batch, Hkv, max_tokens, dh] (dtype), and n_gdn
 * GDN states [batch, H, dv, dk] fp32 ("Loop-9B engineering teardown" §四: the two
 * loop passes keep separate caches).  Bytes = n_fa*2*batch*Hkv*max_tokens*dh*esize
 * + n_gdn*batch*H*dv*dk*4.  The GDN variant's states have H = Hv value heads, and each
 * GDN execution also keeps its last gdn_conv - 1 conv inputs [batch, gdn_conv-1, C]
 * (dtype, C = 2*Hk*dk + Hv*dv), counted in state_bytes.  New caches are zero with
 * length 0. */
loop_status loop_cache_create(const loop_model* m, int batch, int max_tokens, loop_cache** out);
loop_status loop_cache_reset(loop_cache* c);          /* length 0, states zeroed (on the default stream) */
loop_status loop_cache_destroy(loop_cache* c);
loop_status loop_cache_length(const loop_cache* c, int* len /* host */);
/* Declare that positions 0..len-1 of every slab and the GDN states hold a valid context
 * written by the caller (e.g. restored from a saved cache); the next prefill or decode
 * step appends at position len.  0 <= len <= max_tokens. */
loop_status loop_cache_set_length(loop_cache* c, int len);
loop_status loop_cache_bytes(const loop_cache* c, size_t* kv_bytes, size_t* state_bytes /* host */);
/* Device pointers to one slab / state (for inspection and tests). */
loop_status loop_cache_kv(const loop_cache* c, int fa_slot, void** k, void** v);
loop_status loop_cache_state(const loop_cache* c, int gdn_slot, float** s);

/* ---------------------------------------------------------------- forward
 * Prefill: ids [B, T] int32 device (B = cache batch) are appended at the cache's
 * current length L; logits_last [B, vocab] fp32 device receives the logits of the
 * last new position.  T + L <= max_tokens, else LOOP_ERR_CAPACITY. */
loop_status loop_prefill(loop_model* m, loop_cache* c, const int32_t* ids, int B, int T,
                         float* logits_last, void* stream);
/* Hidden states in, hidden states out (models without embedding): h_in, h_out
 * [B, T, d] dtype device; h_out is the state after the last execution, before any
 * final norm. Appends to the cache like loop_prefill. */
loop_status loop_forward_hidden(loop_model* m, loop_cache* c, const void* h_in, void* h_out,
                                int B, int T, void* stream);
/* One decode step: tok [B] int32 device; logits [B, vocab] fp32 device (may be NULL);
 * next_tok [B] int32 device = argmax (lowest index on ties). */
loop_status loop_decode_step(loop_model* m, loop_cache* c, const int32_t* tok, float* logits,
                             int32_t* next_tok, void* stream);

/* Hidden-state taps ("原地套圈" investigation §03: the draft models read the target's
 * hidden states at execution indices [3, 27, 51, 53, 54] -- the end of the head, of the
 * first and second loop pass, and two tail layers).  While taps are set, every
 * loop_prefill / loop_forward_hidden / loop_decode_step of this model also writes, for
 * i < n, the hidden state of its new tokens after execution exec[i] to out[i]
 * ([B*T, d] dtype, device, caller-owned, rows in token-major order): outside the loop
 * block the layer's output h; inside it the mean of the two residual streams after that
 * execution's mix, (X'_0 + X'_1) / 2.  max_rows is the row capacity of every buffer: a
 * call with more than max_rows new tokens returns LOOP_ERR_CAPACITY and launches nothing.
 * exec[i] must lie in [0, n_executions) and be distinct (LOOP_ERR_INVALID_ARG).  n = 0
 * clears the taps.  exec and out are host arrays, copied; the buffers must stay valid
 * while set. */
loop_status loop_set_taps(loop_model* m, int n, const int32_t* exec /* host [n] */,
                          void* const* out /* host [n] of device pointers */, long max_rows);

/* ---------------------------------------------------------------- per-op entry points
 * All pointers device, caller-owned, contiguous unless a row stride is given.  */

/* Chunked gated delta rule ("Loop-9B engineering teardown" §三: constant-size state
 * updated with a gate and the delta rule).  Per (b, h), for t = 0..T-1:
 *   S <- exp(g_t) S;  S <- S + beta_t (v_t - S k_t) k_t^T;  o_t = scale * S q_t
 * computed C = chunk tokens at a time (UT-transform form; exact up to rounding).
 * q, k [B, T, H, dk] dtype (already L2-normalised); v [B, T, H, dv] dtype;
 * g (log decay, <= 0), beta [B, T, H] fp32; state [B, H, dv, dk] fp32 in/out;
 * out [B, T, H, dv] dtype.  Supported: (dk, dv) in {(64,64), (128,128)}, chunk 64.
 * workspace: device scratch of loop_gdn_workspace_bytes(B, T, H, dk, dv) bytes for the
 * two-pass scan (every chunk's intra-chunk solve in parallel, then the sequential state
 * pass), or NULL for a single-pass kernel that needs no scratch (slower).  With a
 * workspace, q, k, v and the workspace must be 16-byte aligned (LOOP_ERR_UNSUPPORTED
 * otherwise).  Calls that share a workspace must not overlap on the GPU. */
loop_status gdn_chunk_fwd(const void* q, const void* k, const void* v, const float* g,
                          const float* beta, float* state, void* out, int B, int T, int H,
                          int dk, int dv, int chunk, float scale, void* workspace, int dtype,
                          void* stream);
size_t loop_gdn_workspace_bytes(int B, int T, int H, int dk, int dv);

/* The GDN input projection with gdn_prep fused into its epilogue: the product x W_in^T
 * (x [M, d] row stride ldx, W_in [2*H*dk + H*dv + 2*H, d]) is never stored; each row's
 * q, k heads are L2-normalised from the fp32 accumulators and written with v, g and beta
 * exactly as gdn_prep writes them.  Built for the prefill shapes only: bf16, M > 128,
 * dk = dv = 128, H even and <= 16, 16-byte aligned x, W_in, q, k, v (LOOP_ERR_UNSUPPORTED
 * otherwise: use loop_linear + gdn_prep). */
loop_status gdn_in_proj(const void* x, int ldx, const void* w_in, const float* a_bias,
                        const float* b_bias, void* q, void* k, void* v, float* g, float* beta,
                        int M, int d, int H, int dk, int dv, float eps, int dtype, void* stream);

/* GDN variant input preparation ("原地套圈" investigation §01, backbone qwen3_5_text): from
 * P [B*T, ld_p] (row blocks q | k (Hk heads) | v | z (Hv heads) | a | b (Hv)): the q | k | v
 * channels c pass through a causal depthwise conv and SiLU,
 *   y_t[c] = silu(sum_{j<conv} conv_w[c][j] * x_{t-(conv-1)+j}[c]),
 * where inputs before the call's first token come from conv_state [B, conv-1, C] (dtype,
 * in/out: afterwards it holds the last conv-1 inputs); then q, k are L2-normalised per head
 * (x / sqrt(sum x^2 + eps)) and written once per value head h that reads key head
 * h / (Hv/Hk): q, k [B*T, Hv, dk]; v [B*T, Hv, dv]; g = -softplus(a + a_bias),
 * beta = sigmoid(b + b_bias) [B*T, Hv] fp32.  conv must be 4; (dk, dv) as gdn_chunk_fwd. */
loop_status gdn_conv_prep(const void* P, int ld_p, const void* conv_w, void* conv_state,
                          const float* a_bias, const float* b_bias, void* q, void* k, void* v,
                          float* g, float* beta, int B, int T, int Hk, int Hv, int dk, int dv,
                          int conv, float eps, int dtype, void* stream);

/* Gated output norm of the GDN variant: y [M, H, dv] = RMSNorm(o) * w * silu(z) per head
 * (RMSNorm over dv with eps inside the root); o [M, H, dv], z rows of stride ld_z
 * elements ([M, H*dv] blocks), w [dv]; y may equal o.  dv a multiple of 32, <= 256. */
loop_status gdn_gated_norm(const void* o, const void* z, int ld_z, const void* w, void* y, int M, int H,
                           int dv, float eps, int dtype, void* stream);

/* One token of the same recurrence per sequence: q, k [B, H, dk]; v, out [B, H, dv];
 * g, beta [B, H] fp32; state [B, H, dv, dk] fp32 in/out. */
loop_status gdn_step(const void* q, const void* k, const void* v, const float* g,
                     const float* beta, float* state, void* out, int B, int H, int dk, int dv,
                     float scale, int dtype, void* stream);

/* GDN input preparation from the layer's input projection P [M, ld_p] (row blocks
 * q | k | v | a | b, see loop_layer_weights): q, k L2-normalised per head
 * (x / sqrt(sum x^2 + eps)), g = -softplus(a + a_bias), beta = sigmoid(b + b_bias).
 * Outputs q, k [M, H, dk], v [M, H, dv] dtype; g, beta [M, H] fp32. */
loop_status gdn_prep(const void* P, int ld_p, const float* a_bias, const float* b_bias,
                     void* q, void* k, void* v, float* g, float* beta, int M, int H, int dk,
                     int dv, float eps, int dtype, void* stream);

/* Grouped-query softmax attention with the sigmoid output gate ("Loop-9B
 * engineering teardown" §三):
 *   out[b,t,h] = sigmoid(gate[b,t,h]) * sum_p softmax_p(q[b,t,h].k[b,g,p] / sqrt(dh)) v[b,g,p]
 * with g = h / (Hq/Hkv); query t sits at position q_off + t; causal: p <= q_off + t;
 * p ranges over 0..Tkv-1.  q [B, Tq, Hq, dh] (row stride ld_q elements between
 * tokens, >= Hq*dh); gate likewise (ld_gate; NULL = no gate); k, v [B, Hkv, kv_cap, dh]
 * (per-execution slab layout; kv_cap >= Tkv); out [B, Tq, Hq, dh] contiguous.
 * q and k are used as given (already QK-normed and rotated).
 * workspace: device scratch of loop_gqa_workspace_bytes(...) bytes, or NULL (then a
 * single pass over the keys is used).
 * Kernels by shape: bf16 with Tq >= 16, dh 256 and 128 % (Hq/Hkv) == 0 runs the tcgen05
 * flash kernel; bf16 with Tq == 1 runs a flash-decode kernel (dh 128/256 with <= 16, dh 64
 * with <= 4 q heads per KV head); other calls run one warp per query row.  The tiled kernels
 * need 16-byte aligned q, k, v, gate and row strides that are multiples of 8 elements: a
 * call whose shape selects one of them with buffers that are not is refused with
 * LOOP_ERR_UNSUPPORTED (never run on a slower kernel). */
loop_status gqa_attn(const void* q, int ld_q, const void* k, const void* v, int kv_cap,
                     const void* gate, int ld_gate, void* out, int B, int Tq, int Tkv, int q_off,
                     int Hq, int Hkv, int dh, int causal, void* workspace, int dtype, void* stream);
size_t loop_gqa_workspace_bytes(int B, int Tq, int Tkv, int Hq, int dh);

/* gqa_attn without allocation.  The pages have no counterpart to this entry point; it
 * exists for callers that cannot allocate device memory for a workspace -- e.g. a host
 * runtime that has given all free device memory to its own pool, or a latency-critical
 * loop that must not take the implicit device synchronisation of cudaMalloc/cudaFree.
 * Same arguments and result as gqa_attn (minus `workspace`); the split-K scratch is a
 * fixed 32 MiB array in the library's device memory, held on every GPU that loads the
 * library until the process exits.  A problem whose scratch exceeds 32 MiB is rejected
 * with LOOP_ERR_CAPACITY and nothing is launched; the scratch is the split-K partials of the
 * kernel that the call's shape selects, B*Tq*Hq*splits*(dh+2)*4 bytes when that kernel
 * splits the keys (single-token decode, the row kernel) and none otherwise (bf16 multi-token
 * queries with head dim 256); it never exceeds loop_gqa_workspace_bytes.  The first
 * call on each device (with that device current) looks the array's address up with
 * cudaGetSymbolAddress; make that first call before any stream capture.  Every call
 * shares the array: calls that overlap on the GPU (different streams, or different host
 * threads on one device) race on it.  The array keeps the last call's contents, but
 * every slot a call reads is written by that call first, so nothing needs clearing.
 * Allocates nothing: no cudaMalloc, cudaFree or allocating library routine. */
loop_status gqa_attn_noalloc(const void* q, int ld_q, const void* k, const void* v, int kv_cap,
                             const void* gate, int ld_gate, void* out, int B, int Tq, int Tkv,
                             int q_off, int Hq, int Hkv, int dh, int causal, int dtype, void* stream);

/* gqa_attn with the query side of "Loop-9B engineering teardown" §三 fused in: q are the
 * raw query rows of the input projection (row stride ld_q), and the kernel applies
 * QK-norm and rotary to them as it loads them, q' = rope(rmsnorm(q) * q_norm) (RMSNorm
 * over the dh dims with eps inside the root; dims [0, rotary_dims) rotated in adjacent
 * pairs (2j, 2j+1) by angle pos * rope_base^(-2j/rotary_dims), pos = q_off + t).  k and v
 * are the slab as fa_prep writes it (keys already normed and rotated).  Built for the
 * tensor-core kernel only: bf16, dh 256, Tq >= 16, 128 % (Hq/Hkv) == 0, rotary_dims <=
 * dh/2, 16-byte aligned q, q_norm, k, v, gate; other calls return LOOP_ERR_UNSUPPORTED.
 * Needs no workspace.  The rotary angles are evaluated in fp64 by each query row's
 * threads (the model's own forward passes a per-call cos/sin table instead). */
loop_status gqa_attn_fused_q(const void* q, int ld_q, const void* q_norm, int rotary_dims, float rope_base,
                             float eps, const void* k, const void* v, int kv_cap, const void* gate,
                             int ld_gate, void* out, int B, int Tq, int Tkv, int q_off, int Hq, int Hkv,
                             int dh, int causal, int dtype, void* stream);

/* QK-norm + partial rotary + KV write for one FA execution.  From P [M = B*T, ld_p]
 * (row blocks q | gate | k | v): q_out [M, Hq, dh] = rope(rmsnorm(q) * q_norm);
 * k = rope(rmsnorm(k) * k_norm) and v are written to the slabs k_cache, v_cache
 * [B, Hkv, kv_cap, dh] at positions pos0 .. pos0+T-1.  Rotary: dims [0, rotary_dims)
 * in adjacent pairs (2j, 2j+1), angle = pos * base^(-2j/rotary_dims).  q_out may be NULL:
 * then only the keys and values are written (the queries go raw to gqa_attn_fused_q). */
loop_status fa_prep(const void* P, int ld_p, const void* q_norm, const void* k_norm,
                    void* q_out, void* k_cache, void* v_cache, int kv_cap, int B, int T, int pos0,
                    int Hq, int Hkv, int dh, int rotary_dims, float rope_base, float eps,
                    int dtype, void* stream);

/* mHC two-stream residual, one kernel per layer boundary ("Loop-9B engineering
 * teardown" §五, §六).  Per token, X is [streams=2, d] (dtype), coeffs [8] fp32 =
 * [H_pre(2), H_post(2), H_res(2x2 row-major)].
 *   mode 0 OPEN:  X' = (h, h) from h = X_in [N, d]
 *   mode 1 MIX:   X' = H_res X + H_post^T F with (H_post, H_res) from coeffs_in, F [N, d]
 *   mode 2 ROUTE: X' = X_in (no mixing; X_out may equal X_in or be NULL)
 *   mode 3 MERGE: MIX, then h_out = (X'_0 + X'_1) / 2 [N, d]; no routing, X' not stored
 * Modes 0-2 then route from X': l = RMSNorm(flatten X') W_r + b_r (fp32, no gain),
 * H_pre = sigmoid(l[0:2]), H_post = 2 sigmoid(l[2:4]), H_res = Sinkhorn_iters(exp(l[4:8])),
 * write X_out [N, 2, d], x_in [N, d] = sum_s H_pre[s] X'_s, and coeffs_out [N, 8].
 * Routing reads X' as stored (rounded to dtype).  X_out may equal X_in (in-place MIX).
 * Every array pointer must be 16-byte aligned (LOOP_ERR_INVALID_ARG otherwise); d must
 * be a multiple of 8. */
loop_status mhc_route_mix(int mode, const void* X_in, const void* F, const float* coeffs_in,
                          const float* w_r, const float* b_r, void* X_out, void* x_in,
                          void* h_out, float* coeffs_out, int N, int d, float eps, int iters,
                          int dtype, void* stream);

/* Sinkhorn-Knopp in FP32: M = exp(L - max L); repeat iters: divide rows by their
 * sums, then columns by their sums.  logits, out [N, n, n] fp32; n <= 8. */
loop_status sinkhorn_fp32(const float* logits, float* out, int N, int n, int iters, void* stream);

/* Dense projection Y = X W^T (tcgen05 tensor cores for bf16, FP32 SIMT for f32):
 * X [M, K] (row stride ldx), W [N, K]; epilogue:
 *   0 STORE:  Y [M, N] (dtype, row stride ldy)
 *   1 ADD:    Y = X W^T + R, R [M, N] (row stride ldr) may alias Y
 *   2 SWIGLU: Y [M, N] = silu(X W^T) * (X W2^T), W2 [N, K] (the FFN's up map)
 *   3 F32:    Y [M, N] fp32
 * K must be a multiple of 8 for bf16, and bf16 calls need 16-byte aligned X, W (W2) and
 * a row stride ldx that is a multiple of 8 (TMA); otherwise LOOP_ERR_UNSUPPORTED (bf16 has
 * no slower fallback kernel).
 * bf16 calls with M <= 128 (decode batches, a last position) stream W through every SM
 * with the batch as the MMA's N dimension.
 * workspace: optional device scratch of loop_linear_workspace_bytes(M, N, K, epilogue)
 * bytes (NULL = none), ZERO-FILLED by the caller before its first use.  With it, bf16
 * calls with M <= 128 may split a 128-column tile's K range between CTAs: the parts are
 * summed there in fp32 and the CTA that completes a tile applies the epilogue and
 * zero-fills the tile's slice again, so a completed call leaves the workspace as it
 * found it (a call cut short by a device error may not).  Without it, every tile is
 * computed whole by one CTA.  Calls sharing a workspace must not overlap on the GPU. */
loop_status loop_linear(const void* X, int ldx, const void* W, const void* W2, const void* R,
                        int ldr, void* Y, int ldy, int M, int N, int K, int epilogue,
                        void* workspace, int dtype, void* stream);
size_t loop_linear_workspace_bytes(int M, int N, int K, int epilogue);

/* y = rmsnorm(x [+ r]) * w over rows of length d; if sum_out != NULL it receives x + r
 * (the residual sum).  x, r, sum_out, y [M, d] dtype; w [d] dtype. */
loop_status loop_rmsnorm(const void* x, const void* r, void* sum_out, const void* w, void* y,
                         int M, int d, float eps, int dtype, void* stream);

/* out [M, d] = embed[ids[m]]; ids [M] int32; an id outside [0, vocab) writes zeros
 * and sets device error 1. */
loop_status loop_embed(const int32_t* ids, const void* embed, void* out, int M, int d,
                       int vocab, int dtype, void* stream);

/* next [B] int32 = argmax over logits [B, V] fp32, lowest index on ties. */
loop_status loop_argmax(const float* logits, int32_t* next, int B, int V, void* stream);

/* ---------------------------------------------------------------- per-kernel timing
 * While enabled, the model brackets every kernel launch of loop_prefill /
 * loop_forward_hidden / loop_decode_step with CUDA events on the launch stream and
 * records the launch's algorithmic work (flops = 2 x multiply-adds of the definition;
 * bytes = the tensors the kernel must read and write once).  loop_profile_read
 * synchronises on the recorded events and returns one entry per kernel class
 * ("gemm", "lm_head", "gdn_chunk", "gdn_step", "attention", "mhc", ...), summed over
 * everything recorded since loop_profile_enable(m, 1).  Events add a few microseconds
 * of host time per launch. */
typedef struct loop_profile_entry {
  char name[24];
  int launches;       /* kernel launches of this class */
  double ms;          /* summed event time */
  double flops;       /* summed algorithmic flops */
  double bytes;       /* summed algorithmic HBM bytes */
} loop_profile_entry;
loop_status loop_profile_enable(loop_model* m, int on);
loop_status loop_profile_read(loop_model* m, loop_profile_entry* out /* host [cap] */, int cap, int* n /* host */);

#ifdef __cplusplus
}
#endif
#endif /* LOOP_B200_H */
