// C ABI (include/loop.h): argument checking and dispatch to the kernels / runtime.
// Nothing here computes; every step runs in a CUDA kernel.
#include <cstdio>
#include <new>

#include "common.cuh"
#include "runtime.h"

using namespace lk;

#define REQUIRE(cond, st, msg) \
  do {                         \
    if (!(cond)) return fail(st, msg); \
  } while (0)

static loop_status launched(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return LOOP_OK;
  if (e == cudaErrorNotSupported) return fail(LOOP_ERR_UNSUPPORTED, std::string(what) + ": shape not supported");
  return cuda_fail(e, what);
}

static bool dtype_ok(int dt) { return dt == LOOP_F32 || dt == LOOP_BF16; }
static cudaStream_t S(void* s) { return (cudaStream_t)s; }

loop_status gqa_check_args(const char* who, const void* q, int ld_q, const void* k, const void* v, int kv_cap,
                           const void* gate, int ld_gate, const void* out, int B, int Tq, int Tkv, int q_off, int Hq,
                           int Hkv, int dh, int causal, int dtype, bool* empty) {
  const std::string w = std::string(who) + ": ";
  *empty = false;
  if (!dtype_ok(dtype)) return fail(LOOP_ERR_INVALID_ARG, w + "bad dtype");
  if (B < 0 || Tq < 0 || Tkv < 0 || q_off < 0) return fail(LOOP_ERR_INVALID_ARG, w + "negative size");
  if (B == 0 || Tq == 0) {
    *empty = true;
    return LOOP_OK;
  }
  if (!q || !k || !v || !out) return fail(LOOP_ERR_INVALID_ARG, w + "NULL argument");
  if (!gqa_supported(dh, Hq, Hkv)) return fail(LOOP_ERR_UNSUPPORTED, w + "head dim or head ratio not supported");
  if (kv_cap < Tkv) return fail(LOOP_ERR_SHAPE, w + "kv_cap < Tkv");
  if (ld_q < Hq * dh || (gate && ld_gate < Hq * dh)) return fail(LOOP_ERR_SHAPE, w + "row stride smaller than Hq*dh");
  if (causal && q_off + Tq > Tkv) return fail(LOOP_ERR_SHAPE, w + "causal attention needs q_off + Tq <= Tkv");
  return LOOP_OK;
}

extern "C" {

const char* loop_version(void) { return "loop-b200 0.1 (sm_100a)"; }

loop_status loop_device_error(int* code_out) {
  REQUIRE(code_out, LOOP_ERR_INVALID_ARG, "code_out is NULL");
  *code_out = read_and_clear_device_error();
  return *code_out == DEV_WAIT_TIMEOUT ? LOOP_ERR_TIMEOUT : LOOP_OK;
}

loop_status loop_wait_selftest(long long cycles, void* stream) {
  REQUIRE(cycles > 0 && cycles <= 4000000000LL, LOOP_ERR_INVALID_ARG, "cycles must be in (0, 4e9]");
  return launched(lk::wait_selftest(cycles, S(stream)), "loop_wait_selftest");
}

static loop_status check_config(const loop_config* c) {
  REQUIRE(c, LOOP_ERR_INVALID_ARG, "config is NULL");
  REQUIRE(dtype_ok(c->dtype), LOOP_ERR_INVALID_ARG, "dtype must be LOOP_F32 or LOOP_BF16");
  REQUIRE(c->d > 0 && c->ffn > 0 && c->n_layers > 0 && c->group > 0 && c->loop_passes >= 0, LOOP_ERR_INVALID_ARG,
          "dimensions must be positive");
  REQUIRE(c->d % 8 == 0 && c->ffn % 8 == 0, LOOP_ERR_SHAPE, "d and ffn must be multiples of 8");
  REQUIRE(0 <= c->loop_start && c->loop_start <= c->loop_end && c->loop_end <= c->n_layers, LOOP_ERR_INVALID_ARG,
          "need 0 <= loop_start <= loop_end <= n_layers");
  REQUIRE(c->mhc_streams == 2, LOOP_ERR_UNSUPPORTED, "only the two-stream mHC is built");
  REQUIRE(c->sinkhorn_iters >= 0, LOOP_ERR_INVALID_ARG, "sinkhorn_iters must be >= 0");
  REQUIRE(gdn_supported(c->gdn_dk, c->gdn_dv) && c->gdn_heads > 0, LOOP_ERR_UNSUPPORTED,
          "GDN head sizes (dk, dv) must be (64, 64) or (128, 128)");
  REQUIRE(c->gdn_variant == 0 || c->gdn_variant == 1, LOOP_ERR_INVALID_ARG, "gdn_variant must be 0 or 1");
  if (c->gdn_variant == 0)
    REQUIRE(c->gdn_v_heads == 0 || c->gdn_v_heads == c->gdn_heads, LOOP_ERR_INVALID_ARG,
            "the plain GDN has as many value heads as key heads");
  else
    REQUIRE(gdn_variant_supported(c->gdn_heads, c->gdn_v_heads ? c->gdn_v_heads : c->gdn_heads, c->gdn_dk, c->gdn_dv,
                                  c->gdn_conv),
            LOOP_ERR_UNSUPPORTED, "GDN variant: value heads a multiple of the key heads, conv 4");
  REQUIRE(c->gdn_chunk == 64, LOOP_ERR_UNSUPPORTED, "GDN chunk must be 64");
  REQUIRE(gqa_supported(c->fa_head_dim, c->fa_q_heads, c->fa_kv_heads), LOOP_ERR_UNSUPPORTED,
          "FA head dim must be 64, 128 or 256 and Hq a multiple of Hkv (ratio <= 32)");
  REQUIRE(c->rotary_dims >= 0 && c->rotary_dims <= c->fa_head_dim && c->rotary_dims % 2 == 0, LOOP_ERR_INVALID_ARG,
          "rotary_dims must be even and <= head dim");
  REQUIRE(c->eps >= 0.f && c->rope_base > 0.f, LOOP_ERR_INVALID_ARG, "eps >= 0 and rope_base > 0 required");
  if (c->with_embedding) REQUIRE(c->vocab > 0, LOOP_ERR_INVALID_ARG, "vocab must be positive");
  return LOOP_OK;
}

loop_status loop_schedule(const loop_config* cfg, int32_t* table, int capacity, int* n_exec, int* n_fa,
                          int* n_gdn) {
  loop_status st = check_config(cfg);
  if (st != LOOP_OK) return st;
  auto rows = build_schedule(*cfg);
  int fa = 0;
  for (auto& r : rows) fa += r.kind;
  if (n_exec) *n_exec = (int)rows.size();
  if (n_fa) *n_fa = fa;
  if (n_gdn) *n_gdn = (int)rows.size() - fa;
  if (!table) return LOOP_OK;
  REQUIRE(capacity >= (int)rows.size(), LOOP_ERR_CAPACITY, "table capacity smaller than the number of executions");
  for (size_t i = 0; i < rows.size(); ++i) {
    table[5 * i + 0] = rows[i].exec;
    table[5 * i + 1] = rows[i].layer;
    table[5 * i + 2] = rows[i].kind;
    table[5 * i + 3] = rows[i].slot;
    table[5 * i + 4] = rows[i].in_loop;
  }
  return LOOP_OK;
}

loop_status loop_model_create(const loop_config* cfg, const loop_weights* w, loop_model** out) {
  REQUIRE(out, LOOP_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  loop_status st = check_config(cfg);
  if (st != LOOP_OK) return st;
  REQUIRE(w && w->layers, LOOP_ERR_INVALID_ARG, "weights or weights->layers is NULL");
  REQUIRE(w->n_layers == cfg->n_layers, LOOP_ERR_SHAPE, "weights->n_layers differs from config n_layers");
  if (cfg->with_embedding)
    REQUIRE(w->embed && w->final_norm && w->lm_head, LOOP_ERR_INVALID_ARG, "embed, final_norm and lm_head required");
  for (int l = 0; l < cfg->n_layers; ++l) {
    const loop_layer_weights& L = w->layers[l];
    const bool fa = (l % cfg->group) == cfg->group - 1;
    bool ok = L.attn_norm && L.w_in && L.w_out && L.ffn_norm && L.w_gate && L.w_up && L.w_down;
    ok = ok && (fa ? (L.q_norm && L.k_norm) : (L.gdn_a_bias && L.gdn_b_bias));
    if (!fa && cfg->gdn_variant == 1) ok = ok && L.gdn_conv_w && L.gdn_o_norm;
    if (l >= cfg->loop_start && l < cfg->loop_end && cfg->loop_passes > 0) ok = ok && L.mhc_w_r && L.mhc_b_r;
    if (!ok) return fail(LOOP_ERR_INVALID_ARG, "layer " + std::to_string(l) + ": a required weight pointer is NULL");
  }
  loop_model* m = new (std::nothrow) loop_model();
  REQUIRE(m, LOOP_ERR_OOM, "host allocation failed");
  m->cfg = *cfg;
  m->layers.assign(w->layers, w->layers + cfg->n_layers);
  m->embed = w->embed;
  m->final_norm = w->final_norm;
  m->lm_head = w->lm_head;
  m->sched = build_schedule(*cfg);
  for (auto& r : m->sched) {
    if (r.kind) m->n_fa++; else m->n_gdn++;
    if (r.in_loop) {
      if (m->first_loop < 0) m->first_loop = r.exec;
      m->last_loop = r.exec;
    }
  }
  m->esize = cfg->dtype == LOOP_BF16 ? 2 : 4;
  m->gdn_hv = cfg->gdn_v_heads ? cfg->gdn_v_heads : cfg->gdn_heads;
  m->gdn_ch = 2 * cfg->gdn_heads * cfg->gdn_dk + m->gdn_hv * cfg->gdn_dv;
  m->in_gdn = cfg->gdn_variant == 1 ? m->gdn_ch + m->gdn_hv * cfg->gdn_dv + 2 * m->gdn_hv
                                    : 2 * cfg->gdn_heads * cfg->gdn_dk + cfg->gdn_heads * cfg->gdn_dv + 2 * cfg->gdn_heads;
  m->in_fa = 2 * cfg->fa_q_heads * cfg->fa_head_dim + 2 * cfg->fa_kv_heads * cfg->fa_head_dim;
  *out = m;
  return LOOP_OK;
}

loop_status loop_model_destroy(loop_model* m) {
  delete m;
  return LOOP_OK;
}

loop_status loop_cache_create(const loop_model* m, int batch, int max_tokens, loop_cache** out) {
  REQUIRE(m && out, LOOP_ERR_INVALID_ARG, "model or out is NULL");
  REQUIRE(batch > 0 && max_tokens > 0, LOOP_ERR_INVALID_ARG, "batch and max_tokens must be positive");
  *out = nullptr;
  const loop_config& c = m->cfg;
  loop_cache* k = new (std::nothrow) loop_cache();
  REQUIRE(k, LOOP_ERR_OOM, "host allocation failed");
  k->model = m;
  k->batch = batch;
  k->max_tokens = max_tokens;
  k->kv_slab_elems = (size_t)batch * c.fa_kv_heads * max_tokens * c.fa_head_dim;
  k->state_elems = (size_t)batch * m->gdn_hv * c.gdn_dv * c.gdn_dk;
  k->conv_elems = c.gdn_variant == 1 ? (size_t)batch * (c.gdn_conv - 1) * m->gdn_ch : 0;
  cudaError_t e = k->kv.ensure(std::max<size_t>(256, (size_t)m->n_fa * 2 * k->kv_slab_elems * m->esize));
  if (e == cudaSuccess) e = k->state.ensure(std::max<size_t>(256, (size_t)m->n_gdn * k->state_elems * sizeof(float)));
  if (e == cudaSuccess) e = k->conv.ensure(std::max<size_t>(256, (size_t)m->n_gdn * k->conv_elems * m->esize));
  if (e == cudaSuccess) e = cudaMemset(k->state.p, 0, k->state.bytes);
  if (e == cudaSuccess) e = cudaMemset(k->conv.p, 0, k->conv.bytes);
  if (e != cudaSuccess) {
    delete k;
    return cuda_fail(e, "cache allocation");
  }
  *out = k;
  return LOOP_OK;
}

loop_status loop_cache_reset(loop_cache* c) {
  REQUIRE(c, LOOP_ERR_INVALID_ARG, "cache is NULL");
  cudaError_t e = cudaMemset(c->state.p, 0, c->state.bytes);
  if (e == cudaSuccess) e = cudaMemset(c->conv.p, 0, c->conv.bytes);
  if (e != cudaSuccess) return cuda_fail(e, "cache reset");
  c->len = 0;
  return LOOP_OK;
}

loop_status loop_cache_destroy(loop_cache* c) {
  delete c;
  return LOOP_OK;
}

loop_status loop_cache_length(const loop_cache* c, int* len) {
  REQUIRE(c && len, LOOP_ERR_INVALID_ARG, "NULL argument");
  *len = c->len;
  return LOOP_OK;
}

loop_status loop_cache_set_length(loop_cache* c, int len) {
  REQUIRE(c, LOOP_ERR_INVALID_ARG, "cache is NULL");
  REQUIRE(len >= 0 && len <= c->max_tokens, LOOP_ERR_CAPACITY, "length outside 0..max_tokens");
  c->len = len;
  return LOOP_OK;
}

loop_status loop_cache_bytes(const loop_cache* c, size_t* kv_bytes, size_t* state_bytes) {
  REQUIRE(c, LOOP_ERR_INVALID_ARG, "cache is NULL");
  const loop_model* m = c->model;
  if (kv_bytes) *kv_bytes = (size_t)m->n_fa * 2 * c->kv_slab_elems * m->esize;
  if (state_bytes) *state_bytes = (size_t)m->n_gdn * (c->state_elems * sizeof(float) + c->conv_elems * m->esize);
  return LOOP_OK;
}

loop_status loop_cache_kv(const loop_cache* c, int fa_slot, void** k, void** v) {
  REQUIRE(c && k && v, LOOP_ERR_INVALID_ARG, "NULL argument");
  REQUIRE(fa_slot >= 0 && fa_slot < c->model->n_fa, LOOP_ERR_INVALID_ARG, "fa_slot out of range");
  char* base = (char*)c->kv.p + (size_t)fa_slot * 2 * c->kv_slab_elems * c->model->esize;
  *k = base;
  *v = base + c->kv_slab_elems * c->model->esize;
  return LOOP_OK;
}

loop_status loop_cache_state(const loop_cache* c, int gdn_slot, float** s) {
  REQUIRE(c && s, LOOP_ERR_INVALID_ARG, "NULL argument");
  REQUIRE(gdn_slot >= 0 && gdn_slot < c->model->n_gdn, LOOP_ERR_INVALID_ARG, "gdn_slot out of range");
  *s = (float*)c->state.p + (size_t)gdn_slot * c->state_elems;
  return LOOP_OK;
}

loop_status loop_prefill(loop_model* m, loop_cache* c, const int32_t* ids, int B, int T, float* logits_last,
                         void* stream) {
  REQUIRE(m && c && ids, LOOP_ERR_INVALID_ARG, "model, cache or ids is NULL");
  REQUIRE(m->cfg.with_embedding, LOOP_ERR_INVALID_ARG, "model has no embedding; use loop_forward_hidden");
  REQUIRE(c->model == m, LOOP_ERR_INVALID_ARG, "cache belongs to another model");
  REQUIRE(B == c->batch && T > 0, LOOP_ERR_SHAPE, "B must equal the cache batch and T > 0");
  REQUIRE((long)c->len + T <= c->max_tokens, LOOP_ERR_CAPACITY, "prefill would overflow the cache");
  return run_forward(m, c, ids, nullptr, nullptr, logits_last, B, T, S(stream));
}

loop_status loop_forward_hidden(loop_model* m, loop_cache* c, const void* h_in, void* h_out, int B, int T,
                                void* stream) {
  REQUIRE(m && c && h_in && h_out, LOOP_ERR_INVALID_ARG, "NULL argument");
  REQUIRE(c->model == m, LOOP_ERR_INVALID_ARG, "cache belongs to another model");
  REQUIRE(B == c->batch && T > 0, LOOP_ERR_SHAPE, "B must equal the cache batch and T > 0");
  REQUIRE((long)c->len + T <= c->max_tokens, LOOP_ERR_CAPACITY, "forward would overflow the cache");
  return run_forward(m, c, nullptr, h_in, h_out, nullptr, B, T, S(stream));
}

loop_status loop_decode_step(loop_model* m, loop_cache* c, const int32_t* tok, float* logits, int32_t* next_tok,
                             void* stream) {
  REQUIRE(m && c && tok && next_tok, LOOP_ERR_INVALID_ARG, "NULL argument");
  REQUIRE(m->cfg.with_embedding, LOOP_ERR_INVALID_ARG, "model has no embedding");
  REQUIRE(c->model == m, LOOP_ERR_INVALID_ARG, "cache belongs to another model");
  REQUIRE(c->len >= 1, LOOP_ERR_INVALID_ARG, "decode needs a prefilled cache");
  REQUIRE(c->len + 1 <= c->max_tokens, LOOP_ERR_CAPACITY, "decode would overflow the cache");
  return run_decode(m, c, tok, logits, next_tok, S(stream));
}

loop_status loop_set_taps(loop_model* m, int n, const int32_t* exec, void* const* out, long max_rows) {
  REQUIRE(m, LOOP_ERR_INVALID_ARG, "model is NULL");
  REQUIRE(n >= 0 && max_rows >= 0, LOOP_ERR_INVALID_ARG, "n and max_rows must be >= 0");
  REQUIRE(n == 0 || (exec && out), LOOP_ERR_INVALID_ARG, "exec or out is NULL");
  const int n_exec = (int)m->sched.size();
  for (int i = 0; i < n; ++i) {
    REQUIRE(exec[i] >= 0 && exec[i] < n_exec, LOOP_ERR_INVALID_ARG,
            "tap execution index " + std::to_string(exec[i]) + " outside [0, " + std::to_string(n_exec) + ")");
    REQUIRE(out[i], LOOP_ERR_INVALID_ARG, "tap buffer is NULL");
    for (int j = 0; j < i; ++j) REQUIRE(exec[j] != exec[i], LOOP_ERR_INVALID_ARG, "execution tapped twice");
  }
  m->tap_exec.assign(exec, exec + n);
  m->tap_out.assign(out, out + n);
  m->tap_rows = n ? max_rows : 0;
  return LOOP_OK;
}

// ------------------------------------------------------------------ per-op entry points
size_t loop_gdn_workspace_bytes(int B, int T, int H, int dk, int dv) {
  if (B <= 0 || T <= 0 || H <= 0 || dk <= 0 || dv <= 0) return 0;
  return gdn_workspace_bytes(B, T, H, dk, dv);
}

loop_status gdn_chunk_fwd(const void* q, const void* k, const void* v, const float* g, const float* beta,
                          float* state, void* out, int B, int T, int H, int dk, int dv, int chunk, float scale,
                          void* workspace, int dtype, void* stream) {
  REQUIRE(dtype_ok(dtype), LOOP_ERR_INVALID_ARG, "bad dtype");
  REQUIRE(B >= 0 && T >= 0 && H > 0, LOOP_ERR_INVALID_ARG, "negative size");
  if (B == 0 || T == 0) return LOOP_OK;
  REQUIRE(q && k && v && g && beta && state && out, LOOP_ERR_INVALID_ARG, "NULL argument");
  REQUIRE(chunk == 64, LOOP_ERR_UNSUPPORTED, "chunk must be 64");
  REQUIRE(gdn_supported(dk, dv), LOOP_ERR_UNSUPPORTED, "(dk, dv) must be (64, 64) or (128, 128)");
  return launched(gdn_chunk(q, k, v, g, beta, state, out, B, T, H, dk, dv, scale, dtype, S(stream), workspace),
                  "gdn_chunk_fwd");
}

loop_status gdn_step(const void* q, const void* k, const void* v, const float* g, const float* beta, float* state,
                     void* out, int B, int H, int dk, int dv, float scale, int dtype, void* stream) {
  REQUIRE(dtype_ok(dtype), LOOP_ERR_INVALID_ARG, "bad dtype");
  REQUIRE(B >= 0 && H > 0, LOOP_ERR_INVALID_ARG, "bad size");
  if (B == 0) return LOOP_OK;
  REQUIRE(q && k && v && g && beta && state && out, LOOP_ERR_INVALID_ARG, "NULL argument");
  REQUIRE(gdn_supported(dk, dv), LOOP_ERR_UNSUPPORTED, "(dk, dv) must be (64, 64) or (128, 128)");
  return launched(lk::gdn_step(q, k, v, g, beta, state, out, B, H, dk, dv, scale, dtype, S(stream)), "gdn_step");
}

loop_status gdn_conv_prep(const void* P, int ld_p, const void* conv_w, void* conv_state, const float* a_bias,
                          const float* b_bias, void* q, void* k, void* v, float* g, float* beta, int B, int T, int Hk,
                          int Hv, int dk, int dv, int conv, float eps, int dtype, void* stream) {
  REQUIRE(dtype_ok(dtype), LOOP_ERR_INVALID_ARG, "bad dtype");
  REQUIRE(B >= 0 && T >= 0, LOOP_ERR_INVALID_ARG, "negative size");
  if (B == 0 || T == 0) return LOOP_OK;
  REQUIRE(P && conv_w && conv_state && a_bias && b_bias && q && k && v && g && beta, LOOP_ERR_INVALID_ARG,
          "NULL argument");
  REQUIRE(gdn_variant_supported(Hk, Hv, dk, dv, conv), LOOP_ERR_UNSUPPORTED,
          "Hv a multiple of Hk, (dk, dv) (64, 64) or (128, 128), conv 4");
  REQUIRE(ld_p >= 2 * Hk * dk + 2 * Hv * dv + 2 * Hv, LOOP_ERR_SHAPE, "ld_p smaller than the projection width");
  return launched(lk::gdn_conv_prep(P, ld_p, conv_w, conv_state, a_bias, b_bias, q, k, v, g, beta, B, T, Hk, Hv, dk,
                                    dv, conv, eps, dtype, S(stream)),
                  "gdn_conv_prep");
}

loop_status gdn_gated_norm(const void* o, const void* z, int ld_z, const void* w, void* y, int M, int H, int dv,
                           float eps, int dtype, void* stream) {
  REQUIRE(dtype_ok(dtype), LOOP_ERR_INVALID_ARG, "bad dtype");
  REQUIRE(M >= 0 && H > 0 && dv > 0, LOOP_ERR_INVALID_ARG, "bad size");
  if (M == 0) return LOOP_OK;
  REQUIRE(o && z && w && y, LOOP_ERR_INVALID_ARG, "NULL argument");
  REQUIRE(dv % 32 == 0 && dv <= 256, LOOP_ERR_UNSUPPORTED, "dv must be a multiple of 32, <= 256");
  REQUIRE(ld_z >= H * dv, LOOP_ERR_SHAPE, "ld_z smaller than H*dv");
  return launched(lk::gdn_gated_norm(o, z, ld_z, w, y, M, H, dv, eps, dtype, S(stream)), "gdn_gated_norm");
}

loop_status gdn_in_proj(const void* x, int ldx, const void* w_in, const float* a_bias, const float* b_bias, void* q,
                        void* k, void* v, float* g, float* beta, int M, int d, int H, int dk, int dv, float eps,
                        int dtype, void* stream) {
  REQUIRE(dtype_ok(dtype), LOOP_ERR_INVALID_ARG, "bad dtype");
  REQUIRE(M >= 0 && d > 0 && H > 0, LOOP_ERR_INVALID_ARG, "bad size");
  if (M == 0) return LOOP_OK;
  REQUIRE(x && w_in && a_bias && b_bias && q && k && v && g && beta, LOOP_ERR_INVALID_ARG, "NULL argument");
  REQUIRE(ldx >= d, LOOP_ERR_SHAPE, "ldx < d");
  REQUIRE(dtype == LOOP_BF16 && M > 128 && dk == 128 && dv == 128 && H % 2 == 0 && H <= 16 && d % 8 == 0,
          LOOP_ERR_UNSUPPORTED, "built for bf16, M > 128, dk = dv = 128, even H <= 16, d a multiple of 8");
  const GdnEpi ep{q, k, v, g, beta, a_bias, b_bias, eps, H};
  return launched(linear_gdn(x, ldx, w_in, M, d, ep, S(stream)), "gdn_in_proj");
}

loop_status gdn_prep(const void* P, int ld_p, const float* a_bias, const float* b_bias, void* q, void* k, void* v,
                     float* g, float* beta, int M, int H, int dk, int dv, float eps, int dtype, void* stream) {
  REQUIRE(dtype_ok(dtype), LOOP_ERR_INVALID_ARG, "bad dtype");
  REQUIRE(M >= 0 && H > 0 && dk > 0 && dv > 0, LOOP_ERR_INVALID_ARG, "bad size");
  if (M == 0) return LOOP_OK;
  REQUIRE(P && a_bias && b_bias && q && k && v && g && beta, LOOP_ERR_INVALID_ARG, "NULL argument");
  REQUIRE(ld_p >= 2 * H * dk + H * dv + 2 * H, LOOP_ERR_SHAPE, "ld_p smaller than the projection width");
  return launched(lk::gdn_prep(P, ld_p, a_bias, b_bias, q, k, v, g, beta, M, H, dk, dv, eps, dtype, S(stream)),
                  "gdn_prep");
}

size_t loop_gqa_workspace_bytes(int B, int Tq, int Tkv, int Hq, int dh) {
  if (B <= 0 || Tq <= 0 || Tkv <= 0 || Hq <= 0 || dh <= 0) return 0;
  return gqa_workspace_bytes(B, Tq, Tkv, Hq, dh);
}

loop_status gqa_attn(const void* q, int ld_q, const void* k, const void* v, int kv_cap, const void* gate, int ld_gate,
                     void* out, int B, int Tq, int Tkv, int q_off, int Hq, int Hkv, int dh, int causal,
                     void* workspace, int dtype, void* stream) {
  bool empty = false;
  loop_status st = gqa_check_args("gqa_attn", q, ld_q, k, v, kv_cap, gate, ld_gate, out, B, Tq, Tkv, q_off, Hq, Hkv, dh,
                                  causal, dtype, &empty);
  if (st != LOOP_OK || empty) return st;
  return launched(lk::gqa_attn(q, ld_q, k, v, kv_cap, gate, ld_gate, out, B, Tq, Tkv, q_off, Hq, Hkv, dh, causal,
                               workspace, dtype, S(stream)),
                  "gqa_attn");
}

loop_status gqa_attn_fused_q(const void* q, int ld_q, const void* q_norm, int rotary_dims, float rope_base, float eps,
                             const void* k, const void* v, int kv_cap, const void* gate, int ld_gate, void* out, int B,
                             int Tq, int Tkv, int q_off, int Hq, int Hkv, int dh, int causal, int dtype, void* stream) {
  bool empty = false;
  loop_status st = gqa_check_args("gqa_attn_fused_q", q, ld_q, k, v, kv_cap, gate, ld_gate, out, B, Tq, Tkv, q_off, Hq,
                                  Hkv, dh, causal, dtype, &empty);
  if (st != LOOP_OK || empty) return st;
  REQUIRE(q_norm, LOOP_ERR_INVALID_ARG, "q_norm is NULL");
  REQUIRE(rotary_dims >= 0 && rotary_dims % 2 == 0 && rotary_dims <= dh / 2, LOOP_ERR_INVALID_ARG,
          "rotary_dims must be even and <= dh / 2");
  REQUIRE(eps >= 0.f && rope_base > 0.f, LOOP_ERR_INVALID_ARG, "eps >= 0 and rope_base > 0 required");
  const QNorm qn{q_norm, rotary_dims, rope_base, eps, nullptr, 0};
  return launched(lk::gqa_attn(q, ld_q, k, v, kv_cap, gate, ld_gate, out, B, Tq, Tkv, q_off, Hq, Hkv, dh, causal,
                               nullptr, dtype, S(stream), &qn),
                  "gqa_attn_fused_q");
}

loop_status fa_prep(const void* P, int ld_p, const void* q_norm, const void* k_norm, void* q_out, void* k_cache,
                    void* v_cache, int kv_cap, int B, int T, int pos0, int Hq, int Hkv, int dh, int rotary_dims,
                    float rope_base, float eps, int dtype, void* stream) {
  REQUIRE(dtype_ok(dtype), LOOP_ERR_INVALID_ARG, "bad dtype");
  REQUIRE(B >= 0 && T >= 0 && pos0 >= 0, LOOP_ERR_INVALID_ARG, "negative size");
  if (B == 0 || T == 0) return LOOP_OK;
  REQUIRE(P && q_norm && k_norm && k_cache && v_cache, LOOP_ERR_INVALID_ARG, "NULL argument");
  REQUIRE(gqa_supported(dh, Hq, Hkv), LOOP_ERR_UNSUPPORTED, "head dim or head ratio not supported");
  REQUIRE(pos0 + T <= kv_cap, LOOP_ERR_CAPACITY, "positions past the slab capacity");
  REQUIRE(ld_p >= 2 * Hq * dh + 2 * Hkv * dh, LOOP_ERR_SHAPE, "ld_p smaller than the projection width");
  REQUIRE(rotary_dims >= 0 && rotary_dims <= dh && rotary_dims % 2 == 0, LOOP_ERR_INVALID_ARG, "bad rotary_dims");
  return launched(lk::fa_prep(P, ld_p, q_norm, k_norm, q_out, k_cache, v_cache, kv_cap, B, T, pos0, Hq, Hkv, dh,
                              rotary_dims, rope_base, eps, dtype, S(stream)),
                  "fa_prep");
}

loop_status mhc_route_mix(int mode, const void* X_in, const void* F, const float* coeffs_in, const float* w_r,
                          const float* b_r, void* X_out, void* x_in, void* h_out, float* coeffs_out, int N, int d,
                          float eps, int iters, int dtype, void* stream) {
  REQUIRE(dtype_ok(dtype), LOOP_ERR_INVALID_ARG, "bad dtype");
  REQUIRE(mode >= MHC_OPEN && mode <= MHC_MERGE, LOOP_ERR_INVALID_ARG, "mode must be 0..3");
  REQUIRE(N >= 0 && d > 0 && iters >= 0, LOOP_ERR_INVALID_ARG, "bad size");
  REQUIRE(d % 8 == 0, LOOP_ERR_SHAPE, "d must be a multiple of 8");
  if (N == 0) return LOOP_OK;
  REQUIRE(X_in, LOOP_ERR_INVALID_ARG, "X_in is NULL");
  if (mode == MHC_MIX || mode == MHC_MERGE) REQUIRE(F && coeffs_in, LOOP_ERR_INVALID_ARG, "MIX/MERGE need F, coeffs_in");
  if (mode == MHC_MERGE) REQUIRE(h_out, LOOP_ERR_INVALID_ARG, "MERGE needs h_out");
  if (mode != MHC_MERGE) REQUIRE(w_r && b_r && x_in && coeffs_out, LOOP_ERR_INVALID_ARG, "routing needs w_r, b_r, x_in, coeffs_out");
  if (mode == MHC_OPEN || mode == MHC_MIX) REQUIRE(X_out, LOOP_ERR_INVALID_ARG, "OPEN/MIX need X_out");
  const void* ptrs[] = {X_in, F, coeffs_in, X_out, x_in, h_out, coeffs_out};
  for (const void* p : ptrs)
    REQUIRE(((uintptr_t)p & 15) == 0, LOOP_ERR_INVALID_ARG, "mhc_route_mix: array pointers must be 16-byte aligned");
  return launched(mhc(mode, X_in, F, coeffs_in, w_r, b_r, X_out, x_in, h_out, coeffs_out, N, d, eps, iters, dtype,
                      S(stream)),
                  "mhc_route_mix");
}

loop_status sinkhorn_fp32(const float* logits, float* out, int N, int n, int iters, void* stream) {
  REQUIRE(N >= 0 && n >= 1 && n <= 8 && iters >= 0, LOOP_ERR_INVALID_ARG, "need N >= 0, 1 <= n <= 8, iters >= 0");
  if (N == 0) return LOOP_OK;
  REQUIRE(logits && out, LOOP_ERR_INVALID_ARG, "NULL argument");
  return launched(sinkhorn(logits, out, N, n, iters, S(stream)), "sinkhorn_fp32");
}

size_t loop_linear_workspace_bytes(int M, int N, int K, int epilogue) {
  if (M <= 0 || N <= 0 || K <= 0 || epilogue < EPI_STORE || epilogue > EPI_F32) return 0;
  return linear_workspace_bytes(M, N, K, epilogue);
}

loop_status loop_linear(const void* X, int ldx, const void* W, const void* W2, const void* R, int ldr, void* Y,
                        int ldy, int M, int N, int K, int epilogue, void* workspace, int dtype, void* stream) {
  REQUIRE(dtype_ok(dtype), LOOP_ERR_INVALID_ARG, "bad dtype");
  REQUIRE(epilogue >= EPI_STORE && epilogue <= EPI_F32, LOOP_ERR_INVALID_ARG, "epilogue must be 0..3");
  REQUIRE(M >= 0 && N >= 0 && K > 0, LOOP_ERR_INVALID_ARG, "bad size");
  if (M == 0 || N == 0) return LOOP_OK;
  REQUIRE(X && W && Y, LOOP_ERR_INVALID_ARG, "NULL argument");
  REQUIRE(ldx >= K && ldy >= N, LOOP_ERR_SHAPE, "row stride smaller than the row");
  if (epilogue == EPI_ADD) REQUIRE(R && ldr >= N, LOOP_ERR_INVALID_ARG, "ADD needs R with ldr >= N");
  if (epilogue == EPI_SWIGLU) REQUIRE(W2, LOOP_ERR_INVALID_ARG, "SWIGLU needs W2");
  if (dtype == LOOP_BF16) REQUIRE(K % 8 == 0 && ldx % 8 == 0, LOOP_ERR_SHAPE, "bf16 needs K and ldx multiples of 8");
  const size_t ws_bytes = workspace ? linear_workspace_bytes(M, N, K, epilogue) : 0;
  return launched(linear(X, ldx, W, W2, R, ldr, Y, ldy, M, N, K, epilogue, dtype, S(stream), workspace, ws_bytes),
                  "loop_linear");
}

loop_status loop_rmsnorm(const void* x, const void* r, void* sum_out, const void* w, void* y, int M, int d, float eps,
                         int dtype, void* stream) {
  REQUIRE(x && w && y, LOOP_ERR_INVALID_ARG, "NULL argument");
  REQUIRE(dtype_ok(dtype), LOOP_ERR_INVALID_ARG, "bad dtype");
  REQUIRE(M >= 0 && d > 0 && d % 8 == 0, LOOP_ERR_SHAPE, "d must be a positive multiple of 8");
  return launched(rmsnorm(x, r, sum_out, w, y, M, d, eps, dtype, S(stream)), "loop_rmsnorm");
}

loop_status loop_embed(const int32_t* ids, const void* embed, void* out, int M, int d, int vocab, int dtype,
                       void* stream) {
  REQUIRE(ids && embed && out, LOOP_ERR_INVALID_ARG, "NULL argument");
  REQUIRE(dtype_ok(dtype), LOOP_ERR_INVALID_ARG, "bad dtype");
  REQUIRE(M >= 0 && vocab > 0 && d > 0 && d % 8 == 0, LOOP_ERR_SHAPE, "d must be a positive multiple of 8");
  return launched(lk::embed(ids, embed, out, M, d, vocab, dtype, S(stream)), "loop_embed");
}

loop_status loop_argmax(const float* logits, int32_t* next, int B, int V, void* stream) {
  REQUIRE(logits && next, LOOP_ERR_INVALID_ARG, "NULL argument");
  REQUIRE(B >= 0 && V > 0, LOOP_ERR_INVALID_ARG, "bad size");
  return launched(lk::argmax(logits, next, B, V, S(stream)), "loop_argmax");
}

}  // extern "C"
