// Model runtime for the looped hybrid decoder ("Loop-9B engineering teardown" §二-§六).
//
// Schedule: head layers once, the loop block loop_passes times with the same weights
// (B(B(h))), tail layers once.  Cache manager: every execution owns its cache slot
// (§四): FA executions a KV slab each, GDN executions a state each.  Forward: per
// execution, pre-norm mixer + SwiGLU FFN; inside the loop block the two-stream mHC
// kernel runs once per layer boundary (open -> mix+route ... -> merge, §六).
#include <cmath>
#include <cstring>

#include "common.cuh"
#include "runtime.h"

using namespace lk;

static thread_local std::string g_last_error;

loop_status fail(loop_status st, const std::string& msg) {
  g_last_error = msg;
  return st;
}
loop_status cuda_fail(cudaError_t e, const char* what) {
  g_last_error = std::string(what) + ": " + cudaGetErrorString(e);
  return e == cudaErrorMemoryAllocation ? LOOP_ERR_OOM : LOOP_ERR_CUDA;
}
extern "C" const char* loop_last_error(void) { return g_last_error.c_str(); }

DevBuf::~DevBuf() {
  if (p) cudaFree(p);
}
cudaError_t DevBuf::ensure(size_t want) {
  if (want <= bytes) return cudaSuccess;
  if (p) cudaFree(p);
  p = nullptr;
  bytes = 0;
  cudaError_t e = cudaMalloc(&p, want);
  if (e == cudaSuccess) bytes = want;
  return e;
}

std::vector<ExecRow> build_schedule(const loop_config& c) {
  std::vector<ExecRow> rows;
  int e = 0, n_fa = 0, n_gdn = 0;
  auto push = [&](int layer, int in_loop) {
    const int kind = (layer % c.group == c.group - 1) ? 1 : 0;
    const int slot = kind ? n_fa++ : n_gdn++;
    rows.push_back({e++, layer, kind, slot, in_loop});
  };
  for (int l = 0; l < c.loop_start; ++l) push(l, 0);
  for (int p = 0; p < c.loop_passes; ++p)
    for (int l = c.loop_start; l < c.loop_end; ++l) push(l, 1);
  for (int l = c.loop_end; l < c.n_layers; ++l) push(l, 0);
  return rows;
}

// ------------------------------------------------------------------ workspace
static loop_status ensure_workspace(loop_model* m, long M, int B, int Tq, int Tkv_max) {
  const loop_config& c = m->cfg;
  const size_t es = m->esize;
  const int d = c.d;
  const int n_in = m->in_gdn > m->in_fa ? m->in_gdn : m->in_fa;
  const int o_w = std::max(c.gdn_heads * c.gdn_dv, c.fa_q_heads * c.fa_head_dim);
  struct Need { DevBuf* b; size_t bytes; } need[] = {
      {&m->h, M * d * es},
      {&m->X, M * c.mhc_streams * d * es},
      {&m->x_in, M * d * es},
      {&m->xn, M * d * es},
      {&m->proj, M * n_in * es},
      {&m->gq, M * std::max(c.gdn_heads * c.gdn_dk, c.fa_q_heads * c.fa_head_dim) * es},
      {&m->gk, M * c.gdn_heads * c.gdn_dk * es},
      {&m->gv, M * c.gdn_heads * c.gdn_dv * es},
      {&m->gg, M * c.gdn_heads * sizeof(float)},
      {&m->gb, M * c.gdn_heads * sizeof(float)},
      {&m->o, M * o_w * es},
      {&m->mix, M * d * es},
      {&m->u, M * d * es},
      {&m->un, M * d * es},
      {&m->act, M * c.ffn * es},
      {&m->F, M * d * es},
      {&m->coeffs, M * 8 * sizeof(float)},
      {&m->attn_ws, gqa_workspace_bytes(B, Tq, Tkv_max, c.fa_q_heads, c.fa_head_dim)},
      {&m->last, (size_t)B * d * es},
  };
  for (auto& n : need) {
    cudaError_t e = n.b->ensure(n.bytes < 256 ? 256 : n.bytes);
    if (e != cudaSuccess) return cuda_fail(e, "workspace allocation");
  }
  if (M > m->ws_tokens) m->ws_tokens = M;
  return LOOP_OK;
}

#define CK(call, what)                                  \
  do {                                                  \
    cudaError_t e_ = (call);                            \
    if (e_ != cudaSuccess) return cuda_fail(e_, what);  \
  } while (0)

// ------------------------------------------------------------------ one decoder layer
// x [M, d] -> writes the layer's result: plain layers h = x + F (into `h_out`),
// looped layers F = mix + f (into m->F).  pos0 = cache length before these tokens.
static loop_status run_layer(loop_model* m, loop_cache* c, const ExecRow& r, const void* x, void* h_out,
                             int B, int T, int pos0, cudaStream_t s) {
  const loop_config& cf = m->cfg;
  const loop_layer_weights& w = m->layers[r.layer];
  const long M = (long)B * T;
  const int d = cf.d, dt = cf.dtype;
  CK(rmsnorm(x, nullptr, nullptr, w.attn_norm, m->xn.p, (int)M, d, cf.eps, dt, s), "rmsnorm (mixer)");
  if (r.kind == 0) {
    const int H = cf.gdn_heads, dk = cf.gdn_dk, dv = cf.gdn_dv;
    CK(linear(m->xn.p, d, w.w_in, nullptr, nullptr, 0, m->proj.p, m->in_gdn, (int)M, m->in_gdn, d, EPI_STORE, dt, s),
       "GDN input projection");
    CK(lk::gdn_prep(m->proj.p, m->in_gdn, w.gdn_a_bias, w.gdn_b_bias, m->gq.p, m->gk.p, m->gv.p, (float*)m->gg.p,
                (float*)m->gb.p, (int)M, H, dk, dv, cf.eps, dt, s),
       "GDN prep");
    float* S = (float*)c->state.p + (size_t)r.slot * c->state_elems;
    const float scale = 1.f / std::sqrt((float)dk);
    if (T == 1)
      CK(lk::gdn_step(m->gq.p, m->gk.p, m->gv.p, (float*)m->gg.p, (float*)m->gb.p, S, m->o.p, B, H, dk, dv, scale, dt, s),
         "GDN step");
    else
      CK(gdn_chunk(m->gq.p, m->gk.p, m->gv.p, (float*)m->gg.p, (float*)m->gb.p, S, m->o.p, B, T, H, dk, dv, scale,
                   dt, s),
         "GDN chunked scan");
    CK(linear(m->o.p, H * dv, w.w_out, nullptr, nullptr, 0, m->mix.p, d, (int)M, d, H * dv, EPI_STORE, dt, s),
       "GDN output projection");
  } else {
    const int Hq = cf.fa_q_heads, Hkv = cf.fa_kv_heads, dh = cf.fa_head_dim;
    CK(linear(m->xn.p, d, w.w_in, nullptr, nullptr, 0, m->proj.p, m->in_fa, (int)M, m->in_fa, d, EPI_STORE, dt, s),
       "FA input projection");
    char* kbase = (char*)c->kv.p + (size_t)r.slot * 2 * c->kv_slab_elems * m->esize;
    char* vbase = kbase + c->kv_slab_elems * m->esize;
    CK(lk::fa_prep(m->proj.p, m->in_fa, w.q_norm, w.k_norm, m->gq.p, kbase, vbase, c->max_tokens, B, T, pos0, Hq, Hkv, dh,
               cf.rotary_dims, cf.rope_base, cf.eps, dt, s),
       "QK-norm / rotary / KV write");
    const char* gate = (const char*)m->proj.p + (size_t)Hq * dh * m->esize;
    CK(lk::gqa_attn(m->gq.p, Hq * dh, kbase, vbase, c->max_tokens, gate, m->in_fa, m->o.p, B, T, pos0 + T, pos0, Hq, Hkv,
                dh, 1, m->attn_ws.p, dt, s),
       "GQA attention");
    CK(linear(m->o.p, Hq * dh, w.w_out, nullptr, nullptr, 0, m->mix.p, d, (int)M, d, Hq * dh, EPI_STORE, dt, s),
       "FA output projection");
  }
  // u = x + mix; FFN on RMSNorm(u)
  CK(rmsnorm(x, m->mix.p, m->u.p, w.ffn_norm, m->un.p, (int)M, d, cf.eps, dt, s), "rmsnorm (FFN)");
  CK(linear(m->un.p, d, w.w_gate, w.w_up, nullptr, 0, m->act.p, cf.ffn, (int)M, cf.ffn, d, EPI_SWIGLU, dt, s),
     "FFN gate/up (SwiGLU)");
  if (r.in_loop)
    CK(linear(m->act.p, cf.ffn, w.w_down, nullptr, m->mix.p, d, m->F.p, d, (int)M, d, cf.ffn, EPI_ADD, dt, s),
       "FFN down (+ mixer output)");
  else
    CK(linear(m->act.p, cf.ffn, w.w_down, nullptr, m->u.p, d, h_out, d, (int)M, d, cf.ffn, EPI_ADD, dt, s),
       "FFN down (+ residual)");
  return LOOP_OK;
}

// All executions over M = B*T new tokens whose hidden states are in m->h.
static loop_status run_stack(loop_model* m, loop_cache* c, int B, int T, cudaStream_t s) {
  const loop_config& cf = m->cfg;
  const long M = (long)B * T;
  const int pos0 = c->len;
  const int dt = cf.dtype;
  for (size_t i = 0; i < m->sched.size(); ++i) {
    const ExecRow& r = m->sched[i];
    if (!r.in_loop) {
      loop_status st = run_layer(m, c, r, m->h.p, m->h.p, B, T, pos0, s);
      if (st != LOOP_OK) return st;
      continue;
    }
    const loop_layer_weights& w = m->layers[r.layer];
    if (r.exec == m->first_loop)
      CK(mhc(MHC_OPEN, m->h.p, nullptr, nullptr, w.mhc_w_r, w.mhc_b_r, m->X.p, m->x_in.p, nullptr, (float*)m->coeffs.p,
             (int)M, cf.d, cf.eps, cf.sinkhorn_iters, dt, s),
         "mHC open");
    loop_status st = run_layer(m, c, r, m->x_in.p, nullptr, B, T, pos0, s);
    if (st != LOOP_OK) return st;
    if (r.exec == m->last_loop) {
      CK(mhc(MHC_MERGE, m->X.p, m->F.p, (float*)m->coeffs.p, nullptr, nullptr, nullptr, nullptr, m->h.p, nullptr,
             (int)M, cf.d, cf.eps, cf.sinkhorn_iters, dt, s),
         "mHC merge");
    } else {
      const loop_layer_weights& wn = m->layers[m->sched[i + 1].layer];
      CK(mhc(MHC_MIX, m->X.p, m->F.p, (float*)m->coeffs.p, wn.mhc_w_r, wn.mhc_b_r, m->X.p, m->x_in.p, nullptr,
             (float*)m->coeffs.p, (int)M, cf.d, cf.eps, cf.sinkhorn_iters, dt, s),
         "mHC mix + route");
    }
  }
  return LOOP_OK;
}

loop_status run_forward(loop_model* m, loop_cache* c, const int32_t* ids, const void* h_in, void* h_out,
                        float* logits_last, int B, int T, cudaStream_t s) {
  const loop_config& cf = m->cfg;
  const long M = (long)B * T;
  loop_status st = ensure_workspace(m, M, B, T, c->max_tokens);
  if (st != LOOP_OK) return st;
  if (ids)
    CK(embed(ids, m->embed, m->h.p, (int)M, cf.d, cf.vocab, cf.dtype, s), "embedding");
  else
    CK(cudaMemcpyAsync(m->h.p, h_in, M * cf.d * m->esize, cudaMemcpyDeviceToDevice, s), "hidden-state input copy");
  st = run_stack(m, c, B, T, s);
  if (st != LOOP_OK) return st;
  c->len += T;
  if (h_out) CK(cudaMemcpyAsync(h_out, m->h.p, M * cf.d * m->esize, cudaMemcpyDeviceToDevice, s), "hidden-state output copy");
  if (logits_last) {
    // final norm of each sequence's last position, then the LM head
    const char* last = (const char*)m->h.p + (size_t)(T - 1) * cf.d * m->esize;
    CK(rmsnorm(last, nullptr, nullptr, m->final_norm, m->last.p, B, cf.d, cf.eps, cf.dtype, s, (long)T * cf.d),
       "final norm");
    CK(linear(m->last.p, cf.d, m->lm_head, nullptr, nullptr, 0, logits_last, cf.vocab, B, cf.vocab, cf.d, EPI_F32,
              cf.dtype, s),
       "LM head");
  }
  return LOOP_OK;
}

loop_status run_decode(loop_model* m, loop_cache* c, const int32_t* tok, float* logits, int32_t* next,
                       cudaStream_t s) {
  const loop_config& cf = m->cfg;
  const int B = c->batch;
  loop_status st = ensure_workspace(m, B, B, 1, c->max_tokens);
  if (st != LOOP_OK) return st;
  // logits go to the caller's buffer if given, else to a workspace buffer
  float* lg = logits;
  if (!lg) {
    static thread_local DevBuf tmp;
    CK(tmp.ensure((size_t)B * cf.vocab * sizeof(float)), "logits buffer");
    lg = (float*)tmp.p;
  }
  CK(embed(tok, m->embed, m->h.p, B, cf.d, cf.vocab, cf.dtype, s), "embedding");
  st = run_stack(m, c, B, 1, s);
  if (st != LOOP_OK) return st;
  c->len += 1;
  CK(rmsnorm(m->h.p, nullptr, nullptr, m->final_norm, m->last.p, B, cf.d, cf.eps, cf.dtype, s), "final norm");
  CK(linear(m->last.p, cf.d, m->lm_head, nullptr, nullptr, 0, lg, cf.vocab, B, cf.vocab, cf.d, EPI_F32, cf.dtype, s),
     "LM head");
  CK(argmax(lg, next, B, cf.vocab, s), "argmax");
  return LOOP_OK;
}
