// Model runtime for the looped hybrid decoder ("Loop-9B engineering teardown" §二-§六).
//
// Schedule: head layers once, the loop block loop_passes times with the same weights
// (B(B(h))), tail layers once.  Cache manager: every execution owns its cache slot
// (§四): FA executions a KV slab each, GDN executions a state each.  Forward: per
// execution, pre-norm mixer + SwiGLU FFN; inside the loop block the two-stream mHC
// kernel runs once per layer boundary (open -> mix+route ... -> merge, §六).
#include <cmath>
#include <cstdio>
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

const char* const kProfNames[P_NCAT] = {"gemm", "lm_head", "rmsnorm", "embed", "gdn_prep", "gdn_chunk", "gdn_step",
                                        "fa_prep", "attention", "mhc", "argmax", "copy", "gdn_norm"};

Profiler::~Profiler() {
  clear();
  for (auto e : pool) cudaEventDestroy(e);
}
cudaEvent_t Profiler::get() {
  if (pool.empty()) {
    cudaEvent_t e;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    return e;
  }
  cudaEvent_t e = pool.back();
  pool.pop_back();
  return e;
}
void Profiler::clear() {
  for (auto& r : recs) {
    pool.push_back(r.a);
    pool.push_back(r.b);
  }
  recs.clear();
}

// Run `launch` (returns cudaError_t); with profiling on, bracket it with events and
// record its algorithmic work.
template <typename F>
static cudaError_t prof(loop_model* m, cudaStream_t s, int cat, int launches, double flops, double bytes, F&& launch) {
  if (!m->prof.on) return launch();
  ProfRec r{cat, launches, m->prof.get(), m->prof.get(), flops, bytes};
  if (!r.a || !r.b) return cudaErrorMemoryAllocation;
  cudaEventRecord(r.a, s);
  cudaError_t e = launch();
  cudaEventRecord(r.b, s);
  m->prof.recs.push_back(r);
  return e;
}

// Algorithmic work of one projection launch (bf16 or fp32 storage).
static void gemm_work(long M, long N, long K, int epi, size_t es, double& flops, double& bytes) {
  const long n_mat = epi == EPI_SWIGLU ? 2 : 1;
  flops = 2.0 * M * N * K * n_mat;
  bytes = (double)es * (M * K + n_mat * N * K) + (epi == EPI_F32 ? 4.0 : (double)es) * M * N +
          (epi == EPI_ADD ? (double)es * M * N : 0.0);
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

#define CK(call, what)                                  \
  do {                                                  \
    cudaError_t e_ = (call);                            \
    if (e_ != cudaSuccess) return cuda_fail(e_, what);  \
  } while (0)

// ------------------------------------------------------------------ workspace
static loop_status ensure_workspace(loop_model* m, long M, int B, int Tq, int Tkv_max, cudaStream_t s) {
  const loop_config& c = m->cfg;
  const size_t es = m->esize;
  const int d = c.d;
  const int n_in = m->in_gdn > m->in_fa ? m->in_gdn : m->in_fa;
  const int Hv = m->gdn_hv;
  const int o_w = std::max(Hv * c.gdn_dv, c.fa_q_heads * c.fa_head_dim);
  struct Need { DevBuf* b; size_t bytes; } need[] = {
      {&m->h, M * d * es},
      {&m->X, M * c.mhc_streams * d * es},
      {&m->x_in, M * d * es},
      {&m->xn, M * d * es},
      {&m->proj, M * n_in * es},
      {&m->gq, M * std::max(Hv * c.gdn_dk, c.fa_q_heads * c.fa_head_dim) * es},
      {&m->gk, M * Hv * c.gdn_dk * es},
      {&m->gv, M * Hv * c.gdn_dv * es},
      {&m->gg, M * Hv * sizeof(float)},
      {&m->gb, M * Hv * sizeof(float)},
      {&m->o, M * o_w * es},
      {&m->mix, M * d * es},
      {&m->u, M * d * es},
      {&m->un, M * d * es},
      {&m->act, M * c.ffn * es},
      {&m->F, M * d * es},
      {&m->coeffs, M * 8 * sizeof(float)},
      {&m->rope, (size_t)Tq * (c.rotary_dims / 2) * sizeof(float2)},
      {&m->attn_ws, gqa_scratch_bytes(B, Tq, Tkv_max, c.fa_q_heads, c.fa_kv_heads, c.fa_head_dim, c.dtype)},
      {&m->gdn_ws, Tq > 1 ? gdn_workspace_bytes(B, Tq, Hv, c.gdn_dk, c.gdn_dv) : 0},
      {&m->last, (size_t)B * d * es},
  };
  for (auto& n : need) {
    cudaError_t e = n.b->ensure(n.bytes < 256 ? 256 : n.bytes);
    if (e != cudaSuccess) return cuda_fail(e, "workspace allocation");
  }
  // partial sums of projections with few rows (<= 128): the layer projections of these
  // tokens and the LM head on each sequence's last position; zero-filled once, and every
  // projection leaves it zero-filled
  size_t gws = 0;
  if (M <= 128) {
    const int ns[4][2] = {{m->in_gdn, EPI_STORE}, {m->in_fa, EPI_STORE}, {d, EPI_ADD}, {c.ffn, EPI_SWIGLU}};
    for (auto& n : ns) gws = std::max(gws, linear_workspace_bytes((int)M, n[0], d, n[1]));
  }
  if (B <= 128) gws = std::max(gws, linear_workspace_bytes(B, c.vocab, d, EPI_F32));
  if (gws > m->gemm_ws.bytes) {
    CK(m->gemm_ws.ensure(gws), "projection workspace allocation");
    CK(cudaMemsetAsync(m->gemm_ws.p, 0, m->gemm_ws.bytes, s), "projection workspace zero fill");
  }
  if (M > m->ws_tokens) m->ws_tokens = M;
  return LOOP_OK;
}

// ------------------------------------------------------------------ one decoder layer
// x [M, d] -> writes the layer's result: plain layers h = x + F (into `h_out`),
// looped layers F = mix + f (into m->F).  pos0 = cache length before these tokens.
static loop_status run_layer(loop_model* m, loop_cache* c, const ExecRow& r, const void* x, void* h_out,
                             int B, int T, int pos0, cudaStream_t s) {
  const loop_config& cf = m->cfg;
  const loop_layer_weights& w = m->layers[r.layer];
  const long M = (long)B * T;
  const int d = cf.d, dt = cf.dtype;
  const double es = (double)m->esize;
  double fl, by;
  CK(prof(m, s, P_RMSNORM, 1, 0, es * (2.0 * M * d + d),
          [&] { return rmsnorm(x, nullptr, nullptr, w.attn_norm, m->xn.p, (int)M, d, cf.eps, dt, s); }),
     "rmsnorm (mixer)");
  if (r.kind == 0) {
    // H: heads of the recurrence (the variant's value heads); Hk: key heads
    const int H = m->gdn_hv, Hk = cf.gdn_heads, dk = cf.gdn_dk, dv = cf.gdn_dv;
    const bool variant = cf.gdn_variant == 1;
    // prefill-sized bf16 batches: the preparation (L2 norms, gates) runs in the projection's
    // epilogue, so the projection is never stored
    const bool fused_prep = !variant && dt == BF16 && M > 128 && dk == 128 && dv == 128 && H % 2 == 0 && H <= 16;
    gemm_work(M, m->in_gdn, d, EPI_STORE, m->esize, fl, by);
    if (fused_prep) {
      const GdnEpi ep{m->gq.p, m->gk.p, m->gv.p, (float*)m->gg.p, (float*)m->gb.p, w.gdn_a_bias, w.gdn_b_bias,
                      cf.eps, H};
      CK(prof(m, s, P_GEMM, 1, fl, by, [&] { return linear_gdn(m->xn.p, d, w.w_in, (int)M, d, ep, s); }),
         "GDN input projection + preparation");
    } else {
      CK(prof(m, s, P_GEMM, 1, fl, by,
              [&] { return linear(m->xn.p, d, w.w_in, nullptr, nullptr, 0, m->proj.p, m->in_gdn, (int)M, m->in_gdn,
                                  d, EPI_STORE, dt, s, m->gemm_ws.p, m->gemm_ws.bytes); }),
         "GDN input projection");
    }
    // the decode step reads the stored projection itself (norms and gates inside the step)
    const bool step_from_proj = !fused_prep && !variant && T == 1;
    if (fused_prep || step_from_proj) {
    } else if (variant) {
      void* conv_state = (char*)c->conv.p + (size_t)r.slot * c->conv_elems * m->esize;
      // P's q | k | v channels read conv times, the conv inputs before this call, outputs once
      const double bytes = (double)M * (es * (cf.gdn_conv * (double)m->gdn_ch + 2.0 * H * dk + H * dv) + 16.0 * H) +
                           4.0 * B * (cf.gdn_conv - 1) * m->gdn_ch * es;
      CK(prof(m, s, P_GDN_PREP, 2, 0, bytes,
              [&] { return lk::gdn_conv_prep(m->proj.p, m->in_gdn, w.gdn_conv_w, conv_state, w.gdn_a_bias,
                                             w.gdn_b_bias, m->gq.p, m->gk.p, m->gv.p, (float*)m->gg.p, (float*)m->gb.p,
                                             B, T, Hk, H, dk, dv, cf.gdn_conv, cf.eps, dt, s); }),
         "GDN conv prep");
    } else {
      CK(prof(m, s, P_GDN_PREP, 1, 0, (double)M * (es * (m->in_gdn + 2.0 * H * dk + H * dv) + 8.0 * H),
              [&] { return lk::gdn_prep(m->proj.p, m->in_gdn, w.gdn_a_bias, w.gdn_b_bias, m->gq.p, m->gk.p, m->gv.p,
                                        (float*)m->gg.p, (float*)m->gb.p, (int)M, H, dk, dv, cf.eps, dt, s); }),
         "GDN prep");
    }
    float* S = (float*)c->state.p + (size_t)r.slot * c->state_elems;
    const float scale = 1.f / std::sqrt((float)dk);
    // bytes: q, k, v in, o out, gates, and the fp32 state read + written once
    const double st_bytes = 8.0 * B * H * dk * dv;
    const double io_bytes = (double)M * H * (es * (2.0 * dk + 2.0 * dv) + 8.0);
    if (step_from_proj)
      CK(prof(m, s, P_GDN_STEP, 1, 6.0 * B * H * dk * dv,
              (double)M * (es * (2.0 * H * dk + H * dv + 2.0 * H + H * dv)) + st_bytes,
              [&] { return lk::gdn_step_proj(m->proj.p, m->in_gdn, w.gdn_a_bias, w.gdn_b_bias, cf.eps, S, m->o.p, B, H,
                                             dk, dv, scale, dt, s); }),
         "GDN step");
    else if (T == 1)
      CK(prof(m, s, P_GDN_STEP, 1, 6.0 * B * H * dk * dv, io_bytes + st_bytes,
              [&] { return lk::gdn_step(m->gq.p, m->gk.p, m->gv.p, (float*)m->gg.p, (float*)m->gb.p, S, m->o.p, B, H,
                                        dk, dv, scale, dt, s); }),
         "GDN step");
    else {
      // flops of the chunked form per 64-token chunk and head (A and P, substitution, U, O, state)
      const double C = 64.0, chunks = (double)B * H * ((T + 63) / 64);
      const double per_chunk = 2.0 * C * C * dk + C * C * (dk + dv) + 2.0 * C * dk * dv * 3 + C * C * dv;
      CK(prof(m, s, P_GDN_CHUNK, 2, chunks * per_chunk, io_bytes + st_bytes,
              [&] { return gdn_chunk(m->gq.p, m->gk.p, m->gv.p, (float*)m->gg.p, (float*)m->gb.p, S, m->o.p, B, T, H,
                                     dk, dv, scale, dt, s, m->gdn_ws.p); }),
         "GDN chunked scan");
    }
    if (variant)   // in place: each head's output row is read whole before it is written
      CK(prof(m, s, P_GDN_NORM, 1, 0, (double)M * H * dv * es * 3.0,
              [&] { return lk::gdn_gated_norm(m->o.p, (const char*)m->proj.p + (size_t)m->gdn_ch * m->esize,
                                              m->in_gdn, w.gdn_o_norm, m->o.p, M, H, dv, cf.eps, dt, s); }),
         "GDN gated output norm");
    gemm_work(M, d, H * dv, EPI_STORE, m->esize, fl, by);
    CK(prof(m, s, P_GEMM, 1, fl, by,
            [&] { return linear(m->o.p, H * dv, w.w_out, nullptr, nullptr, 0, m->mix.p, d, (int)M, d, H * dv, EPI_STORE,
                                dt, s, m->gemm_ws.p, m->gemm_ws.bytes); }),
       "GDN output projection");
  } else {
    const int Hq = cf.fa_q_heads, Hkv = cf.fa_kv_heads, dh = cf.fa_head_dim;
    char* kbase = (char*)c->kv.p + (size_t)r.slot * 2 * c->kv_slab_elems * m->esize;
    char* vbase = kbase + c->kv_slab_elems * m->esize;
    const char* gate = (const char*)m->proj.p + (size_t)Hq * dh * m->esize;
    // prefill-sized bf16 batches: QK-norm, rotary and the KV write run in the projection's
    // epilogue (normed, rotated q to a compact buffer; k, v into the slab; the gate block to
    // its place in the projection buffer), so neither a preparation kernel nor a pass over
    // the queries remains
    auto al16 = [](const void* p) { return ((uintptr_t)p % 16) == 0; };
    const bool fused_fa = dt == BF16 && M > 128 && dh == 256 && cf.rotary_dims <= 64 && al16(w.w_in) &&
                          al16(w.q_norm) && al16(w.k_norm);
    // otherwise multi-token bf16 queries go raw to the tensor-core attention kernel, which
    // applies their QK-norm and rotary as it stages them; the prep kernel then writes K and V
    const bool fuse_q = !fused_fa && dt == BF16 && dh == 256 && T >= 16 && 128 % (Hq / Hkv) == 0 &&
                        cf.rotary_dims <= dh / 2;
    gemm_work(M, m->in_fa, d, EPI_STORE, m->esize, fl, by);
    if (fused_fa) {
      const FaEpi fe{m->gq.p, (void*)gate, m->in_fa, kbase, vbase, c->max_tokens, w.q_norm, w.k_norm, cf.eps, Hq, Hkv,
                     cf.rotary_dims, (const float2*)m->rope.p, T, pos0};
      CK(prof(m, s, P_GEMM, 1, fl, by, [&] { return linear_fa(m->xn.p, d, w.w_in, (int)M, d, fe, s); }),
         "FA input projection + QK-norm / rotary / KV write");
    } else {
      CK(prof(m, s, P_GEMM, 1, fl, by,
              [&] { return linear(m->xn.p, d, w.w_in, nullptr, nullptr, 0, m->proj.p, m->in_fa, (int)M, m->in_fa, d,
                                  EPI_STORE, dt, s, m->gemm_ws.p, m->gemm_ws.bytes); }),
         "FA input projection");
      CK(prof(m, s, P_FA_PREP, 1, 0, (double)M * es * (2.0 * ((fuse_q ? 0 : Hq) + 2 * Hkv) * dh),
              [&] { return lk::fa_prep(m->proj.p, m->in_fa, w.q_norm, w.k_norm, fuse_q ? nullptr : m->gq.p, kbase,
                                       vbase, c->max_tokens, B, T, pos0, Hq, Hkv, dh, cf.rotary_dims, cf.rope_base,
                                       cf.eps, dt, s, (const float2*)m->rope.p); }),
         "QK-norm / rotary / KV write");
    }
    // causal (query, key) pairs: sum over new tokens of (pos0 + t + 1)
    const double pairs = (double)B * ((double)T * pos0 + (double)T * (T + 1) / 2.0);
    const double attn_bytes = es * ((double)M * Hq * dh * 3.0 + (double)B * Hkv * (pos0 + T) * dh * 2.0);
    const QNorm qn{w.q_norm, cf.rotary_dims, cf.rope_base, cf.eps, (const float2*)m->rope.p, pos0};
    CK(prof(m, s, P_ATTN, gqa_launches(B, T, pos0 + T, Hq, Hkv, dh, dt, m->attn_ws.p != nullptr), 4.0 * Hq * dh * pairs, attn_bytes,
            [&] {
              return fuse_q ? lk::gqa_attn(m->proj.p, m->in_fa, kbase, vbase, c->max_tokens, gate, m->in_fa, m->o.p, B,
                                           T, pos0 + T, pos0, Hq, Hkv, dh, 1, nullptr, dt, s, &qn)
                            : lk::gqa_attn(m->gq.p, Hq * dh, kbase, vbase, c->max_tokens, gate, m->in_fa, m->o.p, B, T,
                                           pos0 + T, pos0, Hq, Hkv, dh, 1, m->attn_ws.p, dt, s);
            }),
       "GQA attention");
    gemm_work(M, d, Hq * dh, EPI_STORE, m->esize, fl, by);
    CK(prof(m, s, P_GEMM, 1, fl, by,
            [&] { return linear(m->o.p, Hq * dh, w.w_out, nullptr, nullptr, 0, m->mix.p, d, (int)M, d, Hq * dh,
                                EPI_STORE, dt, s, m->gemm_ws.p, m->gemm_ws.bytes); }),
       "FA output projection");
  }
  // u = x + mix; FFN on RMSNorm(u).  Only plain layers add f to u (h = u + f); looped
  // layers add it to mix (F = mix + f), so there u is not stored.
  void* u_out = r.in_loop ? nullptr : m->u.p;
  CK(prof(m, s, P_RMSNORM, 1, 0, es * ((u_out ? 4.0 : 3.0) * M * d + d),
          [&] { return rmsnorm(x, m->mix.p, u_out, w.ffn_norm, m->un.p, (int)M, d, cf.eps, dt, s); }),
     "rmsnorm (FFN)");
  gemm_work(M, cf.ffn, d, EPI_SWIGLU, m->esize, fl, by);
  CK(prof(m, s, P_GEMM, 1, fl, by,
          [&] { return linear(m->un.p, d, w.w_gate, w.w_up, nullptr, 0, m->act.p, cf.ffn, (int)M, cf.ffn, d, EPI_SWIGLU,
                              dt, s, m->gemm_ws.p, m->gemm_ws.bytes); }),
     "FFN gate/up (SwiGLU)");
  gemm_work(M, d, cf.ffn, EPI_ADD, m->esize, fl, by);
  const void* res = r.in_loop ? m->mix.p : m->u.p;
  void* dst = r.in_loop ? m->F.p : h_out;
  CK(prof(m, s, P_GEMM, 1, fl, by,
          [&] { return linear(m->act.p, cf.ffn, w.w_down, nullptr, res, d, dst, d, (int)M, d, cf.ffn, EPI_ADD, dt, s, m->gemm_ws.p, m->gemm_ws.bytes); }),
     "FFN down (+ residual)");
  return LOOP_OK;
}

static const float* wr_t(loop_model* m, int layer);

// All executions over M = B*T new tokens whose hidden states are in m->h.
static loop_status run_stack(loop_model* m, loop_cache* c, int B, int T, cudaStream_t s) {
  const loop_config& cf = m->cfg;
  const long M = (long)B * T;
  const int pos0 = c->len;
  const int dt = cf.dtype;
  // rotary cos/sin for these positions, shared by every full-attention execution
  if (m->n_fa > 0 && cf.rotary_dims > 0)
    CK(prof(m, s, P_FA_PREP, 1, 0, 8.0 * T * (cf.rotary_dims / 2),
            [&] { return rope_table((float2*)m->rope.p, T, pos0, cf.rotary_dims, cf.rope_base, s); }),
       "rotary table");
  // the hidden state after execution e, if e is tapped: a copy of h outside the loop block,
  // the mean of the two streams after e's mix inside it
  auto tap_of = [&](int e) -> void* {
    for (size_t k = 0; k < m->tap_exec.size(); ++k)
      if (m->tap_exec[k] == e) return m->tap_out[k];
    return nullptr;
  };
  auto copy_tap = [&](void* dst) -> cudaError_t {
    return prof(m, s, P_COPY, 1, 0, 2.0 * M * cf.d * m->esize, [&] {
      return cudaMemcpyAsync(dst, m->h.p, M * cf.d * m->esize, cudaMemcpyDeviceToDevice, s);
    });
  };
  for (size_t i = 0; i < m->sched.size(); ++i) {
    const ExecRow& r = m->sched[i];
    void* tap = tap_of(r.exec);
    if (!r.in_loop) {
      loop_status st = run_layer(m, c, r, m->h.p, m->h.p, B, T, pos0, s);
      if (st != LOOP_OK) return st;
      if (tap) CK(copy_tap(tap), "hidden-state tap copy");
      continue;
    }
    const loop_layer_weights& w = m->layers[r.layer];
    const double es = (double)m->esize, tok = (double)M;
    if (r.exec == m->first_loop)
      CK(prof(m, s, P_MHC, 1, 0, tok * (es * 4.0 * cf.d + 32.0),
              [&] { return mhc(MHC_OPEN, m->h.p, nullptr, nullptr, w.mhc_w_r, w.mhc_b_r, m->X.p, m->x_in.p, nullptr,
                               (float*)m->coeffs.p, (int)M, cf.d, cf.eps, cf.sinkhorn_iters, dt, s,
                               wr_t(m, r.layer)); }),
         "mHC open");
    loop_status st = run_layer(m, c, r, m->x_in.p, nullptr, B, T, pos0, s);
    if (st != LOOP_OK) return st;
    if (r.exec == m->last_loop) {
      CK(prof(m, s, P_MHC, 1, 0, tok * (es * 4.0 * cf.d + 32.0),
              [&] { return mhc(MHC_MERGE, m->X.p, m->F.p, (float*)m->coeffs.p, nullptr, nullptr, nullptr, nullptr,
                               m->h.p, nullptr, (int)M, cf.d, cf.eps, cf.sinkhorn_iters, dt, s); }),
         "mHC merge");
      if (tap) CK(copy_tap(tap), "hidden-state tap copy");
    } else {
      if (tap)
        CK(prof(m, s, P_MHC, 1, 0, tok * (es * 4.0 * cf.d + 32.0),
                [&] { return mhc(MHC_MERGE, m->X.p, m->F.p, (float*)m->coeffs.p, nullptr, nullptr, nullptr, nullptr,
                                 tap, nullptr, (int)M, cf.d, cf.eps, cf.sinkhorn_iters, dt, s); }),
           "hidden-state tap (stream mean)");
      const loop_layer_weights& wn = m->layers[m->sched[i + 1].layer];
      // read X (2d) + F (d), write X' (2d) + x_in (d), coefficients in/out
      CK(prof(m, s, P_MHC, 1, 0, tok * (es * 6.0 * cf.d + 64.0),
              [&] { return mhc(MHC_MIX, m->X.p, m->F.p, (float*)m->coeffs.p, wn.mhc_w_r, wn.mhc_b_r, m->X.p, m->x_in.p,
                               nullptr, (float*)m->coeffs.p, (int)M, cf.d, cf.eps, cf.sinkhorn_iters, dt, s,
                               wr_t(m, m->sched[i + 1].layer)); }),
         "mHC mix + route");
    }
  }
  return LOOP_OK;
}

// One-time preparation on the first forward (on the caller's stream): transposed copies
// of the looped layers' routing maps.
static loop_status prepare(loop_model* m, cudaStream_t s) {
  if (m->wrt_ready) return LOOP_OK;
  const loop_config& c = m->cfg;
  const size_t per = (size_t)2 * c.d * 8;
  CK(m->wrt.ensure(std::max<size_t>(256, (size_t)c.n_layers * per * sizeof(float))), "routing-map copy allocation");
  for (int l = 0; l < c.n_layers; ++l)
    if (m->layers[l].mhc_w_r)
      CK(transpose_wr(m->layers[l].mhc_w_r, (float*)m->wrt.p + l * per, 2 * c.d, s), "routing-map transpose");
  m->wrt_ready = true;
  return LOOP_OK;
}

static const float* wr_t(loop_model* m, int layer) {
  return (const float*)m->wrt.p + (size_t)layer * 2 * m->cfg.d * 8;
}

loop_status run_forward(loop_model* m, loop_cache* c, const int32_t* ids, const void* h_in, void* h_out,
                        float* logits_last, int B, int T, cudaStream_t s) {
  const loop_config& cf = m->cfg;
  const long M = (long)B * T;
  if (!m->tap_exec.empty() && M > m->tap_rows)
    return fail(LOOP_ERR_CAPACITY, "more new tokens (" + std::to_string(M) + ") than the tap buffers hold (" +
                                       std::to_string(m->tap_rows) + " rows)");
  loop_status st = ensure_workspace(m, M, B, T, c->max_tokens, s);
  if (st != LOOP_OK) return st;
  st = prepare(m, s);
  if (st != LOOP_OK) return st;
  const double es = (double)m->esize;
  if (ids)
    CK(prof(m, s, P_EMBED, 1, 0, (double)M * (2.0 * es * cf.d + 4.0),
            [&] { return embed(ids, m->embed, m->h.p, (int)M, cf.d, cf.vocab, cf.dtype, s); }),
       "embedding");
  else
    CK(cudaMemcpyAsync(m->h.p, h_in, M * cf.d * m->esize, cudaMemcpyDeviceToDevice, s), "hidden-state input copy");
  st = run_stack(m, c, B, T, s);
  if (st != LOOP_OK) return st;
  c->len += T;
  if (h_out) CK(cudaMemcpyAsync(h_out, m->h.p, M * cf.d * m->esize, cudaMemcpyDeviceToDevice, s), "hidden-state output copy");
  if (logits_last) {
    // final norm of each sequence's last position, then the LM head
    const char* last = (const char*)m->h.p + (size_t)(T - 1) * cf.d * m->esize;
    CK(prof(m, s, P_RMSNORM, 1, 0, es * (2.0 * B * cf.d + cf.d),
            [&] { return rmsnorm(last, nullptr, nullptr, m->final_norm, m->last.p, B, cf.d, cf.eps, cf.dtype, s,
                                 (long)T * cf.d); }),
       "final norm");
    double fl, by;
    gemm_work(B, cf.vocab, cf.d, EPI_F32, m->esize, fl, by);
    CK(prof(m, s, P_LMHEAD, 1, fl, by,
            [&] { return linear(m->last.p, cf.d, m->lm_head, nullptr, nullptr, 0, logits_last, cf.vocab, B, cf.vocab,
                                cf.d, EPI_F32, cf.dtype, s, m->gemm_ws.p, m->gemm_ws.bytes); }),
       "LM head");
  }
  return LOOP_OK;
}

loop_status run_decode(loop_model* m, loop_cache* c, const int32_t* tok, float* logits, int32_t* next,
                       cudaStream_t s) {
  const loop_config& cf = m->cfg;
  const int B = c->batch;
  if (!m->tap_exec.empty() && B > m->tap_rows)
    return fail(LOOP_ERR_CAPACITY, "more new tokens (" + std::to_string(B) + ") than the tap buffers hold (" +
                                       std::to_string(m->tap_rows) + " rows)");
  loop_status st = ensure_workspace(m, B, B, 1, c->max_tokens, s);
  if (st != LOOP_OK) return st;
  st = prepare(m, s);
  if (st != LOOP_OK) return st;
  // logits go to the caller's buffer if given, else to a workspace buffer
  float* lg = logits;
  if (!lg) {
    static thread_local DevBuf tmp;
    CK(tmp.ensure((size_t)B * cf.vocab * sizeof(float)), "logits buffer");
    lg = (float*)tmp.p;
  }
  const double es = (double)m->esize;
  CK(prof(m, s, P_EMBED, 1, 0, (double)B * (2.0 * es * cf.d + 4.0),
          [&] { return embed(tok, m->embed, m->h.p, B, cf.d, cf.vocab, cf.dtype, s); }),
     "embedding");
  st = run_stack(m, c, B, 1, s);
  if (st != LOOP_OK) return st;
  c->len += 1;
  CK(prof(m, s, P_RMSNORM, 1, 0, es * (2.0 * B * cf.d + cf.d),
          [&] { return rmsnorm(m->h.p, nullptr, nullptr, m->final_norm, m->last.p, B, cf.d, cf.eps, cf.dtype, s); }),
     "final norm");
  double fl, by;
  gemm_work(B, cf.vocab, cf.d, EPI_F32, m->esize, fl, by);
  CK(prof(m, s, P_LMHEAD, 1, fl, by,
          [&] { return linear(m->last.p, cf.d, m->lm_head, nullptr, nullptr, 0, lg, cf.vocab, B, cf.vocab, cf.d, EPI_F32,
                              cf.dtype, s, m->gemm_ws.p, m->gemm_ws.bytes); }),
     "LM head");
  CK(prof(m, s, P_ARGMAX, 1, 0, 4.0 * B * cf.vocab + 4.0 * B, [&] { return argmax(lg, next, B, cf.vocab, s); }),
     "argmax");
  return LOOP_OK;
}

// ------------------------------------------------------------------ profiling ABI
extern "C" loop_status loop_profile_enable(loop_model* m, int on) {
  if (!m) return fail(LOOP_ERR_INVALID_ARG, "model is NULL");
  m->prof.clear();
  m->prof.on = on != 0;
  return LOOP_OK;
}

extern "C" loop_status loop_profile_read(loop_model* m, loop_profile_entry* out, int cap, int* n) {
  if (!m || !n) return fail(LOOP_ERR_INVALID_ARG, "NULL argument");
  loop_profile_entry acc[P_NCAT];
  memset(acc, 0, sizeof(acc));
  for (int c = 0; c < P_NCAT; ++c) snprintf(acc[c].name, sizeof(acc[c].name), "%s", kProfNames[c]);
  for (auto& r : m->prof.recs) {
    cudaError_t e = cudaEventSynchronize(r.b);
    if (e != cudaSuccess) return cuda_fail(e, "profile event");
    float ms = 0.f;
    cudaEventElapsedTime(&ms, r.a, r.b);
    acc[r.cat].launches += r.launches;
    acc[r.cat].ms += ms;
    acc[r.cat].flops += r.flops;
    acc[r.cat].bytes += r.bytes;
  }
  int k = 0;
  for (int c = 0; c < P_NCAT; ++c)
    if (acc[c].launches) {
      if (out && k < cap) out[k] = acc[c];
      ++k;
    }
  *n = k;
  return LOOP_OK;
}
