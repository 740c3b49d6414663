// Model runtime: schedule, per-execution cache manager, activation workspace,
// and the forward orchestration (prefill / hidden-state forward / decode step).
#pragma once
#include <string>
#include <vector>

#include "../../include/loop.h"
#include "internal.h"

struct ExecRow {
  int exec, layer, kind, slot, in_loop;   // kind: 0 GDN, 1 full attention
};

// Execution table of a config: head layers once, the loop block `loop_passes`
// times with shared weights, tail layers once; slots count executions per kind.
std::vector<ExecRow> build_schedule(const loop_config& c);

struct DevBuf {
  void* p = nullptr;
  size_t bytes = 0;
  ~DevBuf();
  cudaError_t ensure(size_t want);   // grow-only
};

// Per-launch event pairs with the launch's algorithmic work (enabled by loop_profile_enable).
struct ProfRec {
  int cat, launches;
  cudaEvent_t a, b;
  double flops, bytes;
};
struct Profiler {
  bool on = false;
  std::vector<ProfRec> recs;
  std::vector<cudaEvent_t> pool;   // events ready for reuse
  ~Profiler();
  cudaEvent_t get();
  void clear();
};
enum ProfCat { P_GEMM, P_LMHEAD, P_RMSNORM, P_EMBED, P_GDN_PREP, P_GDN_CHUNK, P_GDN_STEP, P_FA_PREP, P_ATTN, P_MHC,
               P_ARGMAX, P_COPY, P_GDN_NORM, P_NCAT };
extern const char* const kProfNames[P_NCAT];

struct loop_model {
  loop_config cfg;
  std::vector<loop_layer_weights> layers;
  const void* embed = nullptr;
  const void* final_norm = nullptr;
  const void* lm_head = nullptr;
  std::vector<ExecRow> sched;
  int n_fa = 0, n_gdn = 0;
  int first_loop = -1, last_loop = -1;
  size_t esize = 2;
  // activation workspace, sized for `ws_tokens` tokens
  long ws_tokens = 0;
  DevBuf h, X, x_in, xn, proj, gq, gk, gv, gg, gb, o, mix, u, un, act, F, coeffs, attn_ws, gdn_ws, gemm_ws, rope, last;
  int in_gdn = 0, in_fa = 0;
  int gdn_hv = 0, gdn_ch = 0;    // GDN value heads; conv channels of the variant (q | k | v)
  Profiler prof;
  DevBuf wrt;                    // [n_layers][8][2d] transposed routing maps (looped layers)
  bool wrt_ready = false;
  // hidden-state taps (loop_set_taps): after execution tap_exec[i], the new tokens' hidden
  // state goes to tap_out[i] [rows, d]; calls with more than tap_rows new tokens are refused
  std::vector<int> tap_exec;
  std::vector<void*> tap_out;
  long tap_rows = 0;
};

struct loop_cache {
  const loop_model* model = nullptr;
  int batch = 0, max_tokens = 0, len = 0;
  DevBuf kv, state, conv;
  size_t kv_slab_elems = 0;      // elements of one K (or V) slab
  size_t state_elems = 0;        // floats of one GDN state (all sequences)
  size_t conv_elems = 0;         // elements of one execution's conv inputs (GDN variant; all sequences)
};

// Set the thread's error message; returns `st`.
loop_status fail(loop_status st, const std::string& msg);
loop_status cuda_fail(cudaError_t e, const char* what);

// Argument checks shared by gqa_attn and gqa_attn_noalloc (same arguments, same rules).
// Returns LOOP_OK when the call should proceed; *empty is set when it is a no-op.
loop_status gqa_check_args(const char* who, const void* q, int ld_q, const void* k, const void* v, int kv_cap,
                           const void* gate, int ld_gate, const void* out, int B, int Tq, int Tkv, int q_off, int Hq,
                           int Hkv, int dh, int causal, int dtype, bool* empty);

loop_status run_forward(loop_model* m, loop_cache* c, const int32_t* ids, const void* h_in, void* h_out,
                        float* logits_last, int B, int T, cudaStream_t s);
loop_status run_decode(loop_model* m, loop_cache* c, const int32_t* tok, float* logits, int32_t* next,
                       cudaStream_t s);
