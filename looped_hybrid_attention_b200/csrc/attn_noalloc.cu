// gqa_attn_noalloc: grouped-query attention that allocates no device memory.
//
// gqa_attn takes its split-K scratch (per-split partial maxima, sums and outputs) from
// the caller.  Some callers cannot provide it: a host runtime that has already handed
// all free device memory to its own pool (so a cudaMalloc would fail or fragment it),
// or a latency-critical loop that must not pay the implicit device synchronisation a
// cudaMalloc / cudaFree can bring.  This variant keeps the scratch in a fixed array in
// the library's device memory instead: 32 MiB, present on every GPU that loads the
// library until the process exits.
#include <mutex>
#include <string>

#include "common.cuh"
#include "internal.h"
#include "runtime.h"

namespace {

constexpr size_t kScratchBytes = 32ull << 20;

// Split-K partials of gqa_attn_noalloc (one array per device).
static __device__ __align__(256) unsigned char g_attn_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device, looked up on the first
// call made with that device current.  (In host code the array's name is only a
// host-side stand-in; the kernels need the device address.)
loop_status scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "gqa_attn_noalloc: cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(LOOP_ERR_UNSUPPORTED, "gqa_attn_noalloc: device ordinal >= 64");
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_attn_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "gqa_attn_noalloc: cudaGetSymbolAddress");
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return LOOP_OK;
}

}  // namespace

extern "C" loop_status gqa_attn_noalloc(const void* q, int ld_q, const void* k, const void* v, int kv_cap,
                                        const void* gate, int ld_gate, void* out, int B, int Tq, int Tkv, int q_off,
                                        int Hq, int Hkv, int dh, int causal, int dtype, void* stream) {
  bool empty = false;
  loop_status st = gqa_check_args("gqa_attn_noalloc", q, ld_q, k, v, kv_cap, gate, ld_gate, out, B, Tq, Tkv, q_off,
                                  Hq, Hkv, dh, causal, dtype, &empty);
  if (st != LOOP_OK || empty) return st;
  // The scratch this call's kernels use: the split-K partials of the kernel that its shape
  // selects, at that kernel's split count (0 for kernels without partials).
  const size_t need = lk::gqa_scratch_bytes(B, Tq, Tkv, Hq, Hkv, dh, dtype);
  if (need > kScratchBytes)
    return fail(LOOP_ERR_CAPACITY, "gqa_attn_noalloc: this problem needs " + std::to_string(need) +
                                       " bytes of scratch but the built-in scratch holds " +
                                       std::to_string(kScratchBytes) + " (32 MiB); use gqa_attn with a workspace");
  void* scratch = nullptr;
  st = scratch_address(&scratch);
  if (st != LOOP_OK) return st;
  // Every (row, head, split) slot of the scratch is written before it is read, so the
  // previous call's contents never leak into this one and nothing needs clearing.
  cudaError_t e = lk::gqa_attn(q, ld_q, k, v, kv_cap, gate, ld_gate, out, B, Tq, Tkv, q_off, Hq, Hkv, dh, causal,
                               scratch, dtype, (cudaStream_t)stream);
  if (e == cudaErrorNotSupported) return fail(LOOP_ERR_UNSUPPORTED, "gqa_attn_noalloc: shape not supported");
  if (e != cudaSuccess) return cuda_fail(e, "gqa_attn_noalloc");
  return LOOP_OK;
}
