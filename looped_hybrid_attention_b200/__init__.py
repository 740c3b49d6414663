"""Python binding of libloop_b200.so (the C ABI in include/loop.h).

Argument marshalling only: every computation runs in the library's CUDA kernels.
torch tensors provide device memory and streams; their data pointers are passed
straight through.  There is no CPU path: if the shared library is missing this
module raises at import.
"""
from __future__ import annotations

import ctypes
import os
import re

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libloop_b200.so")
HEADER = os.path.join(HERE, "..", "include", "loop.h")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is not built; run `python looped_hybrid_attention_b200/build.py`")

_lib = ctypes.CDLL(LIB_PATH)

F32, BF16 = 0, 1
EPI_STORE, EPI_ADD, EPI_SWIGLU, EPI_F32 = 0, 1, 2, 3
MHC_OPEN, MHC_MIX, MHC_ROUTE, MHC_MERGE = 0, 1, 2, 3
STATUS = {0: "LOOP_OK", 1: "LOOP_ERR_INVALID_ARG", 2: "LOOP_ERR_SHAPE", 3: "LOOP_ERR_OOM", 4: "LOOP_ERR_CUDA",
          5: "LOOP_ERR_CAPACITY", 6: "LOOP_ERR_TIMEOUT", 7: "LOOP_ERR_UNSUPPORTED"}


class LoopError(RuntimeError):
    def __init__(self, status, msg):
        super().__init__(f"{STATUS.get(status, status)}: {msg}")
        self.status = status


class loop_config(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in (
        "d", "ffn", "vocab", "n_layers", "loop_start", "loop_end", "loop_passes", "group",
        "gdn_heads", "gdn_dk", "gdn_dv", "fa_q_heads", "fa_kv_heads", "fa_head_dim", "rotary_dims",
        "mhc_streams", "sinkhorn_iters", "gdn_chunk")] + [
        ("eps", ctypes.c_float), ("rope_base", ctypes.c_float), ("dtype", ctypes.c_int),
        ("with_embedding", ctypes.c_int), ("gdn_variant", ctypes.c_int), ("gdn_v_heads", ctypes.c_int),
        ("gdn_conv", ctypes.c_int)]


class loop_layer_weights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "attn_norm", "w_in", "gdn_a_bias", "gdn_b_bias", "q_norm", "k_norm", "w_out", "ffn_norm",
        "w_gate", "w_up", "w_down", "mhc_w_r", "mhc_b_r", "gdn_conv_w", "gdn_o_norm")]


class loop_profile_entry(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 24), ("launches", ctypes.c_int), ("ms", ctypes.c_double),
                ("flops", ctypes.c_double), ("bytes", ctypes.c_double)]


class loop_weights(ctypes.Structure):
    _fields_ = [("embed", ctypes.c_void_p), ("final_norm", ctypes.c_void_p), ("lm_head", ctypes.c_void_p),
                ("layers", ctypes.POINTER(loop_layer_weights)), ("n_layers", ctypes.c_int)]


_P, _I, _F, _Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
_SIGS = {
    "loop_last_error": ([], ctypes.c_char_p),
    "loop_version": ([], ctypes.c_char_p),
    "loop_device_error": ([ctypes.POINTER(ctypes.c_int)], _I),
    "loop_wait_selftest": ([ctypes.c_longlong, _P], _I),
    "loop_schedule": ([ctypes.POINTER(loop_config), _P, _I, _P, _P, _P], _I),
    "loop_model_create": ([ctypes.POINTER(loop_config), ctypes.POINTER(loop_weights), ctypes.POINTER(_P)], _I),
    "loop_model_destroy": ([_P], _I),
    "loop_cache_create": ([_P, _I, _I, ctypes.POINTER(_P)], _I),
    "loop_cache_reset": ([_P], _I),
    "loop_cache_destroy": ([_P], _I),
    "loop_cache_length": ([_P, ctypes.POINTER(ctypes.c_int)], _I),
    "loop_cache_set_length": ([_P, _I], _I),
    "loop_cache_bytes": ([_P, ctypes.POINTER(_Z), ctypes.POINTER(_Z)], _I),
    "loop_cache_kv": ([_P, _I, ctypes.POINTER(_P), ctypes.POINTER(_P)], _I),
    "loop_cache_state": ([_P, _I, ctypes.POINTER(_P)], _I),
    "loop_prefill": ([_P, _P, _P, _I, _I, _P, _P], _I),
    "loop_forward_hidden": ([_P, _P, _P, _P, _I, _I, _P], _I),
    "loop_decode_step": ([_P, _P, _P, _P, _P, _P], _I),
    "loop_set_taps": ([_P, _I, _P, _P, ctypes.c_long], _I),
    "gdn_chunk_fwd": ([_P] * 7 + [_I] * 6 + [_F, _P, _I, _P], _I),
    "loop_gdn_workspace_bytes": ([_I] * 5, _Z),
    "gdn_step": ([_P] * 7 + [_I] * 4 + [_F, _I, _P], _I),
    "gdn_in_proj": ([_P, _I, _P, _P, _P, _P, _P, _P, _P, _P] + [_I] * 5 + [_F, _I, _P], _I),
    "gdn_conv_prep": ([_P, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P] + [_I] * 7 + [_F, _I, _P], _I),
    "gdn_gated_norm": ([_P, _P, _I, _P, _P, _I, _I, _I, _F, _I, _P], _I),
    "gdn_prep": ([_P, _I] + [_P] * 7 + [_I] * 4 + [_F, _I, _P], _I),
    "gqa_attn": ([_P, _I, _P, _P, _I, _P, _I, _P] + [_I] * 8 + [_P, _I, _P], _I),
    "loop_gqa_workspace_bytes": ([_I] * 5, _Z),
    "gqa_attn_noalloc": ([_P, _I, _P, _P, _I, _P, _I, _P] + [_I] * 8 + [_I, _P], _I),
    "gqa_attn_fused_q": ([_P, _I, _P, _I, _F, _F, _P, _P, _I, _P, _I, _P] + [_I] * 9 + [_P], _I),
    "fa_prep": ([_P, _I, _P, _P, _P, _P, _P, _I] + [_I] * 7 + [_F, _F, _I, _P], _I),
    "mhc_route_mix": ([_I] + [_P] * 9 + [_I, _I, _F, _I, _I, _P], _I),
    "sinkhorn_fp32": ([_P, _P, _I, _I, _I, _P], _I),
    "loop_linear": ([_P, _I, _P, _P, _P, _I, _P] + [_I] * 5 + [_P, _I, _P], _I),
    "loop_linear_workspace_bytes": ([_I] * 4, _Z),
    "loop_rmsnorm": ([_P] * 5 + [_I, _I, _F, _I, _P], _I),
    "loop_embed": ([_P, _P, _P, _I, _I, _I, _I, _P], _I),
    "loop_argmax": ([_P, _P, _I, _I, _P], _I),
    "loop_profile_enable": ([_P, _I], _I),
    "loop_profile_read": ([_P, _P, _I, ctypes.POINTER(ctypes.c_int)], _I),
}
for _name, (_args, _res) in _SIGS.items():
    _fn = getattr(_lib, _name)
    _fn.argtypes = _args
    _fn.restype = _res


def header_functions():
    """Names of every function declared in include/loop.h."""
    txt = open(HEADER).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(\w+)\s*\(", txt, flags=re.M)) - {"if", "defined"})


def last_error() -> str:
    return _lib.loop_last_error().decode()


def check(status, what=""):
    if status != 0:
        raise LoopError(status, f"{what}: {last_error()}")


def ptr(t):
    """Device (or host) address of a tensor, or None."""
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        import torch
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else stream)


class _DevArray:
    def __init__(self, addr, shape, typestr):
        self.__cuda_array_interface__ = {"shape": tuple(shape), "typestr": typestr, "data": (int(addr), False),
                                         "version": 3, "strides": None}


def device_view(addr, shape, dtype):
    """A torch tensor aliasing library-owned device memory (cache slabs and states)."""
    import torch
    ts = {torch.float32: "<f4", torch.bfloat16: "<V2", torch.int32: "<i4"}[dtype]
    if dtype == torch.bfloat16:      # no bf16 typestr: view as int16 and reinterpret
        t = torch.as_tensor(_DevArray(addr, shape, "<i2"), device="cuda")
        return t.view(torch.bfloat16)
    return torch.as_tensor(_DevArray(addr, shape, ts), device="cuda")


def dtype_code(t):
    import torch
    return BF16 if t.dtype == torch.bfloat16 else F32


def device_error() -> int:
    c = ctypes.c_int(0)
    _lib.loop_device_error(ctypes.byref(c))
    return c.value


def device_error_status() -> int:
    """loop_device_error's status (LOOP_ERR_TIMEOUT after a bounded wait gave up); clears the code."""
    c = ctypes.c_int(0)
    return _lib.loop_device_error(ctypes.byref(c))


def wait_selftest(cycles, stream=None):
    """One bounded wait that runs out after `cycles` SM clock cycles (the error path's self-test)."""
    check(_lib.loop_wait_selftest(int(cycles), _stream(stream)), "loop_wait_selftest")


def make_config(shape) -> loop_config:
    """loop_config from any object with the ModelShape fields."""
    s = shape
    return loop_config(s.d, s.ffn, s.vocab, s.n_layers, s.loop_start, s.loop_end, s.loop_passes, s.group,
                       s.gdn_heads, s.gdn_dk, s.gdn_dv, s.fa_q_heads, s.fa_kv_heads, s.fa_head_dim,
                       s.rotary_dims, s.mhc_streams, s.sinkhorn_iters, s.gdn_chunk, s.eps, s.rope_base,
                       BF16 if s.dtype == "bf16" else F32, 1 if s.with_embedding else 0,
                       getattr(s, "gdn_variant", 0), getattr(s, "gdn_v_heads", 0), getattr(s, "gdn_conv", 4))


def schedule(shape):
    """Execution table from the library: list of (exec, layer, kind, slot, in_loop)."""
    cfg = make_config(shape)
    n = ctypes.c_int(0)
    check(_lib.loop_schedule(ctypes.byref(cfg), None, 0, ctypes.byref(n), None, None), "loop_schedule")
    buf = (ctypes.c_int32 * (5 * n.value))()
    check(_lib.loop_schedule(ctypes.byref(cfg), buf, n.value, ctypes.byref(n), None, None), "loop_schedule")
    return [tuple(buf[5 * i:5 * i + 5]) for i in range(n.value)]


# ----------------------------------------------------------------------------- model + cache

class Model:
    """loop_model over caller-owned device weights (a name -> tensor dict with the layout of include/loop.h)."""

    def __init__(self, shape, weights):
        self.shape = shape
        self.cfg = make_config(shape)
        self.weights = weights            # keep the tensors alive
        s = shape
        layers = (loop_layer_weights * s.n_layers)()
        for l in range(s.n_layers):
            p = f"layers.{l}."
            g = lambda k: ptr(weights.get(p + k)) if (p + k) in weights else None
            fa = (l % s.group) == s.group - 1
            layers[l] = loop_layer_weights(
                g("attn_norm"), g("fa_w_in" if fa else "gdn_w_in"), g("gdn_a_bias"), g("gdn_b_bias"),
                g("fa_q_norm"), g("fa_k_norm"), g("fa_w_out" if fa else "gdn_w_out"), g("ffn_norm"),
                g("ffn_w_gate"), g("ffn_w_up"), g("ffn_w_down"), g("mhc_w_r"), g("mhc_b_r"),
                g("gdn_conv_w"), g("gdn_o_norm"))
        self._layers = layers
        w = loop_weights(ptr(weights.get("embed")), ptr(weights.get("final_norm")), ptr(weights.get("lm_head")),
                         layers, s.n_layers)
        h = ctypes.c_void_p()
        check(_lib.loop_model_create(ctypes.byref(self.cfg), ctypes.byref(w), ctypes.byref(h)), "loop_model_create")
        self.handle = h

    def close(self):
        if getattr(self, "handle", None):
            _lib.loop_model_destroy(self.handle)
            self.handle = None

    __del__ = close

    def profile(self, on=True):
        """Start (clearing) or stop per-kernel event timing inside the model's launches."""
        check(_lib.loop_profile_enable(self.handle, int(on)), "loop_profile_enable")

    def profile_read(self):
        """{kernel class: {launches, ms, flops, bytes}} summed since profile(True)."""
        buf = (loop_profile_entry * 32)()
        n = ctypes.c_int(0)
        check(_lib.loop_profile_read(self.handle, buf, 32, ctypes.byref(n)), "loop_profile_read")
        return {buf[i].name.decode(): {"launches": buf[i].launches, "ms": buf[i].ms, "flops": buf[i].flops,
                                       "bytes": buf[i].bytes} for i in range(min(n.value, 32))}

    def cache(self, batch, max_tokens):
        return Cache(self, batch, max_tokens)

    def prefill(self, cache, ids, logits_last, stream=None):
        B, T = ids.shape
        check(_lib.loop_prefill(self.handle, cache.handle, ptr(ids), B, T, ptr(logits_last), _stream(stream)),
              "loop_prefill")

    def forward_hidden(self, cache, h_in, h_out, stream=None):
        B, T, _ = h_in.shape
        check(_lib.loop_forward_hidden(self.handle, cache.handle, ptr(h_in), ptr(h_out), B, T, _stream(stream)),
              "loop_forward_hidden")

    def decode_step(self, cache, tok, logits, next_tok, stream=None):
        check(_lib.loop_decode_step(self.handle, cache.handle, ptr(tok), ptr(logits), ptr(next_tok),
                                    _stream(stream)), "loop_decode_step")

    def set_taps(self, execs, outs, max_rows):
        """Hidden-state taps after the given executions into the given [rows, d] device tensors ([] clears)."""
        n = len(execs)
        ex = (ctypes.c_int32 * max(n, 1))(*execs)
        ps = (ctypes.c_void_p * max(n, 1))(*[t.data_ptr() for t in outs])
        check(_lib.loop_set_taps(self.handle, n, ex, ps, max_rows), "loop_set_taps")
        self._taps = list(outs)           # keep the buffers alive while set


class Cache:
    def __init__(self, model, batch, max_tokens):
        h = ctypes.c_void_p()
        check(_lib.loop_cache_create(model.handle, batch, max_tokens, ctypes.byref(h)), "loop_cache_create")
        self.handle, self.model, self.batch, self.max_tokens = h, model, batch, max_tokens

    def close(self):
        if getattr(self, "handle", None):
            _lib.loop_cache_destroy(self.handle)
            self.handle = None

    __del__ = close

    def reset(self):
        check(_lib.loop_cache_reset(self.handle), "loop_cache_reset")

    @property
    def length(self):
        n = ctypes.c_int(0)
        check(_lib.loop_cache_length(self.handle, ctypes.byref(n)), "loop_cache_length")
        return n.value

    @length.setter
    def length(self, n):
        check(_lib.loop_cache_set_length(self.handle, int(n)), "loop_cache_set_length")

    def nbytes(self):
        a, b = ctypes.c_size_t(0), ctypes.c_size_t(0)
        check(_lib.loop_cache_bytes(self.handle, ctypes.byref(a), ctypes.byref(b)), "loop_cache_bytes")
        return a.value, b.value

    def kv_ptrs(self, slot):
        k, v = ctypes.c_void_p(), ctypes.c_void_p()
        check(_lib.loop_cache_kv(self.handle, slot, ctypes.byref(k), ctypes.byref(v)), "loop_cache_kv")
        return k.value, v.value

    def state_ptr(self, slot):
        s = ctypes.c_void_p()
        check(_lib.loop_cache_state(self.handle, slot, ctypes.byref(s)), "loop_cache_state")
        return s.value


# ----------------------------------------------------------------------------- per-op calls

def gdn_workspace_bytes(B, T, H, dk, dv):
    return _lib.loop_gdn_workspace_bytes(B, T, H, dk, dv)


def gdn_chunk_fwd(q, k, v, g, beta, state, out, scale, chunk=64, workspace=None, stream=None):
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    check(_lib.gdn_chunk_fwd(ptr(q), ptr(k), ptr(v), ptr(g), ptr(beta), ptr(state), ptr(out), B, T, H, dk, dv,
                             chunk, scale, ptr(workspace), dtype_code(q), _stream(stream)), "gdn_chunk_fwd")


def gdn_step(q, k, v, g, beta, state, out, scale, stream=None):
    B, H, dk = q.shape
    dv = v.shape[-1]
    check(_lib.gdn_step(ptr(q), ptr(k), ptr(v), ptr(g), ptr(beta), ptr(state), ptr(out), B, H, dk, dv, scale,
                        dtype_code(q), _stream(stream)), "gdn_step")


def gdn_prep(P, a_bias, b_bias, q, k, v, g, beta, H, dk, dv, eps, stream=None):
    M = P.shape[0]
    check(_lib.gdn_prep(ptr(P), P.stride(0), ptr(a_bias), ptr(b_bias), ptr(q), ptr(k), ptr(v), ptr(g), ptr(beta),
                        M, H, dk, dv, eps, dtype_code(P), _stream(stream)), "gdn_prep")


def gdn_in_proj(x, w_in, a_bias, b_bias, q, k, v, g, beta, H, dk, dv, eps, stream=None):
    """GDN input projection with the preparation (L2 norms, gates) in its epilogue."""
    M, d = x.shape
    check(_lib.gdn_in_proj(ptr(x), x.stride(0), ptr(w_in), ptr(a_bias), ptr(b_bias), ptr(q), ptr(k), ptr(v), ptr(g),
                           ptr(beta), M, d, H, dk, dv, eps, dtype_code(x), _stream(stream)), "gdn_in_proj")


def gdn_conv_prep(P, conv_w, conv_state, a_bias, b_bias, q, k, v, g, beta, B, T, Hk, Hv, dk, dv, eps, conv=4,
                  stream=None):
    """GDN variant input preparation: conv + SiLU on q|k|v, L2 norm, gates; conv_state updated in place."""
    check(_lib.gdn_conv_prep(ptr(P), P.stride(0), ptr(conv_w), ptr(conv_state), ptr(a_bias), ptr(b_bias), ptr(q),
                             ptr(k), ptr(v), ptr(g), ptr(beta), B, T, Hk, Hv, dk, dv, conv, eps, dtype_code(P),
                             _stream(stream)), "gdn_conv_prep")


def gdn_gated_norm(o, z, ld_z, w, y, M, H, dv, eps, stream=None):
    check(_lib.gdn_gated_norm(ptr(o), ptr(z), ld_z, ptr(w), ptr(y), M, H, dv, eps, dtype_code(o), _stream(stream)),
          "gdn_gated_norm")


def gqa_workspace_bytes(B, Tq, Tkv, Hq, dh):
    return _lib.loop_gqa_workspace_bytes(B, Tq, Tkv, Hq, dh)


def gqa_attn(q, ld_q, k, v, kv_cap, gate, ld_gate, out, B, Tq, Tkv, q_off, Hq, Hkv, dh, causal=True,
             workspace=None, stream=None):
    check(_lib.gqa_attn(ptr(q), ld_q, ptr(k), ptr(v), kv_cap, ptr(gate), ld_gate, ptr(out), B, Tq, Tkv, q_off,
                        Hq, Hkv, dh, int(causal), ptr(workspace), dtype_code(q), _stream(stream)), "gqa_attn")


def gqa_attn_noalloc(q, ld_q, k, v, kv_cap, gate, ld_gate, out, B, Tq, Tkv, q_off, Hq, Hkv, dh, causal=True,
                     stream=None):
    """gqa_attn with the split-K scratch in the library's fixed device array (allocates nothing)."""
    check(_lib.gqa_attn_noalloc(ptr(q), ld_q, ptr(k), ptr(v), kv_cap, ptr(gate), ld_gate, ptr(out), B, Tq, Tkv,
                                q_off, Hq, Hkv, dh, int(causal), dtype_code(q), _stream(stream)), "gqa_attn_noalloc")


def gqa_attn_fused_q(q, ld_q, q_norm, rotary_dims, rope_base, eps, k, v, kv_cap, gate, ld_gate, out, B, Tq, Tkv,
                     q_off, Hq, Hkv, dh, causal=True, stream=None):
    """gqa_attn on raw query rows: QK-norm and rotary applied by the attention kernel."""
    check(_lib.gqa_attn_fused_q(ptr(q), ld_q, ptr(q_norm), rotary_dims, rope_base, eps, ptr(k), ptr(v), kv_cap,
                                ptr(gate), ld_gate, ptr(out), B, Tq, Tkv, q_off, Hq, Hkv, dh, int(causal),
                                dtype_code(q), _stream(stream)), "gqa_attn_fused_q")


def fa_prep(P, q_norm, k_norm, q_out, k_cache, v_cache, kv_cap, B, T, pos0, Hq, Hkv, dh, rotary_dims, rope_base,
            eps, stream=None):
    check(_lib.fa_prep(ptr(P), P.stride(0), ptr(q_norm), ptr(k_norm), ptr(q_out), ptr(k_cache), ptr(v_cache),
                       kv_cap, B, T, pos0, Hq, Hkv, dh, rotary_dims, rope_base, eps, dtype_code(P),
                       _stream(stream)), "fa_prep")


def mhc_route_mix(mode, X_in, F, coeffs_in, w_r, b_r, X_out, x_in, h_out, coeffs_out, N, d, eps, iters,
                  dtype, stream=None):
    check(_lib.mhc_route_mix(mode, ptr(X_in), ptr(F), ptr(coeffs_in), ptr(w_r), ptr(b_r), ptr(X_out), ptr(x_in),
                             ptr(h_out), ptr(coeffs_out), N, d, eps, iters, dtype, _stream(stream)), "mhc_route_mix")


def sinkhorn_fp32(logits, out, iters, stream=None):
    N, n, _ = logits.shape
    check(_lib.sinkhorn_fp32(ptr(logits), ptr(out), N, n, iters, _stream(stream)), "sinkhorn_fp32")


def linear_workspace_bytes(M, N, K, epilogue):
    return _lib.loop_linear_workspace_bytes(M, N, K, epilogue)


def linear(X, W, Y, epilogue=EPI_STORE, W2=None, R=None, workspace=None, stream=None):
    M, K = X.shape
    N = W.shape[0]
    check(_lib.loop_linear(ptr(X), X.stride(0), ptr(W), ptr(W2), ptr(R), R.stride(0) if R is not None else 0,
                           ptr(Y), Y.stride(0), M, N, K, epilogue, ptr(workspace), dtype_code(X), _stream(stream)),
          "loop_linear")


def rmsnorm(x, w, y, eps, r=None, sum_out=None, stream=None):
    M, d = x.shape
    check(_lib.loop_rmsnorm(ptr(x), ptr(r), ptr(sum_out), ptr(w), ptr(y), M, d, eps, dtype_code(x),
                            _stream(stream)), "loop_rmsnorm")


def embed(ids, E, out, stream=None):
    M = ids.numel()
    V, d = E.shape
    check(_lib.loop_embed(ptr(ids), ptr(E), ptr(out), M, d, V, dtype_code(E), _stream(stream)), "loop_embed")


def argmax(logits, out, stream=None):
    B, V = logits.shape
    check(_lib.loop_argmax(ptr(logits), ptr(out), B, V, _stream(stream)), "loop_argmax")
