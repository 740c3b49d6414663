"""Whole-model forward of the looped hybrid decoder (oracle, test infrastructure only).

[teardown] §二 / [wiki] §二: executions run in schedule order; the loop block is
B(B(h)) with the same weights in both passes.  [teardown] §六: entering the loop
block copies h into two residual streams and leaving it averages them; the
head and tail layers are plain pre-norm residual layers.  [teardown] §四: every
execution keeps its own cache (KV for full attention, state for GDN).

One decoder layer (pre-norm; READING: one mHC per decoder layer, the layer's
residual branch F = mixer + FFN output):
    mix = Mixer(RMSNorm(x));  u = x + mix;  f = FFN(RMSNorm(u));  F = mix + f
    plain layer:  h <- h + F
    looped layer: x = sum_s H_pre[s] X_s;  X_s <- sum_t H_res[s,t] X_t + H_post[s] F
"""
from __future__ import annotations

import numpy as np

from . import ops, schedule


class Weights:
    """Name -> float64 array, widened lazily from the synthetic weight tensors."""

    def __init__(self, tensors):
        self._t = tensors
        self._c = {}

    def __getitem__(self, name):
        if name not in self._c:
            self._c[name] = ops.f64(self._t[name])
        return self._c[name]

    def layer(self, l):
        p = f"layers.{l}."
        return lambda key: self[p + key]


def new_cache():
    return {"kv": {}, "state": {}, "len": 0}


def layer_branch(shape, W, l, kind, slot, x, cache, pos0):
    """F = mix + f for stored layer l on tokens x [T, d] at positions pos0..pos0+T-1; updates the cache slot."""
    s = shape
    lw = W.layer(l)
    a = ops.rmsnorm(x, lw("attn_norm"), s.eps)
    if kind == "gdn" and getattr(s, "gdn_variant", 0) == 1:
        Hk, Hv, dk, dv = s.gdn_heads, s.gdn_v_heads or s.gdn_heads, s.gdn_dk, s.gdn_dv
        S0 = cache["state"].get(slot)
        if S0 is None:
            S0 = np.zeros((Hv, dv, dk))                # READING: zero state and conv inputs at sequence start
        conv0 = cache.setdefault("conv", {}).get(slot)
        mix, S, conv = ops.gdn_mixer_v2(a, lw("gdn_w_in"), lw("gdn_conv_w"), lw("gdn_a_bias"), lw("gdn_b_bias"),
                                        lw("gdn_o_norm"), lw("gdn_w_out"), S0, conv0, Hk, Hv, dk, dv, s.eps)
        cache["state"][slot] = S
        cache["conv"][slot] = conv
    elif kind == "gdn":
        H, dk, dv = s.gdn_heads, s.gdn_dk, s.gdn_dv
        S0 = cache["state"].get(slot)
        if S0 is None:
            S0 = np.zeros((H, dv, dk))                 # READING: zero state at sequence start
        mix, S = ops.gdn_mixer(a, lw("gdn_w_in"), lw("gdn_a_bias"), lw("gdn_b_bias"), lw("gdn_w_out"),
                               S0, H, dk, dv, s.eps)
        cache["state"][slot] = S
    else:
        Kc, Vc = cache["kv"].get(slot, (None, None))
        mix, K, V = ops.fa_mixer(a, lw("fa_w_in"), lw("fa_q_norm"), lw("fa_k_norm"), lw("fa_w_out"),
                                 Kc, Vc, pos0, s.fa_q_heads, s.fa_kv_heads, s.fa_head_dim,
                                 s.rotary_dims, s.rope_base, s.eps)
        cache["kv"][slot] = (K, V)
    u = x + mix
    f = ops.swiglu_ffn(ops.rmsnorm(u, lw("ffn_norm"), s.eps), lw("ffn_w_gate"), lw("ffn_w_up"),
                       lw("ffn_w_down"))
    return mix + f


def run_stack(shape, W, h, cache, taps=None):
    """Run every execution on new tokens h [T, d] of one sequence; returns the hidden state after the last one.

    cache holds this sequence's per-execution state; positions continue from
    cache['len'].  If `taps` is a list, the hidden state after each execution
    is appended (inside the loop block: the mean of the two streams).
    """
    s = shape
    rows = schedule.table(s)
    loop_rows = [r[0] for r in rows if r[4]]
    first, last = (loop_rows[0], loop_rows[-1]) if loop_rows else (-1, -1)
    pos0 = cache["len"]
    h = ops.f64(h)
    X = None
    for e, l, kind, slot, in_loop in rows:
        if in_loop:
            if e == first:
                X = ops.mhc_open(h, s.mhc_streams)
            lw = W.layer(l)
            H_pre, H_post, H_res = ops.mhc_coeffs(X, lw("mhc_w_r"), lw("mhc_b_r"), s.eps, s.sinkhorn_iters)
            x = ops.mhc_read(X, H_pre)
            F = layer_branch(s, W, l, kind, slot, x, cache, pos0)
            X = ops.mhc_write(X, F, H_post, H_res)
            if e == last:
                h = ops.mhc_merge(X)
            if taps is not None:
                taps.append(ops.mhc_merge(X))
        else:
            h = h + layer_branch(s, W, l, kind, slot, h, cache, pos0)
            if taps is not None:
                taps.append(h.copy())
    cache["len"] = pos0 + h.shape[0]
    return h


def forward_hidden(shape, W, h, caches=None, taps=None):
    """Hidden states in, hidden states out (before any final norm): h [B, T, d] -> [B, T, d]."""
    h = ops.f64(h)
    B = h.shape[0]
    if caches is None:
        caches = [new_cache() for _ in range(B)]
    out = np.stack([run_stack(shape, W, h[b], caches[b], taps if b == 0 else None) for b in range(B)])
    return out, caches


def prefill(shape, W, ids, caches=None):
    """Token ids [B, T] -> logits of the last position [B, V], with the filled per-execution caches.

    READING: prefill returns last-position logits only (what decoding needs).
    """
    ids = np.asarray(ids)
    B = ids.shape[0]
    if caches is None:
        caches = [new_cache() for _ in range(B)]
    E = W["embed"]
    logits = []
    for b in range(B):
        h = run_stack(shape, W, E[ids[b]], caches[b])
        logits.append(ops.lm_logits(h[-1:], W["final_norm"], W["lm_head"], shape.eps)[0])
    return np.stack(logits), caches


def decode_step(shape, W, caches, tok):
    """One greedy decode step: tok [B] -> (logits [B, V], next token [B])."""
    tok = np.asarray(tok)
    E = W["embed"]
    logits = []
    for b in range(tok.shape[0]):
        h = run_stack(shape, W, E[tok[b:b + 1]], caches[b])
        logits.append(ops.lm_logits(h, W["final_norm"], W["lm_head"], shape.eps)[0])
    logits = np.stack(logits)
    return logits, ops.greedy(logits)
