"""Pins of the oracle's GDN variant (short causal conv + gated output norm, value heads >= key heads).

The pages name the backbone only ("原地套圈" investigation §01: qwen3_5_text); the variant's
steps are this build's reading of that backbone's Gated-DeltaNet layer.  Each step is pinned
here against a library routine, a by-hand restatement or an invariant.
"""
import math

import numpy as np
import pytest
import scipy.signal

import synth
from oracle import model as omodel
from oracle import ops

EPS = 1e-6
RNG = np.random.default_rng(4321)


def sig(z):
    return 1.0 / (1.0 + math.exp(-z))


def test_causal_conv_matches_fir_filter_and_carries_state():
    T, C, K = 11, 5, 4
    x, w = RNG.normal(size=(T, C)), RNG.normal(size=(C, K))
    y, st = ops.causal_conv_silu(x, w, None)
    for c in range(C):
        pre = scipy.signal.lfilter(w[c, ::-1], [1.0], x[:, c])     # FIR: sum_j b[j] x[t - j]
        assert np.allclose(y[:, c], pre / (1 + np.exp(-pre)), rtol=1e-12, atol=1e-14)
    assert np.array_equal(st, x[-(K - 1):])
    # two segments with the state carried equal one pass
    y1, s1 = ops.causal_conv_silu(x[:4], w, None)
    y2, s2 = ops.causal_conv_silu(x[4:], w, s1)
    assert np.allclose(np.concatenate([y1, y2]), y, atol=1e-14) and np.array_equal(s2, st)
    # a segment shorter than the kernel keeps the older inputs in the state
    y3, s3 = ops.causal_conv_silu(x[4:5], w, s1)
    assert np.array_equal(s3, np.concatenate([x[2:4], x[4:5]]))
    assert np.allclose(y3, y[4:5], atol=1e-14)


def test_causal_conv_by_hand():
    x, w = RNG.normal(size=(3, 2)), RNG.normal(size=(2, 4))
    st = RNG.normal(size=(3, 2))
    y, _ = ops.causal_conv_silu(x, w, st)
    ext = np.concatenate([st, x])
    for t in range(3):
        for c in range(2):
            pre = sum(w[c, j] * ext[t + j, c] for j in range(4))    # w[:, 3] weighs the current token
            assert abs(y[t, c] - pre * sig(pre)) < 1e-14


def test_gated_rmsnorm_by_hand():
    o, z, w = RNG.normal(size=(2, 3, 4)), RNG.normal(size=(2, 3, 4)), 1 + 0.2 * RNG.normal(size=4)
    y = ops.gated_rmsnorm(o, z, w, EPS)
    for t in range(2):
        for h in range(3):
            r = math.sqrt(sum(v * v for v in o[t, h]) / 4 + EPS)
            for i in range(4):
                assert abs(y[t, h, i] - o[t, h, i] / r * w[i] * z[t, h, i] * sig(z[t, h, i])) < 1e-14


def _mixer_v2_by_hand(x, w_in, conv_w, a_bias, b_bias, o_norm, w_out, S0, conv0, Hk, Hv, dk, dv):
    """Token by token: projection, conv + SiLU (state carried), L2 norm, gates, delta rule on value
    head h with key head h // (Hv/Hk), gated output norm, output map."""
    K = conv_w.shape[1]
    C = 2 * Hk * dk + Hv * dv
    hist = [list(r) for r in conv0]                               # K-1 previous conv inputs
    S = S0.copy()
    outs = []
    for t in range(len(x)):
        p = w_in @ x[t]
        ch = list(p[:C])
        z = p[C:C + Hv * dv].reshape(Hv, dv)
        a, b = p[C + Hv * dv:C + Hv * dv + Hv], p[C + Hv * dv + Hv:]
        win = hist + [ch]
        y = [0.0] * C
        for c in range(C):
            pre = sum(conv_w[c, j] * win[j][c] for j in range(K))
            y[c] = pre * sig(pre)
        hist = win[1:]
        q = np.array(y[:Hk * dk]).reshape(Hk, dk)
        k = np.array(y[Hk * dk:2 * Hk * dk]).reshape(Hk, dk)
        v = np.array(y[2 * Hk * dk:]).reshape(Hv, dv)
        q = q / np.sqrt((q * q).sum(-1, keepdims=True) + EPS)
        k = k / np.sqrt((k * k).sum(-1, keepdims=True) + EPS)
        o = np.zeros((Hv, dv))
        for h in range(Hv):
            g = h // (Hv // Hk)
            alpha = 1.0 / (1.0 + math.exp(a[h] + a_bias[h]))
            beta = sig(b[h] + b_bias[h])
            S[h] *= alpha
            S[h] += beta * np.outer(v[h] - S[h] @ k[g], k[g])
            oh = S[h] @ q[g] / math.sqrt(dk)
            r = math.sqrt((oh * oh).mean() + EPS)
            o[h] = oh / r * o_norm * z[h] / (1 + np.exp(-z[h]))
        outs.append(w_out @ o.reshape(-1))
    return np.array(outs), S, np.array(hist)


@pytest.mark.parametrize("T,Hk,Hv", [(1, 1, 2), (3, 1, 2), (2, 2, 2), (5, 2, 4)])
def test_gdn_mixer_v2_by_hand(T, Hk, Hv):
    r = np.random.default_rng(10 * T + Hv)
    d, dk, dv, K = 6, 3, 2, 4
    C = 2 * Hk * dk + Hv * dv
    x = r.normal(size=(T, d))
    w_in = r.normal(size=(C + Hv * dv + 2 * Hv, d)) * 0.7
    conv_w = r.normal(size=(C, K))
    a_bias, b_bias = r.normal(size=Hv), r.normal(size=Hv)
    o_norm = 1 + 0.3 * r.normal(size=dv)
    w_out = r.normal(size=(d, Hv * dv))
    S0 = r.normal(size=(Hv, dv, dk))
    conv0 = r.normal(size=(K - 1, C))
    got, S, conv = ops.gdn_mixer_v2(x, w_in, conv_w, a_bias, b_bias, o_norm, w_out, S0, conv0, Hk, Hv, dk, dv, EPS)
    ref, S_ref, conv_ref = _mixer_v2_by_hand(x, w_in, conv_w, a_bias, b_bias, o_norm, w_out, S0, conv0, Hk, Hv, dk, dv)
    assert np.allclose(got, ref, rtol=1e-11, atol=1e-12)
    assert np.allclose(S, S_ref, rtol=1e-11, atol=1e-12)
    assert np.allclose(conv, conv_ref, atol=0)


VARIANT_TINY = synth.TINY.with_(gdn_variant=1, gdn_v_heads=8, with_embedding=True, vocab=300)


def test_variant_stack_segmented_prefill_and_decode():
    """The conv inputs and states carried in the cache: two prefill segments (the second shorter
    than the conv kernel) equal one, and a decode step equals the next prefill position."""
    s = VARIANT_TINY
    W = omodel.Weights(synth.make_weights(s, seed=3, std=0.05))
    ids = synth.uniform_ids((1, 14), s.vocab, 3).numpy()
    full, _ = omodel.prefill(s, W, ids)
    l1, c = omodel.prefill(s, W, ids[:, :12])
    l2, c = omodel.prefill(s, W, ids[:, 12:14], c)
    assert np.allclose(l2, full, rtol=1e-10, atol=1e-12)
    lg, _ = omodel.prefill(s, W, ids[:, :13])
    _, c = omodel.prefill(s, W, ids[:, :12])
    lg_dec, _ = omodel.decode_step(s, W, c, ids[:, 12])
    assert np.allclose(lg_dec, lg, rtol=1e-10, atol=1e-12)


def test_variant_weight_shapes():
    s = VARIANT_TINY
    names = dict((n, shp) for n, shp, _ in synth.weight_names(s))
    Hk, Hv, dk, dv = s.gdn_heads, s.gdn_v_heads, s.gdn_dk, s.gdn_dv
    assert names["layers.0.gdn_w_in"] == (2 * Hk * dk + 2 * Hv * dv + 2 * Hv, s.d)
    assert names["layers.0.gdn_conv_w"] == (2 * Hk * dk + Hv * dv, 4)
    assert names["layers.0.gdn_w_out"] == (s.d, Hv * dv)
    assert names["layers.0.gdn_o_norm"] == (dv,)
    assert "layers.3.gdn_conv_w" not in names          # layer 3 is the group's full-attention layer
