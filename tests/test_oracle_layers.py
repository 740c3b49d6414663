"""Pins of the oracle's composite functions, written out by hand for one and two tokens.

Each test restates a layer-level function of the oracle token by token and head by head
with explicit scalar/vector formulas (no oracle helper on the checking side), on tiny
dimensions where every index is visible, so that a dropped term, a swapped operand or a
mis-placed scale in the composition fails:

  - GDN mixer ("Loop-9B engineering teardown" §三: gate + delta rule, constant state):
    projections, L2 norm of q and k (eps inside the root), decay exp(-softplus(a + a_bias)),
    beta = sigmoid(b + b_bias), state update, output scale 1/sqrt(dk) on the read-out only,
    output map;
  - full-attention mixer (same page §三: GQA, QK normalisation, partial interleaved rotary,
    output gate): RMSNorm of q and k with gains, rotation of the first pair(s), softmax over
    cached + causal keys with scale 1/sqrt(dh), sigmoid(gate) before the output map;
  - the layer's residual branch (same page §五: one mHC per decoder layer): u = x + mix,
    f = FFN(RMSNorm(u)), F = mix + f;
  - the LM head: RMSNorm with the final gain, then the untied head;
  - one looped execution of the stack (same page §五, §六): route from the streams, read,
    branch, write.
"""
import math

import numpy as np
import pytest

import synth
from oracle import model as omodel
from oracle import ops

EPS = 1e-6


def sig(z):
    return 1.0 / (1.0 + math.exp(-z))


def rms(vec, gain):
    return [vec[i] / math.sqrt(sum(t * t for t in vec) / len(vec) + EPS) * gain[i] for i in range(len(vec))]


def matvec(W, x):
    """W [out, in] times x [in], as explicit sums."""
    return [sum(W[o][i] * x[i] for i in range(len(x))) for o in range(len(W))]


# ----------------------------------------------------------------------------- GDN mixer

def _gdn_by_hand(x, w_in, a_bias, b_bias, w_out, S0, H, dk, dv):
    """Token-by-token, head-by-head restatement; returns outputs [T][d] and states [H][dv][dk]."""
    S = [[[float(S0[h][i][j]) for j in range(dk)] for i in range(dv)] for h in range(H)]
    outs = []
    for t in range(len(x)):
        p = matvec(w_in, x[t])
        o_cat = []
        for h in range(H):
            q = p[h * dk:(h + 1) * dk]
            k = p[H * dk + h * dk:H * dk + (h + 1) * dk]
            v = p[2 * H * dk + h * dv:2 * H * dk + (h + 1) * dv]
            a = p[2 * H * dk + H * dv + h]
            b = p[2 * H * dk + H * dv + H + h]
            qn = math.sqrt(sum(c * c for c in q) + EPS)
            kn = math.sqrt(sum(c * c for c in k) + EPS)
            q = [c / qn for c in q]
            k = [c / kn for c in k]
            alpha = 1.0 / (1.0 + math.exp(a + a_bias[h]))        # exp(-softplus(z)) = 1 / (1 + e^z)
            beta = sig(b + b_bias[h])
            Sh = S[h]
            for i in range(dv):
                for j in range(dk):
                    Sh[i][j] *= alpha
            pred = [sum(Sh[i][j] * k[j] for j in range(dk)) for i in range(dv)]
            for i in range(dv):
                for j in range(dk):
                    Sh[i][j] += beta * (v[i] - pred[i]) * k[j]
            o_cat += [sum(Sh[i][j] * q[j] for j in range(dk)) / math.sqrt(dk) for i in range(dv)]
        outs.append(matvec(w_out, o_cat))
    return np.array(outs), np.array(S)


@pytest.mark.parametrize("T", [1, 2, 3])
def test_gdn_mixer_by_hand(T):
    r = np.random.default_rng(40 + T)
    d, H, dk, dv = 5, 2, 3, 2
    x = r.normal(size=(T, d))
    w_in = r.normal(size=(2 * H * dk + H * dv + 2 * H, d)) * 0.7
    a_bias, b_bias = r.normal(size=H), r.normal(size=H)
    w_out = r.normal(size=(d, H * dv))
    S0 = r.normal(size=(H, dv, dk))
    got, S = ops.gdn_mixer(x, w_in, a_bias, b_bias, w_out, S0, H, dk, dv, EPS)
    ref, S_ref = _gdn_by_hand(x.tolist(), w_in.tolist(), a_bias.tolist(), b_bias.tolist(), w_out.tolist(),
                              S0, H, dk, dv)
    assert np.allclose(got, ref, rtol=1e-12, atol=1e-12)
    assert np.allclose(S, S_ref, rtol=1e-12, atol=1e-12)


# ----------------------------------------------------------------------------- FA mixer

def _rot(vec, pos, r, base):
    out = list(vec)
    for j in range(r // 2):
        ang = pos * base ** (-2.0 * j / r)
        c, s = math.cos(ang), math.sin(ang)
        x0, x1 = vec[2 * j], vec[2 * j + 1]
        out[2 * j], out[2 * j + 1] = x0 * c - x1 * s, x0 * s + x1 * c
    return out


def _fa_by_hand(x, w_in, qg, kg, w_out, Kc, Vc, pos0, Hq, Hkv, dh, r, base):
    """Returns outputs [T][d] and the full key / value lists per KV head."""
    keys = [[list(Kc[p][g]) for p in range(len(Kc))] for g in range(Hkv)]
    vals = [[list(Vc[p][g]) for p in range(len(Vc))] for g in range(Hkv)]
    qs, gates = [], []
    for t in range(len(x)):
        p = matvec(w_in, x[t])
        pos = pos0 + t
        qs.append([_rot(rms(p[h * dh:(h + 1) * dh], qg), pos, r, base) for h in range(Hq)])
        gates.append([p[Hq * dh + h * dh:Hq * dh + (h + 1) * dh] for h in range(Hq)])
        off_k, off_v = 2 * Hq * dh, 2 * Hq * dh + Hkv * dh
        for g in range(Hkv):
            keys[g].append(_rot(rms(p[off_k + g * dh:off_k + (g + 1) * dh], kg), pos, r, base))
            vals[g].append(p[off_v + g * dh:off_v + (g + 1) * dh])
    outs = []
    for t in range(len(x)):
        o_cat = []
        for h in range(Hq):
            g = h // (Hq // Hkv)
            n_vis = pos0 + t + 1                                  # causal: keys at positions <= pos0 + t
            sc = [sum(qs[t][h][i] * keys[g][p][i] for i in range(dh)) / math.sqrt(dh) for p in range(n_vis)]
            m = max(sc)
            e = [math.exp(s - m) for s in sc]
            z = sum(e)
            o = [sum(e[p] / z * vals[g][p][i] for p in range(n_vis)) for i in range(dh)]
            o_cat += [o[i] * sig(gates[t][h][i]) for i in range(dh)]
        outs.append(matvec(w_out, o_cat))
    return np.array(outs), keys, vals


@pytest.mark.parametrize("T,L", [(1, 0), (2, 0), (2, 2)])
def test_fa_mixer_by_hand(T, L):
    r = np.random.default_rng(70 + 3 * T + L)
    d, Hq, Hkv, dh, rd, base = 6, 4, 2, 4, 2, 100.0
    x = r.normal(size=(T, d))
    w_in = r.normal(size=(2 * Hq * dh + 2 * Hkv * dh, d)) * 0.6
    qg, kg = 1 + 0.3 * r.normal(size=dh), 1 + 0.3 * r.normal(size=dh)
    w_out = r.normal(size=(d, Hq * dh))
    Kc = r.normal(size=(L, Hkv, dh)) if L else None
    Vc = r.normal(size=(L, Hkv, dh)) if L else None
    got, K_all, V_all = ops.fa_mixer(x, w_in, qg, kg, w_out, Kc, Vc, L, Hq, Hkv, dh, rd, base, EPS)
    ref, keys, vals = _fa_by_hand(x.tolist(), w_in.tolist(), qg.tolist(), kg.tolist(), w_out.tolist(),
                                  Kc.tolist() if L else [], Vc.tolist() if L else [], L, Hq, Hkv, dh, rd, base)
    assert np.allclose(got, ref, rtol=1e-11, atol=1e-12)
    for g in range(Hkv):
        assert np.allclose(K_all[:, g], np.array(keys[g]), atol=1e-13)
        assert np.allclose(V_all[:, g], np.array(vals[g]), atol=1e-13)


# ----------------------------------------------------------------------------- layer branch and head

TINY1 = synth.ModelShape(d=8, ffn=12, vocab=11, n_layers=4, loop_start=1, loop_end=3, loop_passes=1,
                         gdn_heads=2, gdn_dk=4, gdn_dv=4, fa_q_heads=2, fa_kv_heads=1, fa_head_dim=4,
                         rotary_dims=2, dtype="fp32", with_embedding=True)


@pytest.mark.parametrize("layer,kind", [(0, "gdn"), (3, "fa")])
def test_layer_branch_by_hand(layer, kind):
    """F = mix + FFN(RMSNorm(x + mix)) with mix = Mixer(RMSNorm(x)); the mixer itself is pinned above."""
    s = TINY1
    W = omodel.Weights(synth.make_weights(s, seed=3, std=0.4, gain_std=0.3))
    lw = W.layer(layer)
    r = np.random.default_rng(5 + layer)
    T = 2
    x = r.normal(size=(T, s.d))
    cache = omodel.new_cache()
    F = omodel.layer_branch(s, W, layer, kind, 0, x, cache, 0)
    S = np.zeros((s.gdn_heads, s.gdn_dv, s.gdn_dk))
    a = np.array([rms(list(x[t]), list(lw("attn_norm"))) for t in range(T)])
    if kind == "gdn":
        mix, S_ref = _gdn_by_hand(a.tolist(), lw("gdn_w_in").tolist(), list(lw("gdn_a_bias")),
                                  list(lw("gdn_b_bias")), lw("gdn_w_out").tolist(), S,
                                  s.gdn_heads, s.gdn_dk, s.gdn_dv)
        assert np.allclose(cache["state"][0], S_ref, atol=1e-12)
    else:
        mix, keys, _ = _fa_by_hand(a.tolist(), lw("fa_w_in").tolist(), list(lw("fa_q_norm")), list(lw("fa_k_norm")),
                                   lw("fa_w_out").tolist(), [], [], 0, s.fa_q_heads, s.fa_kv_heads,
                                   s.fa_head_dim, s.rotary_dims, s.rope_base)
        assert np.allclose(cache["kv"][0][0][:, 0], np.array(keys[0]), atol=1e-12)
    ref = []
    for t in range(T):
        u = [x[t][i] + mix[t][i] for i in range(s.d)]                     # u = x + mix
        un = rms(u, list(lw("ffn_norm")))
        gt = matvec(lw("ffn_w_gate").tolist(), un)
        up = matvec(lw("ffn_w_up").tolist(), un)
        hdn = [gt[j] * sig(gt[j]) * up[j] for j in range(s.ffn)]          # silu(gate) * up
        f = matvec(lw("ffn_w_down").tolist(), hdn)
        ref.append([mix[t][i] + f[i] for i in range(s.d)])                # F = mix + f
    assert np.allclose(F, np.array(ref), rtol=1e-11, atol=1e-12)


def test_lm_logits_by_hand():
    s = TINY1
    W = omodel.Weights(synth.make_weights(s, seed=4, std=0.4, gain_std=0.3))
    h = np.random.default_rng(6).normal(size=(2, s.d))
    got = ops.lm_logits(h, W["final_norm"], W["lm_head"], EPS)
    for t in range(2):
        hn = rms(list(h[t]), list(W["final_norm"]))
        ref = [sum(W["lm_head"][v][i] * hn[i] for i in range(s.d)) for v in range(s.vocab)]
        assert np.allclose(got[t], ref, rtol=1e-12, atol=1e-13)
    assert np.array_equal(ops.greedy(got), np.argmax(got, axis=-1))


def test_one_looped_execution_by_hand():
    """A stack whose only loop layer is a GDN layer run once: open, route, read, branch, write, merge."""
    s = synth.ModelShape(d=8, ffn=12, vocab=11, n_layers=2, loop_start=0, loop_end=1, loop_passes=1, group=4,
                         gdn_heads=2, gdn_dk=4, gdn_dv=4, fa_q_heads=2, fa_kv_heads=1, fa_head_dim=4,
                         rotary_dims=2, dtype="fp32", with_embedding=False)
    W = omodel.Weights(synth.make_weights(s, seed=8, std=0.4, gain_std=0.3))
    h = np.random.default_rng(9).normal(size=(1, 1, s.d))
    got, _ = omodel.forward_hidden(s, W, h)
    # execution 0 (layer 0, in the loop): streams X_0 = X_1 = h
    lw = W.layer(0)
    X = [list(h[0, 0]), list(h[0, 0])]
    flat = X[0] + X[1]
    fn = [c / math.sqrt(sum(t * t for t in flat) / len(flat) + EPS) for c in flat]
    l = [sum(fn[i] * lw("mhc_w_r")[i][j] for i in range(2 * s.d)) + lw("mhc_b_r")[j] for j in range(8)]
    pre = [sig(l[0]), sig(l[1])]
    post = [2 * sig(l[2]), 2 * sig(l[3])]
    M = [[math.exp(l[4]), math.exp(l[5])], [math.exp(l[6]), math.exp(l[7])]]
    for _ in range(s.sinkhorn_iters):
        M = [[M[i][j] / (M[i][0] + M[i][1]) for j in range(2)] for i in range(2)]
        M = [[M[i][j] / (M[0][j] + M[1][j]) for j in range(2)] for i in range(2)]
    x_in = [pre[0] * X[0][i] + pre[1] * X[1][i] for i in range(s.d)]
    F = omodel.layer_branch(s, W, 0, "gdn", 0, np.array([x_in]), omodel.new_cache(), 0)[0]
    Xn = [[M[r][0] * X[0][i] + M[r][1] * X[1][i] + post[r] * F[i] for i in range(s.d)] for r in range(2)]
    h1 = [(Xn[0][i] + Xn[1][i]) / 2 for i in range(s.d)]
    # execution 1 (layer 1, a GDN layer outside the loop): plain residual
    F1 = omodel.layer_branch(s, W, 1, "gdn", 1, np.array([h1]), omodel.new_cache(), 0)[0]
    ref = [h1[i] + F1[i] for i in range(s.d)]
    assert np.allclose(got[0, 0], ref, rtol=1e-11, atol=1e-12)
