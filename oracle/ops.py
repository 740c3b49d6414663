"""Operations of one looped-hybrid decoder layer, in float64 (oracle, test infrastructure only).

Every function is the plain definition, written out; no blocking, fusion or
re-association beyond what the definition states.  Inputs may be numpy arrays
or torch tensors (bf16 values are widened exactly); results are float64.

Readings of points the pages leave open are marked READING and listed in the
design notes; all of them follow the plainest form the pages support.
"""
from __future__ import annotations

import numpy as np


def f64(x):
    """Exact widening of a numpy array or torch tensor (any float dtype) to float64."""
    if hasattr(x, "detach"):
        x = x.detach().to("cpu")
        import torch
        if x.dtype == torch.bfloat16 or x.dtype == torch.float16:
            x = x.to(torch.float32)
        return x.numpy().astype(np.float64)
    return np.asarray(x, dtype=np.float64)


# ----------------------------------------------------------------------------- basic maps

def sigmoid(x):
    """1 / (1 + e^-x)."""
    x = np.asarray(x, dtype=np.float64)
    with np.errstate(over="ignore"):
        return 1.0 / (1.0 + np.exp(-x))


def softplus(x):
    """log(1 + e^x), overflow-free."""
    return np.logaddexp(0.0, np.asarray(x, dtype=np.float64))


def silu(x):
    return x * sigmoid(x)


def linear(x, w):
    """y = x W^T for a weight stored [out, in] (nn.Linear convention)."""
    return f64(x) @ f64(w).T


def rmsnorm(x, w, eps):
    """x / sqrt(mean(x^2) + eps) * w over the last axis.

    READING: the pages do not name the norm; the backbone is declared
    qwen3_5_text ([probe] §01), whose layers use pre-norm RMSNorm, so RMSNorm
    with eps inside the square root is used.  w=None means no gain.
    """
    x = f64(x)
    y = x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    return y if w is None else y * f64(w)


def l2norm(x, eps):
    """x / sqrt(sum(x^2) + eps) over the last axis (GDN query/key normalisation)."""
    x = f64(x)
    return x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + eps)


# ----------------------------------------------------------------------------- FFN

def swiglu_ffn(x, w_gate, w_up, w_down):
    """down( silu(x Wg^T) * (x Wu^T) ): the three-matrix SwiGLU FFN ([teardown] §二)."""
    return linear(silu(linear(x, w_gate)) * linear(x, w_up), w_down)


# ----------------------------------------------------------------------------- Gated DeltaNet

def gdn_gates(a, b, a_bias, b_bias):
    """Log-decay g = -softplus(a + a_bias) (so alpha = exp(g) in (0,1)) and beta = sigmoid(b + b_bias).

    READING ([teardown] §三 says only "gate + delta rule"): the Gated-DeltaNet
    form with a softplus decay and a sigmoid write strength.
    """
    g = -softplus(f64(a) + f64(a_bias))
    beta = sigmoid(f64(b) + f64(b_bias))
    return g, beta


def gdn_recurrent(q, k, v, g, beta, S0, scale):
    """Token-by-token gated delta rule ([teardown] §三: a constant-size state updated by gate + delta rule).

    Shapes: q, k [T, H, dk]; v [T, H, dv]; g, beta [T, H]; S0 [H, dv, dk]
    (the state maps keys to values).  For each token t and head:
        S <- alpha_t * S                      (alpha_t = exp(g_t), the gate)
        S <- S + beta_t (v_t - S k_t) k_t^T   (delta rule: move S k_t toward v_t)
        o_t = scale * S q_t
    Returns o [T, H, dv] and the final state [H, dv, dk].
    """
    q, k, v, g, beta = f64(q), f64(k), f64(v), f64(g), f64(beta)
    S = f64(S0).copy()
    T = q.shape[0]
    o = np.zeros(v.shape, dtype=np.float64)
    for t in range(T):
        S *= np.exp(g[t])[:, None, None]
        pred = np.einsum("hij,hj->hi", S, k[t])                 # S k_t
        S += (beta[t][:, None] * (v[t] - pred))[:, :, None] * k[t][:, None, :]
        o[t] = scale * np.einsum("hij,hj->hi", S, q[t])
    return o, S


def gdn_split_projection(P, H, dk, dv):
    """Split the GDN input projection [T, 2*H*dk + H*dv + 2*H] into q, k, v, a, b (row blocks in that order)."""
    T = P.shape[0]
    o = 0
    q = P[:, o:o + H * dk].reshape(T, H, dk); o += H * dk
    k = P[:, o:o + H * dk].reshape(T, H, dk); o += H * dk
    v = P[:, o:o + H * dv].reshape(T, H, dv); o += H * dv
    a = P[:, o:o + H]; o += H
    b = P[:, o:o + H]
    return q, k, v, a, b


def gdn_mixer(x_normed, w_in, a_bias, b_bias, w_out, S0, H, dk, dv, eps):
    """GDN token mixer of one layer: projections, L2-normalised q/k, gates, recurrence, output map.

    READING: 16 heads x dk = dv = 128 at full width, q/k L2-normalised,
    output scale 1/sqrt(dk), no short convolution and no output norm.
    """
    P = linear(x_normed, w_in)
    q, k, v, a, b = gdn_split_projection(P, H, dk, dv)
    q, k = l2norm(q, eps), l2norm(k, eps)
    g, beta = gdn_gates(a, b, a_bias, b_bias)
    o, S = gdn_recurrent(q, k, v, g, beta, S0, 1.0 / np.sqrt(dk))
    return linear(o.reshape(o.shape[0], H * dv), w_out), S


# ----------------------------------------------------------------------------- GDN variant: short conv + gated output norm

def causal_conv_silu(x, w, state):
    """Depthwise causal convolution over time, then SiLU, per channel.

    READING ([probe] §01 names the backbone qwen3_5_text; its Gated-DeltaNet layers pass
    the q, k, v channels through a short causal depthwise convolution and SiLU before the
    recurrence): x [T, C]; w [C, K]; state [K-1, C] = the K-1 inputs before x (zeros at
    sequence start).  y_t[c] = silu(sum_j w[c, j] * x_{t-(K-1)+j}[c]), so w[:, K-1] weighs
    the current token.  Returns y [T, C] and the new state (the last K-1 inputs).
    """
    x, w = f64(x), f64(w)
    K = w.shape[1]
    st = np.zeros((K - 1, x.shape[1])) if state is None else f64(state)
    ext = np.concatenate([st, x], axis=0)                      # [K-1+T, C]
    T = x.shape[0]
    y = np.zeros_like(x)
    for t in range(T):
        for j in range(K):
            y[t] += w[:, j] * ext[t + j]
    return silu(y), ext[T:].copy()


def gated_rmsnorm(o, z, w, eps):
    """Output gate of the variant: RMSNorm of each head's output (gain w over dv) times silu(z).

    o, z [T, H, dv] -> [T, H, dv].  READING: the gated output norm of the qwen3_5_text
    Gated-DeltaNet layer ([probe] §01).
    """
    return rmsnorm(o, w, eps) * silu(f64(z))


def gdn_split_projection_v2(P, Hk, Hv, dk, dv):
    """Split the variant's input projection into q, k (Hk heads), v, z (Hv heads), a, b (Hv)."""
    T = P.shape[0]
    o = 0
    q = P[:, o:o + Hk * dk]; o += Hk * dk
    k = P[:, o:o + Hk * dk]; o += Hk * dk
    v = P[:, o:o + Hv * dv]; o += Hv * dv
    z = P[:, o:o + Hv * dv].reshape(T, Hv, dv); o += Hv * dv
    a = P[:, o:o + Hv]; o += Hv
    b = P[:, o:o + Hv]
    return q, k, v, z, a, b


def gdn_mixer_v2(x_normed, w_in, conv_w, a_bias, b_bias, o_norm, w_out, S0, conv0, Hk, Hv, dk, dv, eps):
    """GDN token mixer of the variant ([probe] §01: backbone qwen3_5_text).

    READING: projections q, k (Hk heads), v, z (Hv heads), a, b (Hv); the q | k | v
    channels pass through causal_conv_silu; q and k are L2-normalised per head; value
    head h reads key head h // (Hv // Hk); gates and recurrence as in gdn_mixer; each
    head's output goes through gated_rmsnorm with z; then the output map.
    Returns (mix, final state [Hv, dv, dk], conv state [K-1, 2*Hk*dk + Hv*dv]).
    """
    P = linear(x_normed, w_in)
    T = P.shape[0]
    q, k, v, z, a, b = gdn_split_projection_v2(P, Hk, Hv, dk, dv)
    y, conv_new = causal_conv_silu(np.concatenate([q, k, v], axis=1), conv_w, conv0)
    q = l2norm(y[:, :Hk * dk].reshape(T, Hk, dk), eps)
    k = l2norm(y[:, Hk * dk:2 * Hk * dk].reshape(T, Hk, dk), eps)
    v = y[:, 2 * Hk * dk:].reshape(T, Hv, dv)
    rep = Hv // Hk
    q, k = np.repeat(q, rep, axis=1), np.repeat(k, rep, axis=1)     # head h -> key head h // rep
    g, beta = gdn_gates(a, b, a_bias, b_bias)
    o, S = gdn_recurrent(q, k, v, g, beta, S0, 1.0 / np.sqrt(dk))
    o = gated_rmsnorm(o, z, o_norm, eps)
    return linear(o.reshape(T, Hv * dv), w_out), S, conv_new


# ----------------------------------------------------------------------------- full attention

def rope(x, pos, rotary_dims, base):
    """Rotate dims [0, rotary_dims) of each head in adjacent pairs (2j, 2j+1) by angle pos * base^(-2j/rotary_dims).

    [teardown] §三: interleaved M-RoPE with rotary factor 0.25, so 64 of the
    256 head dims carry position and the other 192 pass through unchanged.
    For text every M-RoPE section sees the same position, so it is 1-D RoPE.
    READING: "interleaved" pairs adjacent dims; base 10000.
    x [T, H, dh], pos [T] (absolute positions).
    """
    x = f64(x).copy()
    if rotary_dims == 0:
        return x
    j = np.arange(rotary_dims // 2, dtype=np.float64)
    theta = base ** (-2.0 * j / rotary_dims)                        # [r/2]
    ang = np.asarray(pos, dtype=np.float64)[:, None] * theta[None, :]  # [T, r/2]
    c, s = np.cos(ang)[:, None, :], np.sin(ang)[:, None, :]
    x0 = x[..., 0:rotary_dims:2].copy()
    x1 = x[..., 1:rotary_dims:2].copy()
    x[..., 0:rotary_dims:2] = x0 * c - x1 * s
    x[..., 1:rotary_dims:2] = x0 * s + x1 * c
    return x


def attention(q, k, v, q_pos, causal=True):
    """Brute-force GQA softmax attention.

    q [Tq, Hq, dh] at absolute positions q_pos [Tq]; k, v [Tkv, Hkv, dh] at
    positions 0..Tkv-1.  Query head h reads KV head h // (Hq // Hkv).  Scores
    are q.k / sqrt(dh); with `causal`, key position p is visible to a query at
    position t iff p <= t.  Softmax in float64 after subtracting the row max.
    """
    q, k, v = f64(q), f64(k), f64(v)
    Tq, Hq, dh = q.shape
    Tkv, Hkv, _ = k.shape
    rep = Hq // Hkv
    q_pos = np.asarray(q_pos)
    out = np.zeros((Tq, Hq, v.shape[2]), dtype=np.float64)
    kpos = np.arange(Tkv)
    for h in range(Hq):
        kv = h // rep
        s = (q[:, h, :] @ k[:, kv, :].T) / np.sqrt(dh)            # [Tq, Tkv]
        if causal:
            s = np.where(kpos[None, :] <= q_pos[:, None], s, -np.inf)
        s = s - np.max(s, axis=1, keepdims=True)
        p = np.exp(s)
        p /= np.sum(p, axis=1, keepdims=True)
        out[:, h, :] = p @ v[:, kv, :]
    return out


def fa_split_projection(P, Hq, Hkv, dh):
    """Split the FA input projection [T, 2*Hq*dh + 2*Hkv*dh] into q, gate, k, v (row blocks in that order)."""
    T = P.shape[0]
    o = 0
    q = P[:, o:o + Hq * dh].reshape(T, Hq, dh); o += Hq * dh
    gate = P[:, o:o + Hq * dh].reshape(T, Hq, dh); o += Hq * dh
    k = P[:, o:o + Hkv * dh].reshape(T, Hkv, dh); o += Hkv * dh
    v = P[:, o:o + Hkv * dh].reshape(T, Hkv, dh)
    return q, gate, k, v


def fa_qk(q, k, q_norm, k_norm, pos, rotary_dims, base, eps):
    """QK-norm (RMSNorm over the head dim, gain shared by all heads) then partial RoPE ([teardown] §三)."""
    q = rope(rmsnorm(q, q_norm, eps), pos, rotary_dims, base)
    k = rope(rmsnorm(k, k_norm, eps), pos, rotary_dims, base)
    return q, k


def fa_mixer(x_normed, w_in, q_norm, k_norm, w_out, K_cache, V_cache, pos0, Hq, Hkv, dh,
             rotary_dims, base, eps):
    """Full-attention token mixer: GQA 16q/4kv, QK-norm, partial RoPE, causal softmax, sigmoid output gate.

    [teardown] §三: GQA with 16 query and 4 KV heads, QK normalisation and an
    attention output gate.  READING: the gate is elementwise sigmoid(x Wg^T)
    over all q heads, applied before the output map.
    K_cache, V_cache [L, Hkv, dh] hold this execution's earlier tokens
    (normed and rotated keys); returns (mix, K_all, V_all).
    """
    T = x_normed.shape[0]
    P = linear(x_normed, w_in)
    q, gate, k, v = fa_split_projection(P, Hq, Hkv, dh)
    pos = pos0 + np.arange(T)
    q, k = fa_qk(q, k, q_norm, k_norm, pos, rotary_dims, base, eps)
    K_all = np.concatenate([K_cache, k], axis=0) if K_cache is not None else k
    V_all = np.concatenate([V_cache, v], axis=0) if V_cache is not None else v
    o = attention(q, K_all, V_all, pos, causal=True)
    o = o * sigmoid(gate)
    return linear(o.reshape(T, Hq * dh), w_out), K_all, V_all


# ----------------------------------------------------------------------------- mHC

def sinkhorn(logits, iters):
    """Sinkhorn-Knopp projection of exp(logits) toward a doubly stochastic matrix.

    [teardown] §五, [wiki] §二, [probe] §02: the stream-mixing matrix is
    normalised by 20 Sinkhorn iterations (FP32 on the device).  Each
    iteration divides every row by its sum, then every column by its sum.
    The max is subtracted before exp (a no-op on the result).
    logits [..., n, n] -> matrix [..., n, n].
    """
    L = f64(logits)
    M = np.exp(L - np.max(L, axis=(-2, -1), keepdims=True))
    for _ in range(iters):
        M = M / np.sum(M, axis=-1, keepdims=True)
        M = M / np.sum(M, axis=-2, keepdims=True)
    return M


def mhc_coeffs(X, w_r, b_r, eps, iters):
    """Per-token routing of the two-stream residual ([teardown] §五, [wiki] §二; form of the mHC paper named in [probe] §02).

    X [T, n, d] (n = 2 streams).  The n*d-vector of each token is RMS-normed
    (no gain) and mapped by w_r [n*d, 8] (FP32 parameters) plus b_r [8]:
        l[0:2] -> H_pre  = sigmoid           (how the layer reads the streams)
        l[2:4] -> H_post = 2 * sigmoid       (how the layer output is written)
        l[4:8] -> H_res  = Sinkhorn(exp(.))  (2x2 stream mix, row-major)
    READING: the pages fix only the Sinkhorn step; the linear-map-of-RMS-normed
    state parametrisation is this build's stated choice.
    Returns H_pre [T, n], H_post [T, n], H_res [T, n, n].
    """
    X = f64(X)
    T, n, d = X.shape
    flat = X.reshape(T, n * d)
    l = rmsnorm(flat, None, eps) @ f64(w_r) + f64(b_r)
    H_pre = sigmoid(l[:, 0:n])
    H_post = 2.0 * sigmoid(l[:, n:2 * n])
    H_res = sinkhorn(l[:, 2 * n:2 * n + n * n].reshape(T, n, n), iters)
    return H_pre, H_post, H_res


def mhc_read(X, H_pre):
    """Layer input x_in = sum_s H_pre[s] X_s."""
    return np.einsum("ts,tsd->td", f64(H_pre), f64(X))


def mhc_write(X, F, H_post, H_res):
    """X'_s = sum_t H_res[s, t] X_t + H_post[s] F (row s of H_res feeds stream s, as in the [teardown] §六 repro)."""
    return np.einsum("tsu,tud->tsd", f64(H_res), f64(X)) + f64(H_post)[:, :, None] * f64(F)[:, None, :]


def mhc_open(h, n=2):
    """Entering the loop block copies the hidden state into n streams ([teardown] §六)."""
    h = f64(h)
    return np.repeat(h[:, None, :], n, axis=1)


def mhc_merge(X):
    """Leaving the loop block averages the streams ([teardown] §六)."""
    return np.mean(f64(X), axis=1)


# ----------------------------------------------------------------------------- head

def lm_logits(h, final_norm, lm_head, eps):
    """logits = RMSNorm(h) W_lm^T (untied LM head; READING: the pages do not say tied)."""
    return linear(rmsnorm(h, final_norm, eps), lm_head)


def greedy(logits):
    """Greedy next token: argmax over the vocabulary, lowest index on ties."""
    return np.argmax(f64(logits), axis=-1).astype(np.int64)
