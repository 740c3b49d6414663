"""Chunked (UT-transform) form of the gated delta rule -- a cross-check, not part of the oracle forward.

The GPU scan processes C tokens at a time.  This module writes that
re-association out in float64 so the tests can show it equals
`ops.gdn_recurrent` token by token; the oracle forward itself always uses the
recurrence.

Within a chunk with incoming state S0 and cumulative log-decay G_r = sum_{i<=r} g_i,
write gamma_r = exp(G_r).  Unrolling the recurrence S_r = alpha_r S_{r-1} + u_r k_r^T
with u_r = beta_r (v_r - alpha_r S_{r-1} k_r) gives
    S_r = gamma_r S0 + sum_{s<=r} (gamma_r/gamma_s) u_s k_s^T,
so the u_r satisfy the unit lower-triangular system
    (I + A) U = diag(beta) (V - diag(gamma) K S0^T),   A_rs = beta_r (gamma_r/gamma_s) k_r.k_s  (s < r).
With Tm = (I + A)^{-1} diag(beta):  W = Tm diag(gamma) K,  U = Tm V - W S0^T,
    O    = scale * [ diag(gamma) Q S0^T + (Q K^T o Gamma o M) U ],  Gamma_rs = gamma_r/gamma_s, M = (s <= r)
    S_C  = gamma_C S0 + U^T diag(gamma_C/gamma) K      (as [dv, dk]: sum_s u_s ((gamma_C/gamma_s) k_s)^T).
"""
from __future__ import annotations

import numpy as np

from .ops import f64


def gdn_chunked(q, k, v, g, beta, S0, scale, C):
    q, k, v, g, beta = f64(q), f64(k), f64(v), f64(g), f64(beta)
    S = f64(S0).copy()
    T, H, dk = q.shape
    dv = v.shape[2]
    o = np.zeros((T, H, dv))
    for h in range(H):
        Sh = S[h]
        for c0 in range(0, T, C):
            c1 = min(T, c0 + C)
            n = c1 - c0
            Q, K, V = q[c0:c1, h], k[c0:c1, h], v[c0:c1, h]
            G = np.cumsum(g[c0:c1, h])
            gam = np.exp(G)
            ratio = np.exp(G[:, None] - G[None, :])                  # gamma_r / gamma_s
            A = np.tril(beta[c0:c1, h][:, None] * ratio * (K @ K.T), -1)
            Tm = np.linalg.solve(np.eye(n) + A, np.diag(beta[c0:c1, h]))
            W = Tm @ (gam[:, None] * K)
            U = Tm @ V - W @ Sh.T
            mask = np.tril(np.ones((n, n)))
            o[c0:c1, h] = scale * ((gam[:, None] * Q) @ Sh.T + ((Q @ K.T) * ratio * mask) @ U)
            Sh = gam[-1] * Sh + U.T @ (np.exp(G[-1] - G)[:, None] * K)
        S[h] = Sh
    return o, S
