"""Pins of the oracle's per-operation definitions: closed forms, library routines, brute force, invariants."""
import numpy as np
import pytest
import scipy.special
import torch

from oracle import gdn_chunked, ops

RNG = np.random.default_rng(1234)


# ----------------------------------------------------------------------------- elementwise

def test_activations_match_library():
    x = RNG.normal(size=1000) * 8
    assert np.allclose(ops.sigmoid(x), scipy.special.expit(x), rtol=1e-14, atol=0)
    t = torch.tensor(x, dtype=torch.float64)
    assert np.allclose(ops.silu(x), torch.nn.functional.silu(t).numpy(), rtol=1e-13, atol=1e-300)
    assert np.allclose(ops.softplus(x), torch.nn.functional.softplus(t).numpy(), rtol=1e-13)
    assert ops.softplus(800.0) == 800.0 and ops.silu(0.0) == 0.0


def test_rmsnorm_properties():
    x = RNG.normal(size=(7, 64)) * 3
    y = ops.rmsnorm(x, None, 0.0)
    assert np.allclose(np.sqrt(np.mean(y * y, axis=-1)), 1.0, atol=1e-14)
    assert np.allclose(ops.rmsnorm(5 * x, None, 0.0), y, atol=1e-14)           # scale invariance
    w = RNG.normal(size=64)
    assert np.allclose(ops.rmsnorm(x, w, 0.0), y * w, atol=1e-14)
    # library routine: torch's rms_norm (same eps convention: inside the root)
    ref = torch.nn.functional.rms_norm(torch.tensor(x), (64,), torch.tensor(w), eps=1e-6).numpy()
    assert np.allclose(ops.rmsnorm(x, w, 1e-6), ref, rtol=1e-12, atol=1e-14)


def test_l2norm_unit_and_direction():
    x = RNG.normal(size=(5, 3, 128))
    y = ops.l2norm(x, 0.0)
    assert np.allclose(np.linalg.norm(y, axis=-1), 1.0, atol=1e-14)
    assert np.allclose(y * np.linalg.norm(x, axis=-1, keepdims=True), x, atol=1e-13)


def test_swiglu_matches_torch():
    x = RNG.normal(size=(4, 32))
    wg, wu, wd = RNG.normal(size=(48, 32)), RNG.normal(size=(48, 32)), RNG.normal(size=(32, 48))
    t = lambda a: torch.tensor(a)
    ref = torch.nn.functional.linear(torch.nn.functional.silu(torch.nn.functional.linear(t(x), t(wg)))
                                     * torch.nn.functional.linear(t(x), t(wu)), t(wd)).numpy()
    assert np.allclose(ops.swiglu_ffn(x, wg, wu, wd), ref, rtol=1e-12, atol=1e-12)


# ----------------------------------------------------------------------------- Sinkhorn

def _closed_form_2x2(A):
    """Doubly stochastic scaling of a positive 2x2 matrix: [[p, 1-p], [1-p, p]]."""
    p = np.sqrt(A[0, 0] * A[1, 1]) / (np.sqrt(A[0, 0] * A[1, 1]) + np.sqrt(A[0, 1] * A[1, 0]))
    return np.array([[p, 1 - p], [1 - p, p]])


def test_sinkhorn_2x2_closed_form():
    for _ in range(200):
        L = RNG.uniform(-1, 1, size=(2, 2))
        M = ops.sinkhorn(L, 20)
        assert np.allclose(M, _closed_form_2x2(np.exp(L)), atol=1e-8)
        assert np.allclose(ops.sinkhorn(L, 400), _closed_form_2x2(np.exp(L)), atol=1e-14)


def test_sinkhorn_columns_exact_rows_converge():
    L = RNG.normal(size=(64, 2, 2)) * 2
    prev = None
    for it in range(1, 21):
        M = ops.sinkhorn(L, it)
        assert np.allclose(M.sum(axis=-2), 1.0, atol=1e-14)      # each iteration ends on a column step
        err = np.abs(M.sum(axis=-1) - 1.0).max(axis=-1)
        if prev is not None:
            assert np.all(err <= prev + 1e-15)                    # row error never grows
        prev = err


def test_sinkhorn_toy_repro_assertion(golden):
    """[teardown] §六: 2x2 logits ~ 0.5 N(0,1); after 20 iterations row and column sums are 1 within 1e-2."""
    atol = golden["sinkhorn_toy_atol"]["value"]
    for _ in range(100):
        M = ops.sinkhorn(RNG.normal(size=(2, 2)) * 0.5, golden["sinkhorn_iters"]["value"])
        assert np.allclose(M.sum(-1), 1, atol=atol) and np.allclose(M.sum(-2), 1, atol=atol)


def test_sinkhorn_is_a_diagonal_scaling_and_log_domain_equivalent():
    """For n x n: M = diag(r) exp(L) diag(c) (rank-1 ratio), equal to a log-domain Sinkhorn written independently."""
    for n in (2, 3, 4):
        L = RNG.normal(size=(n, n))
        M = ops.sinkhorn(L, 20)
        R = M / np.exp(L)
        assert np.linalg.matrix_rank(R, tol=1e-10 * np.abs(R).max()) == 1
        f, g = np.zeros(n), np.zeros(n)                          # log-domain scalings
        for _ in range(20):
            f = -scipy.special.logsumexp(L + g[None, :], axis=1)
            g = -scipy.special.logsumexp(L + f[:, None], axis=0)
        assert np.allclose(M, np.exp(L + f[:, None] + g[None, :]), atol=1e-13)


def test_sinkhorn_permutation_equivariance():
    L = RNG.normal(size=(3, 3))
    P = np.eye(3)[[2, 0, 1]]
    assert np.allclose(ops.sinkhorn(P @ L @ P.T, 20), P @ ops.sinkhorn(L, 20) @ P.T, atol=1e-14)


# ----------------------------------------------------------------------------- GDN

def _gdn_inputs(T, H, dk, dv, seed=0, strong_decay=False):
    r = np.random.default_rng(seed)
    q = ops.l2norm(r.normal(size=(T, H, dk)), 1e-6)
    k = ops.l2norm(r.normal(size=(T, H, dk)), 1e-6)
    v = r.normal(size=(T, H, dv))
    a = r.normal(size=(T, H)) * (3.0 if strong_decay else 1.0)
    g, beta = ops.gdn_gates(a, r.normal(size=(T, H)), np.zeros(H), np.zeros(H))
    S0 = r.normal(size=(H, dv, dk)) * 0.3
    return q, k, v, g, beta, S0


def test_gdn_gates_closed_forms():
    a = RNG.normal(size=100) * 4
    g, beta = ops.gdn_gates(a, a, 0.0, 0.0)
    assert np.allclose(np.exp(g), scipy.special.expit(-a), rtol=1e-13)   # exp(-softplus(a)) = sigmoid(-a)
    assert np.allclose(beta, scipy.special.expit(a), rtol=1e-14)
    assert np.all(g < 0)


@pytest.mark.parametrize("T,C", [(150, 64), (64, 64), (1, 64), (37, 16), (200, 128)])
def test_gdn_chunked_equals_recurrence(T, C):
    q, k, v, g, beta, S0 = _gdn_inputs(T, 3, 32, 24, seed=T + C, strong_decay=(T == 200))
    o1, S1 = ops.gdn_recurrent(q, k, v, g, beta, S0, 0.17)
    o2, S2 = gdn_chunked.gdn_chunked(q, k, v, g, beta, S0, 0.17, C)
    assert np.allclose(o1, o2, rtol=1e-10, atol=1e-12)
    assert np.allclose(S1, S2, rtol=1e-10, atol=1e-12)


def test_gdn_transition_matrix_form_brute_force():
    """S_t = S_{t-1} [alpha_t (I - beta_t k_t k_t^T)] + beta_t v_t k_t^T with explicit dk x dk matrices."""
    T, H, dk, dv = 8, 2, 6, 5
    q, k, v, g, beta, S0 = _gdn_inputs(T, H, dk, dv, seed=7)
    o, S = ops.gdn_recurrent(q, k, v, g, beta, S0, 1.0)
    for h in range(H):
        Sb = S0[h].copy()
        for t in range(T):
            At = np.exp(g[t, h]) * (np.eye(dk) - beta[t, h] * np.outer(k[t, h], k[t, h]))
            Sb = Sb @ At + beta[t, h] * np.outer(v[t, h], k[t, h])
            assert np.allclose(o[t, h], Sb @ q[t, h], atol=1e-13)
        assert np.allclose(S[h], Sb, atol=1e-13)


def test_gdn_decay_one_beta_zero_keeps_state():
    T, H, dk, dv = 20, 2, 16, 8
    q, k, v, _, _, S0 = _gdn_inputs(T, H, dk, dv, seed=3)
    o, S = ops.gdn_recurrent(q, k, v, np.zeros((T, H)), np.zeros((T, H)), S0, 0.5)
    assert np.array_equal(S, S0)
    assert np.allclose(o, 0.5 * np.einsum("hij,thj->thi", S0, q), atol=1e-14)


def test_gdn_delta_rule_write_and_overwrite():
    H, dk, dv = 1, 16, 8
    r = np.random.default_rng(5)
    S0 = r.normal(size=(H, dv, dk))
    kk = ops.l2norm(r.normal(size=(1, H, dk)), 0.0)
    v1, v2 = r.normal(size=(1, H, dv)), r.normal(size=(1, H, dv))
    ones, zeros = np.ones((1, H)), np.zeros((1, H))
    _, S = ops.gdn_recurrent(kk, kk, v1, zeros, ones, S0, 1.0)      # alpha = 1, beta = 1, |k| = 1
    assert np.allclose(S[0] @ kk[0, 0], v1[0, 0], atol=1e-13)       # S_new k = v exactly
    _, S = ops.gdn_recurrent(np.concatenate([kk, kk]), np.concatenate([kk, kk]), np.concatenate([v1, v2]),
                             np.zeros((2, H)), np.ones((2, H)), S0, 1.0)
    assert np.allclose(S[0] @ kk[0, 0], v2[0, 0], atol=1e-13)       # the same key is overwritten, not summed


def test_gdn_orthonormal_keys_are_exact_memory():
    dk, dv = 8, 5
    r = np.random.default_rng(9)
    Qm, _ = np.linalg.qr(r.normal(size=(dk, dk)))
    keys = Qm.T[:, None, :]                                          # [T=dk, H=1, dk] orthonormal rows
    vals = r.normal(size=(dk, 1, dv))
    _, S = ops.gdn_recurrent(keys, keys, vals, np.zeros((dk, 1)), np.ones((dk, 1)), np.zeros((1, dv, dk)), 1.0)
    for j in range(dk):
        assert np.allclose(S[0] @ keys[j, 0], vals[j, 0], atol=1e-13)


def test_gdn_zero_decay_forgets():
    H, dk, dv = 2, 8, 4
    q, k, v, _, beta, S0 = _gdn_inputs(1, H, dk, dv, seed=11)
    _, S = ops.gdn_recurrent(q, k, v, np.full((1, H), -np.inf), beta, S0, 1.0)   # alpha = 0
    assert np.allclose(S, beta[0][:, None, None] * np.einsum("hi,hj->hij", v[0], k[0]), atol=1e-15)


# ----------------------------------------------------------------------------- RoPE + attention

def test_rope_zero_dims_is_identity_and_preserves_norm():
    x = RNG.normal(size=(9, 3, 32))
    assert np.array_equal(ops.rope(x, np.arange(9), 0, 10000.0), x)
    y = ops.rope(x, np.arange(9) * 7, 16, 10000.0)
    assert np.allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1), atol=1e-12)
    assert np.array_equal(y[..., 16:], x[..., 16:])                 # only the rotary dims move


def test_rope_matches_complex_rotation():
    x = RNG.normal(size=(6, 2, 24))
    pos = np.array([0, 1, 5, 100, 4095, 131071])
    r = 8
    z = x[..., 0:r:2] + 1j * x[..., 1:r:2]
    theta = 10000.0 ** (-np.arange(r // 2) * 2.0 / r)
    z = z * np.exp(1j * pos[:, None, None] * theta[None, None, :])
    y = ops.rope(x, pos, r, 10000.0)
    assert np.allclose(y[..., 0:r:2], z.real, atol=1e-9) and np.allclose(y[..., 1:r:2], z.imag, atol=1e-9)


def test_rope_relative_position():
    q, k = RNG.normal(size=(1, 1, 64)), RNG.normal(size=(1, 1, 64))
    dots = [np.sum(ops.rope(q, [m], 64, 10000.0) * ops.rope(k, [m - 3], 64, 10000.0)) for m in (3, 10, 500)]
    assert np.allclose(dots, dots[0], atol=1e-10)


def test_attention_matches_torch_sdpa_gqa():
    Tq, Hq, Hkv, dh = 13, 8, 2, 16
    q, k, v = RNG.normal(size=(Tq, Hq, dh)), RNG.normal(size=(Tq, Hkv, dh)), RNG.normal(size=(Tq, Hkv, dh))
    o = ops.attention(q, k, v, np.arange(Tq))
    tq = torch.tensor(q).transpose(0, 1)
    tk = torch.tensor(k).transpose(0, 1).repeat_interleave(Hq // Hkv, dim=0)
    tv = torch.tensor(v).transpose(0, 1).repeat_interleave(Hq // Hkv, dim=0)
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=True).transpose(0, 1).numpy()
    assert np.allclose(o, ref, rtol=1e-12, atol=1e-12)


def test_attention_offsets_and_special_cases():
    Hq, Hkv, dh = 4, 1, 8
    k, v = RNG.normal(size=(10, Hkv, dh)), RNG.normal(size=(10, Hkv, dh))
    q = RNG.normal(size=(3, Hq, dh))
    full = ops.attention(np.concatenate([RNG.normal(size=(7, Hq, dh)), q]), k, v, np.arange(10))
    assert np.allclose(ops.attention(q, k, v, np.arange(7, 10)), full[7:], atol=1e-14)   # decode rows = prefill rows
    one = ops.attention(q[:1], k[:1], v[:1], [0])
    assert np.allclose(one, np.repeat(v[:1], Hq, axis=1), atol=1e-15)                   # one key: output = v
    zero = ops.attention(np.zeros((10, Hq, dh)), k, v, np.arange(10))
    prefix_mean = np.cumsum(v, axis=0) / np.arange(1, 11)[:, None, None]
    assert np.allclose(zero, np.repeat(prefix_mean, Hq, axis=1), atol=1e-13)            # q = 0: causal mean


# ----------------------------------------------------------------------------- mHC

def test_mhc_zero_routing_closed_form():
    X = RNG.normal(size=(5, 2, 16))
    H_pre, H_post, H_res = ops.mhc_coeffs(X, np.zeros((32, 8)), np.zeros(8), 1e-6, 20)
    assert np.allclose(H_pre, 0.5) and np.allclose(H_post, 1.0) and np.allclose(H_res, 0.5)


def test_mhc_stream_sum_conservation():
    X, F = RNG.normal(size=(6, 2, 16)), RNG.normal(size=(6, 16))
    H_pre, H_post, H_res = ops.mhc_coeffs(X, RNG.normal(size=(32, 8)), RNG.normal(size=8), 1e-6, 20)
    Xn = ops.mhc_write(X, F, H_post, H_res)
    # columns of H_res sum to 1 after the last Sinkhorn step, so the stream total is kept
    assert np.allclose(Xn.sum(1), X.sum(1) + H_post.sum(1)[:, None] * F, atol=1e-12)
    # routing reads from the RMS-normed flat state: a per-token rescale of X changes nothing
    a = ops.mhc_coeffs(3.7 * X, RNG.normal(size=(32, 8)) * 0, np.ones(8), 0.0, 20)
    b = ops.mhc_coeffs(X, RNG.normal(size=(32, 8)) * 0, np.ones(8), 0.0, 20)
    assert all(np.allclose(u, w) for u, w in zip(a, b))


def test_mhc_coeffs_by_hand():
    """One token written out without the helper functions."""
    X = RNG.normal(size=(1, 2, 4))
    w_r, b_r = RNG.normal(size=(8, 8)), RNG.normal(size=8)
    flat = np.concatenate([X[0, 0], X[0, 1]])
    l = flat / np.sqrt(np.mean(flat ** 2) + 1e-6) @ w_r + b_r
    H_pre, H_post, H_res = ops.mhc_coeffs(X, w_r, b_r, 1e-6, 20)
    assert np.allclose(H_pre[0], 1 / (1 + np.exp(-l[0:2])))
    assert np.allclose(H_post[0], 2 / (1 + np.exp(-l[2:4])))
    M = np.exp(l[4:8]).reshape(2, 2)
    for _ in range(20):
        M = M / M.sum(1, keepdims=True)
        M = M / M.sum(0, keepdims=True)
    assert np.allclose(H_res[0], M)
    x_in = ops.mhc_read(X, H_pre)
    assert np.allclose(x_in[0], H_pre[0, 0] * X[0, 0] + H_pre[0, 1] * X[0, 1])
    F = RNG.normal(size=(1, 4))
    Xn = ops.mhc_write(X, F, H_post, H_res)
    assert np.allclose(Xn[0, 0], H_res[0, 0, 0] * X[0, 0] + H_res[0, 0, 1] * X[0, 1] + H_post[0, 0] * F[0])
    assert np.allclose(Xn[0, 1], H_res[0, 1, 0] * X[0, 0] + H_res[0, 1, 1] * X[0, 1] + H_post[0, 1] * F[0])
