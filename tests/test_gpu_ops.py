"""Per-op parity: each C-ABI entry point on the GPU against the oracle on the same seeded inputs."""
import numpy as np
import pytest
import torch

import synth
from conftest import TOL, rel_l2, to64
from oracle import ops

pytestmark = pytest.mark.gpu

DT = {"fp32": torch.float32, "bf16": torch.bfloat16}
# GDN states are fp32 for both storage types (the bf16 inputs are exact in fp32)
STATE_TOL = {"fp32": TOL["fp32"], "bf16": TOL["gdn_state"]}


def rnd(shape, seed, name, std=1.0, dtype="fp32", dev="cuda"):
    return synth.normal(shape, std, seed, name).to(DT[dtype]).to(dev)


# ----------------------------------------------------------------------------- Sinkhorn + mHC

@pytest.mark.parametrize("n", [2, 3, 4])
def test_sinkhorn_fp32(cuda, n):
    import looped_hybrid_attention_b200 as L
    N = 1000
    Lg = rnd((N, n, n), 0, f"sk{n}", std=2.0)
    out = torch.empty_like(Lg)
    L.sinkhorn_fp32(Lg, out, 20)
    ref = ops.sinkhorn(to64(Lg), 20)
    assert np.abs(to64(out) - ref).max() <= TOL["sinkhorn"]
    # zero iterations = normalised exp only
    L.sinkhorn_fp32(Lg, out, 0)
    e = np.exp(to64(Lg) - to64(Lg).max(axis=(1, 2), keepdims=True))
    assert np.abs(to64(out) - e).max() < 1e-6


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("d,N", [(256, 37), (4096, 19), (4096, 64), (4096, 100), (4096, 1501), (4096, 4133),
                                  (256, 2050), (1024, 1100), (2048, 1057), (8192, 1030)])
def test_mhc_modes(cuda, dtype, d, N):
    import looped_hybrid_attention_b200 as L
    code = L.BF16 if dtype == "bf16" else L.F32
    eps, iters = 1e-6, 20
    h = rnd((N, d), 1, "h", dtype=dtype)
    F = rnd((N, d), 2, "F", dtype=dtype)
    w_r = rnd((2 * d, 8), 3, "wr", std=0.02)
    b_r = rnd((8,), 4, "br", std=0.5)
    X = torch.empty((N, 2, d), dtype=DT[dtype], device=cuda)
    x_in = torch.empty((N, d), dtype=DT[dtype], device=cuda)
    c0 = torch.empty((N, 8), device=cuda)
    tol = TOL[dtype]
    # OPEN: X = (h, h), route from it
    L.mhc_route_mix(L.MHC_OPEN, h, None, None, w_r, b_r, X, x_in, None, c0, N, d, eps, iters, code)
    Xo = ops.mhc_open(to64(h))
    assert np.array_equal(to64(X), Xo)
    pre, post, res = ops.mhc_coeffs(Xo, to64(w_r), to64(b_r), eps, iters)
    c = to64(c0)
    assert rel_l2(c[:, 0:2], pre) < 1e-5 and rel_l2(c[:, 2:4], post) < 1e-5
    assert np.abs(c[:, 4:8].reshape(N, 2, 2) - res).max() <= TOL["sinkhorn"]
    assert rel_l2(to64(x_in), ops.mhc_read(Xo, c[:, 0:2])) < tol
    # MIX: X' = H_res X + H_post F, then route from X' as stored
    X_prev = X.clone()
    c1 = torch.empty_like(c0)
    L.mhc_route_mix(L.MHC_MIX, X, F, c0, w_r, b_r, X, x_in, None, c1, N, d, eps, iters, code)
    Xm = ops.mhc_write(to64(X_prev), to64(F), c[:, 2:4], c[:, 4:8].reshape(N, 2, 2))
    assert rel_l2(to64(X), Xm) < tol
    pre, post, res = ops.mhc_coeffs(to64(X), to64(w_r), to64(b_r), eps, iters)
    c = to64(c1)
    assert rel_l2(c[:, 0:2], pre) < 1e-5 and rel_l2(c[:, 2:4], post) < 1e-5
    assert np.abs(c[:, 4:8].reshape(N, 2, 2) - res).max() <= TOL["sinkhorn"]
    assert rel_l2(to64(x_in), ops.mhc_read(to64(X), pre)) < tol
    # ROUTE only: X unchanged
    X_keep = X.clone()
    L.mhc_route_mix(L.MHC_ROUTE, X, None, None, w_r, b_r, None, x_in, None, c1, N, d, eps, iters, code)
    assert torch.equal(X, X_keep)
    assert rel_l2(to64(c1), c) < 1e-6
    # MERGE: mix then average the streams
    hm = torch.empty((N, d), dtype=DT[dtype], device=cuda)
    L.mhc_route_mix(L.MHC_MERGE, X, F, c1, None, None, None, None, hm, None, N, d, eps, iters, code)
    Xm = ops.mhc_write(to64(X), to64(F), c[:, 2:4], c[:, 4:8].reshape(N, 2, 2))
    assert rel_l2(to64(hm), ops.mhc_merge(Xm)) < tol


def test_mhc_zero_routing_is_plain_residual(cuda):
    import looped_hybrid_attention_b200 as L
    N, d = 10, 256
    h = rnd((N, d), 5, "h0")
    F = rnd((N, d), 6, "F0")
    X = torch.empty((N, 2, d), device=cuda)
    x_in = torch.empty((N, d), device=cuda)
    c = torch.empty((N, 8), device=cuda)
    z = torch.zeros((2 * d, 8), device=cuda)
    L.mhc_route_mix(L.MHC_OPEN, h, None, None, z, z[0], X, x_in, None, c, N, d, 1e-6, 20, L.F32)
    assert torch.allclose(c, torch.tensor([0.5, 0.5, 1, 1, 0.5, 0.5, 0.5, 0.5], device=cuda))
    assert torch.allclose(x_in, h, atol=1e-6)
    hm = torch.empty_like(h)
    L.mhc_route_mix(L.MHC_MERGE, X, F, c, None, None, None, None, hm, None, N, d, 1e-6, 20, L.F32)
    assert torch.allclose(hm, h + F, atol=1e-5)


def _residual_logit_sets():
    """2x2 residual logits with spreads (max - min) from 0.1 to 100: both sides of the 40 at which
    the fused kernel's Sinkhorn changes from the row-odds recurrence to literal divisions."""
    r = np.random.default_rng(17)
    sets = []
    for spread in (0.1, 1.0, 4.0, 10.0, 25.0, 39.5, 40.5, 60.0, 100.0):
        for _ in range(3):
            l = r.uniform(0.0, 1.0, size=4)
            l = (l - l.min()) / (l.max() - l.min()) * spread - spread / 2
            sets.append(l)
    return sets


@pytest.mark.parametrize("dtype,d,N", [("fp32", 256, 10), ("fp32", 256, 1100), ("bf16", 4096, 10),
                                       ("bf16", 4096, 64), ("bf16", 4096, 1100)])
def test_mhc_sinkhorn_of_bias_only_routing(cuda, dtype, d, N):
    """With w_r = 0 the routing logits are exactly b_r for every token, so the fused kernel's
    H_res is the 20-iteration Sinkhorn of exp(b_r[4:8]) and must match it within 1e-6 (FP32
    Sinkhorn, "Loop-9B engineering teardown" §五), in the routing of OPEN and of MIX."""
    import looped_hybrid_attention_b200 as L
    code = L.BF16 if dtype == "bf16" else L.F32
    h = rnd((N, d), 31, "hs", dtype=dtype)
    F = rnd((N, d), 32, "Fs", dtype=dtype)
    w_r = torch.zeros((2 * d, 8), device=cuda)
    X = torch.empty((N, 2, d), dtype=DT[dtype], device=cuda)
    x_in = torch.empty((N, d), dtype=DT[dtype], device=cuda)
    c0, c1 = torch.empty((N, 8), device=cuda), torch.empty((N, 8), device=cuda)
    worst = 0.0
    for l4 in _residual_logit_sets():
        b = np.concatenate([np.array([0.3, -1.2, 0.8, 2.5]), l4]).astype(np.float32)
        b_r = torch.tensor(b, device=cuda)
        ref = ops.sinkhorn(b[4:8].astype(np.float64).reshape(2, 2), 20)
        L.mhc_route_mix(L.MHC_OPEN, h, None, None, w_r, b_r, X, x_in, None, c0, N, d, 1e-6, 20, code)
        L.mhc_route_mix(L.MHC_MIX, X, F, c0, w_r, b_r, X, x_in, None, c1, N, d, 1e-6, 20, code)
        for c in (to64(c0), to64(c1)):
            assert np.isfinite(c).all()
            err = np.abs(c[:, 4:8].reshape(N, 2, 2) - ref[None]).max()
            worst = max(worst, err)
            assert err <= TOL["sinkhorn"], (l4, err)
            assert np.abs(c[:, 0:2] - ops.sigmoid(b[0:2].astype(np.float64))).max() < 1e-6
            assert np.abs(c[:, 2:4] - 2 * ops.sigmoid(b[2:4].astype(np.float64))).max() < 2e-6
    assert worst <= TOL["sinkhorn"]


@pytest.mark.parametrize("N", [10, 1100])
def test_mhc_extreme_routing_logits(cuda, N):
    """Residual logits 95 apart: one row of exp(l - max) sums to a denormal, where a
    reciprocal-and-multiply normalisation would overflow; the Sinkhorn must still match."""
    import looped_hybrid_attention_b200 as L
    d = 256
    h = rnd((N, d), 11, "hx", dtype="bf16")
    X = torch.empty((N, 2, d), dtype=torch.bfloat16, device=cuda)
    x_in = torch.empty((N, d), dtype=torch.bfloat16, device=cuda)
    c = torch.empty((N, 8), device=cuda)
    w_r = torch.zeros((2 * d, 8), device=cuda)
    b_r = torch.tensor([0.0, 0.0, 0.0, 0.0, 0.0, 1.0, -95.0, -95.0], device=cuda)
    L.mhc_route_mix(L.MHC_OPEN, h, None, None, w_r, b_r, X, x_in, None, c, N, d, 1e-6, 20, L.BF16)
    pre, post, res = ops.mhc_coeffs(ops.mhc_open(to64(h)), to64(w_r), to64(b_r), 1e-6, 20)
    got = to64(c)
    assert np.isfinite(got).all()
    assert np.abs(got[:, 4:8].reshape(N, 2, 2) - res).max() < 1e-5
    assert np.abs(got[:, 0:4] - np.concatenate([pre, post], axis=1)).max() < 1e-6


# ----------------------------------------------------------------------------- norms, embedding, argmax

@pytest.mark.parametrize("d", [4096, 256, 2048, 6144, 520])
@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_rmsnorm_with_residual(cuda, dtype, d):
    """Widths for every register layout of the row (1, 2 or 3 eight-element pieces per
    thread) and one (d = 520) that takes the shared-memory kernel."""
    import looped_hybrid_attention_b200 as L
    M = 33
    x, r = rnd((M, d), 7, "x", dtype=dtype), rnd((M, d), 8, "r", dtype=dtype)
    w = rnd((d,), 9, "w", dtype=dtype, std=0.1) + 1
    y, s = torch.empty_like(x), torch.empty_like(x)
    L.rmsnorm(x, w, y, 1e-6)
    assert rel_l2(to64(y), ops.rmsnorm(to64(x), to64(w), 1e-6)) < TOL[dtype]
    L.rmsnorm(x, w, y, 1e-6, r=r, sum_out=s)
    assert rel_l2(to64(s), to64(x) + to64(r)) < TOL[dtype]
    assert rel_l2(to64(y), ops.rmsnorm(to64(s), to64(w), 1e-6)) < TOL[dtype]


def test_embed_and_argmax(cuda):
    import looped_hybrid_attention_b200 as L
    V, d = 1000, 256
    E = rnd((V, d), 10, "E", dtype="bf16")
    ids = synth.uniform_ids((77,), V, 0).to(cuda)
    out = torch.empty((77, d), dtype=torch.bfloat16, device=cuda)
    L.embed(ids, E, out)
    assert torch.equal(out, E[ids.long()])
    assert L.device_error() == 0
    bad = ids.clone()
    bad[3] = V
    L.embed(bad, E, out)
    torch.cuda.synchronize()
    assert L.device_error() == 1 and torch.all(out[3] == 0)
    lg = rnd((5, 248320), 11, "lg")
    lg[2, 17] = lg[2, 99] = 100.0          # tie -> lowest index
    nx = torch.empty(5, dtype=torch.int32, device=cuda)
    L.argmax(lg, nx)
    ref = ops.greedy(to64(lg))
    assert np.array_equal(nx.cpu().numpy(), ref) and nx[2].item() == 17


# ----------------------------------------------------------------------------- projections

@pytest.mark.parametrize("split_k", [False, True])
@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("M,N,K", [(200, 300, 256), (1, 1000, 512), (130, 64, 4096), (64, 4104, 2048),
                                   (64, 1000, 12288), (16, 130, 520), (17, 384, 8), (33, 4000, 4096),
                                   (100, 200, 1000), (128, 1000, 2048)])
def test_linear_epilogues(cuda, dtype, M, N, K, split_k):
    """Every epilogue against fp64; M <= 128 covers each batch-tile width (16/32/64/128 rows),
    ragged N and K, with the partial-sum workspace (split tiles) and without it (whole tiles)."""
    import looped_hybrid_attention_b200 as L
    ws = None
    if split_k:
        nb = max(L.linear_workspace_bytes(M, N, K, e) for e in (0, 1, 2, 3))
        ws = torch.zeros(max(nb, 16) // 4, device=cuda)
    X = rnd((M, K), 12, "X", dtype=dtype)
    W = rnd((N, K), 13, "W", std=0.02, dtype=dtype)
    W2 = rnd((N, K), 14, "W2", std=0.02, dtype=dtype)
    R = rnd((M, N), 15, "R", dtype=dtype)
    Y = torch.empty((M, N), dtype=DT[dtype], device=cuda)
    ref = ops.linear(to64(X), to64(W))
    L.linear(X, W, Y, L.EPI_STORE, workspace=ws)
    assert rel_l2(to64(Y), ref) < TOL[dtype]
    L.linear(X, W, Y, L.EPI_ADD, R=R, workspace=ws)
    assert rel_l2(to64(Y), ref + to64(R)) < TOL[dtype]
    L.linear(X, W, Y, L.EPI_SWIGLU, W2=W2, workspace=ws)
    assert rel_l2(to64(Y), ops.silu(ref) * ops.linear(to64(X), to64(W2))) < TOL[dtype]
    Yf = torch.empty((M, N), dtype=torch.float32, device=cuda)
    L.linear(X, W, Yf, L.EPI_F32, workspace=ws)
    assert rel_l2(to64(Yf), ref) < (1e-5 if dtype == "fp32" else 1e-4)
    if ws is not None:
        torch.cuda.synchronize()
        assert L.device_error() == 0
        assert int(torch.count_nonzero(ws)) == 0, "a call must leave the workspace zero-filled"


# the projections of one decode step at batch 64 (and the LM head): (N, K, epilogue)
DECODE_GEMMS = [(6176, 4096, "store"), (4096, 2048, "add"), (10240, 4096, "store"), (4096, 4096, "add"),
                (12288, 4096, "swiglu"), (4096, 12288, "add"), (248320, 4096, "f32")]


@pytest.mark.parametrize("N,K,epi", DECODE_GEMMS)
def test_linear_decode_shapes(cuda, N, K, epi):
    """bf16 projections at M = 64 (the decode batch) in the full 9B shapes with the runtime's
    zero-filled workspace, twice in a row (the second call relies on the first leaving the
    workspace zero-filled); sampled output columns against fp64."""
    import looped_hybrid_attention_b200 as L
    M = 64
    code = {"store": L.EPI_STORE, "add": L.EPI_ADD, "swiglu": L.EPI_SWIGLU, "f32": L.EPI_F32}[epi]
    gen = lambda seed: torch.Generator(device=cuda).manual_seed(seed)
    X = torch.randn((M, K), device=cuda, generator=gen(11)).to(torch.bfloat16)
    W = (0.02 * torch.randn((N, K), device=cuda, generator=gen(12))).to(torch.bfloat16)
    W2 = (0.02 * torch.randn((N, K), device=cuda, generator=gen(13))).to(torch.bfloat16) if epi == "swiglu" else None
    R = torch.randn((M, N), device=cuda, generator=gen(14)).to(torch.bfloat16) if epi == "add" else None
    Y = torch.empty((M, N), device=cuda, dtype=torch.float32 if epi == "f32" else torch.bfloat16)
    ws = torch.zeros(L.linear_workspace_bytes(M, N, K, code) // 4 + 1, device=cuda)
    cols = np.unique(np.r_[0:130, N // 2 - 70:N // 2 + 70, N - 130:N])
    xr = to64(X)
    ref = ops.linear(xr, to64(W[cols]))
    if epi == "swiglu":
        ref = ops.silu(ref) * ops.linear(xr, to64(W2[cols]))
    if epi == "add":
        ref = ref + to64(R[:, cols])
    for _ in range(2):
        L.linear(X, W, Y, code, W2=W2, R=R, workspace=ws)
        torch.cuda.synchronize()
        assert L.device_error() == 0
        assert rel_l2(to64(Y[:, cols]), ref) < (1e-4 if epi == "f32" else TOL["bf16"])
        assert int(torch.count_nonzero(ws)) == 0


# ----------------------------------------------------------------------------- Gated DeltaNet

def _gdn_inputs(B, T, H, dk, dv, dtype, seed):
    q = ops.l2norm(synth.normal((B, T, H, dk), 1.0, seed, "q").double().numpy(), 1e-6)
    k = ops.l2norm(synth.normal((B, T, H, dk), 1.0, seed, "k").double().numpy(), 1e-6)
    v = synth.normal((B, T, H, dv), 1.0, seed, "v")
    a = synth.normal((B, T, H), 1.5, seed, "a").double().numpy()
    b = synth.normal((B, T, H), 1.0, seed, "b").double().numpy()
    g, beta = ops.gdn_gates(a, b, 0.0, 0.0)
    S0 = synth.normal((B, H, dv, dk), 0.1, seed, "S0")
    t = lambda x: torch.tensor(x).to(DT[dtype]).cuda() if not torch.is_tensor(x) else x.to(DT[dtype]).cuda()
    return t(q), t(k), t(v), torch.tensor(g, dtype=torch.float32).cuda(), \
        torch.tensor(beta, dtype=torch.float32).cuda(), S0.cuda()


@pytest.mark.parametrize("two_pass", [False, True])
@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("B,T,H,dk", [(2, 150, 3, 64), (1, 64, 2, 128), (1, 1, 2, 128), (2, 200, 2, 128)])
def test_gdn_chunk_vs_recurrence(cuda, dtype, B, T, H, dk, two_pass):
    import looped_hybrid_attention_b200 as L
    q, k, v, g, beta, S = _gdn_inputs(B, T, H, dk, dk, dtype, seed=T + H)
    S0 = S.clone()
    out = torch.empty_like(v)
    scale = 1.0 / np.sqrt(dk)
    ws = torch.empty(L.gdn_workspace_bytes(B, T, H, dk, dk) // 4, device=cuda) if two_pass else None
    L.gdn_chunk_fwd(q, k, v, g, beta, S, out, scale, workspace=ws)
    tol = TOL[dtype]
    for b in range(B):
        o_ref, S_ref = ops.gdn_recurrent(to64(q[b]), to64(k[b]), to64(v[b]), to64(g[b]), to64(beta[b]),
                                         to64(S0[b]), scale)
        assert rel_l2(to64(out[b]), o_ref) < tol
        assert rel_l2(to64(S[b]), S_ref) < STATE_TOL[dtype]


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_gdn_step_and_chunk_continue(cuda, dtype):
    """Chunked prefill of T tokens then single-token steps equals the recurrence over T + 3 tokens."""
    import looped_hybrid_attention_b200 as L
    B, T, H, dk = 3, 70, 4, 128
    q, k, v, g, beta, S = _gdn_inputs(B, T + 3, H, dk, dk, dtype, seed=5)
    S0 = S.clone()
    out = torch.empty((B, T, H, dk), dtype=DT[dtype], device=cuda)
    scale = 1.0 / np.sqrt(dk)
    ws = torch.empty(L.gdn_workspace_bytes(B, T, H, dk, dk) // 4, device=cuda)
    L.gdn_chunk_fwd(q[:, :T].contiguous(), k[:, :T].contiguous(), v[:, :T].contiguous(), g[:, :T].contiguous(),
                    beta[:, :T].contiguous(), S, out, scale, workspace=ws)
    o_steps = []
    for t in range(T, T + 3):
        ot = torch.empty((B, H, dk), dtype=DT[dtype], device=cuda)
        L.gdn_step(q[:, t].contiguous(), k[:, t].contiguous(), v[:, t].contiguous(), g[:, t].contiguous(),
                   beta[:, t].contiguous(), S, ot, scale)
        o_steps.append(ot)
    for b in range(B):
        o_ref, S_ref = ops.gdn_recurrent(to64(q[b]), to64(k[b]), to64(v[b]), to64(g[b]), to64(beta[b]),
                                         to64(S0[b]), scale)
        got = np.concatenate([to64(out[b, :T])] + [to64(o[b])[None] for o in o_steps])
        assert rel_l2(got, o_ref) < TOL[dtype]
        assert rel_l2(to64(S[b]), S_ref) < STATE_TOL[dtype]


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("dk,dv,offset", [(64, 64, 0), (64, 64, 1), (128, 128, 0), (128, 128, 1)])
def test_gdn_step_layouts(cuda, dtype, dk, dv, offset):
    """One recurrent step for both state access paths: four rows per warp with 16/8-byte
    accesses (aligned state) and the plain form (a state that starts 4 bytes past an
    aligned address)."""
    import looped_hybrid_attention_b200 as L
    B, H = 3, 5
    q, k, v, g, beta, S0 = _gdn_inputs(B, 1, H, dk, dv, dtype, seed=21)
    n = B * H * dv * dk
    buf = torch.zeros(n + offset, device=cuda)
    S = buf[offset:].view(B, H, dv, dk)
    S.copy_(S0)
    out = torch.empty((B, H, dv), dtype=DT[dtype], device=cuda)
    scale = 1.0 / np.sqrt(dk)
    L.gdn_step(q[:, 0].contiguous(), k[:, 0].contiguous(), v[:, 0].contiguous(), g[:, 0].contiguous(),
               beta[:, 0].contiguous(), S, out, scale)
    for b in range(B):
        o_ref, S_ref = ops.gdn_recurrent(to64(q[b]), to64(k[b]), to64(v[b]), to64(g[b]), to64(beta[b]),
                                         to64(S0[b]), scale)
        assert rel_l2(to64(out[b]), o_ref[0]) < TOL[dtype]
        assert rel_l2(to64(S[b]), S_ref) < STATE_TOL[dtype]


@pytest.mark.parametrize("two_pass", [False, True])
@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_gdn_extreme_gates(cuda, dtype, two_pass):
    """Gates far from the random-init range: decays from ~1 down to exp(-75) per token (a
    chunk's cumulative log decay reaches the thousands, so many exp(G) underflow to 0), and
    write strengths beta pressed against 0 and 1.  The chunked form never divides by a decay,
    so it must stay finite and match the recurrence."""
    import looped_hybrid_attention_b200 as L
    B, T, H, dk = 1, 300, 2, 128
    q, k, v, _, _, S = _gdn_inputs(B, T, H, dk, dk, dtype, seed=77)
    a = synth.normal((B, T, H), 25.0, 77, "a_x").double().numpy()
    bb = synth.normal((B, T, H), 10.0, 77, "b_x").double().numpy()
    g_np, beta_np = ops.gdn_gates(a, bb, 0.0, 0.0)
    g = torch.tensor(g_np, dtype=torch.float32, device=cuda)
    beta = torch.tensor(beta_np, dtype=torch.float32, device=cuda)
    assert g_np.min() < -50 and (beta_np < 1e-3).any() and (beta_np > 1 - 1e-3).any()
    S0 = S.clone()
    out = torch.empty_like(v)
    scale = 1.0 / np.sqrt(dk)
    ws = torch.empty(L.gdn_workspace_bytes(B, T, H, dk, dk) // 4, device=cuda) if two_pass else None
    L.gdn_chunk_fwd(q, k, v, g, beta, S, out, scale, workspace=ws)
    torch.cuda.synchronize()
    assert torch.isfinite(out.float()).all() and torch.isfinite(S).all()
    o_ref, S_ref = ops.gdn_recurrent(to64(q[0]), to64(k[0]), to64(v[0]), to64(g[0]), to64(beta[0]), to64(S0[0]),
                                     scale)
    # fp32: the chunked form takes each decay exp(G_r - G_s) from the chunk's fp32 cumulative
    # log decays G, so an exponent carries an absolute error up to about |G| 2^-24 -- here
    # |G| reaches 64 * 76 ~ 4,900, i.e. ~3e-4 -- which the recurrence (one factor per token)
    # does not have; the bound for these gates is 1e-4 instead of the 1e-5 of the ordinary range
    tol = 1e-4 if dtype == "fp32" else TOL[dtype]
    assert rel_l2(to64(out[0]), o_ref) < tol
    assert rel_l2(to64(S[0]), S_ref) < 1e-4            # the fp32-grade state bound of both paths


def test_gdn_special_cases(cuda):
    import looped_hybrid_attention_b200 as L
    B, T, H, dk = 1, 100, 2, 64
    q, k, v, g, beta, S = _gdn_inputs(B, T, H, dk, dk, "fp32", seed=9)
    S0 = S.clone()
    out = torch.empty_like(v)
    # decay 1 (g = 0) and beta = 0 leave the state unchanged; o = scale S0 q
    L.gdn_chunk_fwd(q, k, v, torch.zeros_like(g), torch.zeros_like(beta), S, out, 0.5)
    assert torch.allclose(S, S0, rtol=0, atol=1e-6)
    ref = 0.5 * np.einsum("hij,thj->thi", to64(S0[0]), to64(q[0]))
    assert rel_l2(to64(out[0]), ref) < 1e-5
    # T = 0: nothing changes
    L.gdn_chunk_fwd(q[:, :0], k[:, :0], v[:, :0], g[:, :0], beta[:, :0], S, out[:, :0], 0.5)
    assert torch.equal(S, S0)


@pytest.mark.parametrize("H", [16, 6])
def test_gdn_prep(cuda, H):
    """Four heads per warp (H % 4 == 0) and one (H = 6)."""
    import looped_hybrid_attention_b200 as L
    M, dk, dv = 50, 128, 128
    n_in = 2 * H * dk + H * dv + 2 * H
    P = rnd((M, n_in), 20, "P", dtype="bf16")
    ab, bb = rnd((H,), 21, "ab"), rnd((H,), 22, "bb")
    q = torch.empty((M, H, dk), dtype=torch.bfloat16, device=cuda)
    k, v = torch.empty_like(q), torch.empty((M, H, dv), dtype=torch.bfloat16, device=cuda)
    g, beta = torch.empty((M, H), device=cuda), torch.empty((M, H), device=cuda)
    L.gdn_prep(P, ab, bb, q, k, v, g, beta, H, dk, dv, 1e-6)
    rq, rk, rv, ra, rb = ops.gdn_split_projection(to64(P), H, dk, dv)
    assert rel_l2(to64(q), ops.l2norm(rq, 1e-6)) < TOL["bf16"]
    assert rel_l2(to64(k), ops.l2norm(rk, 1e-6)) < TOL["bf16"]
    assert np.array_equal(to64(v), rv)
    gr, br = ops.gdn_gates(ra, rb, to64(ab), to64(bb))
    assert rel_l2(to64(g), gr) < 1e-5 and rel_l2(to64(beta), br) < 1e-5


@pytest.mark.parametrize("M,H", [(300, 16), (8192, 16), (129, 4)])
def test_gdn_in_proj_fused_prep(cuda, M, H):
    """The GDN input projection with the preparation in its epilogue: the same q, k, v, g, beta as
    the stored projection + gdn_prep, and the oracle's split, L2 norms and gates of x W_in^T."""
    import looped_hybrid_attention_b200 as L
    d, dk, dv, eps = 1024, 128, 128, 1e-6
    n_in = 2 * H * dk + H * dv + 2 * H
    x = rnd((M, d), 50, "xg", dtype="bf16")
    w_in = rnd((n_in, d), 51, "wg", std=0.03, dtype="bf16")
    ab, bb = rnd((H,), 52, "abg"), rnd((H,), 53, "bbg")
    out = [torch.empty((M, H, dk), dtype=torch.bfloat16, device=cuda) for _ in range(3)]
    g, beta = torch.empty((M, H), device=cuda), torch.empty((M, H), device=cuda)
    L.gdn_in_proj(x, w_in, ab, bb, *out, g, beta, H, dk, dv, eps)
    P = torch.empty((M, n_in), dtype=torch.bfloat16, device=cuda)
    L.linear(x, w_in, P, L.EPI_STORE)
    ref = [torch.empty_like(o) for o in out]
    g2, beta2 = torch.empty_like(g), torch.empty_like(beta)
    L.gdn_prep(P, ab, bb, *ref, g2, beta2, H, dk, dv, eps)
    torch.cuda.synchronize()
    for o, r in zip(out, ref):                     # the fused path skips the bf16 rounding of P
        assert rel_l2(to64(o), to64(r)) < 5e-3
    rows = np.r_[0:8, M - 8:M]                     # the oracle on sampled rows
    Pn = ops.linear(to64(x[rows]), to64(w_in))
    rq, rk, rv, ra, rb = ops.gdn_split_projection(Pn, H, dk, dv)
    assert rel_l2(to64(out[0][rows]), ops.l2norm(rq, eps)) < TOL["bf16"]
    assert rel_l2(to64(out[1][rows]), ops.l2norm(rk, eps)) < TOL["bf16"]
    assert rel_l2(to64(out[2][rows]), rv) < TOL["bf16"]
    rg, rbeta = ops.gdn_gates(ra, rb, to64(ab), to64(bb))
    assert rel_l2(to64(g[rows]), rg) < 1e-3 and rel_l2(to64(beta[rows]), rbeta) < 1e-3
    with pytest.raises(L.LoopError) as e:          # decode-sized batches take the stored path
        L.gdn_in_proj(x[:64], w_in, ab, bb, *[o[:64] for o in out], g[:64], beta[:64], H, dk, dv, eps)
    assert e.value.status == 7


@pytest.mark.slow
def test_gdn_chunk_full_length_sampled_heads(cuda):
    """The bench's shape (T = 8192, 16 heads x 128, bf16): heads 0 and 15 against the recurrence."""
    import looped_hybrid_attention_b200 as L
    B, T, H, dk = 1, 8192, 16, 128
    q, k, v, g, beta, S = _gdn_inputs(B, T, H, dk, dk, "bf16", seed=77)
    S0 = S.clone()
    out = torch.empty_like(v)
    scale = 1.0 / np.sqrt(dk)
    ws = torch.empty(L.gdn_workspace_bytes(B, T, H, dk, dk) // 4, device=cuda)
    L.gdn_chunk_fwd(q, k, v, g, beta, S, out, scale, workspace=ws)
    for h in (0, 15):
        sl = slice(h, h + 1)
        o_ref, S_ref = ops.gdn_recurrent(to64(q[0, :, sl]), to64(k[0, :, sl]), to64(v[0, :, sl]), to64(g[0, :, sl]),
                                         to64(beta[0, :, sl]), to64(S0[0, sl]), scale)
        assert rel_l2(to64(out[0, :, sl]), o_ref) < TOL["bf16"]
        assert rel_l2(to64(S[0, sl]), S_ref) < STATE_TOL["bf16"]



@pytest.mark.slow
def test_gdn_chunk_long_context(cuda):
    """The long-context prefill shape (T = 131,072, 16 heads x 128, bf16): 2,048 chunks carried
    through one state; head 7's outputs and final state against the token recurrence."""
    import looped_hybrid_attention_b200 as L
    B, T, H, dk = 1, 131072, 16, 128
    gen = torch.Generator(device=cuda).manual_seed(78)
    q = torch.nn.functional.normalize(torch.randn(B, T, H, dk, device=cuda, generator=gen), dim=-1).to(torch.bfloat16)
    k = torch.nn.functional.normalize(torch.randn(B, T, H, dk, device=cuda, generator=gen), dim=-1).to(torch.bfloat16)
    v = torch.randn(B, T, H, dk, device=cuda, generator=gen).to(torch.bfloat16)
    # decays near 1 keep the state's memory long (the regime where position errors would show)
    g = -torch.nn.functional.softplus(torch.randn(B, T, H, device=cuda, generator=gen) - 5.0)
    beta = torch.sigmoid(torch.randn(B, T, H, device=cuda, generator=gen))
    S = 0.1 * torch.randn(B, H, dk, dk, device=cuda, generator=gen)
    S0 = S.clone()
    out = torch.empty_like(v)
    scale = 1.0 / np.sqrt(dk)
    ws = torch.empty(L.gdn_workspace_bytes(B, T, H, dk, dk) // 4, device=cuda)
    L.gdn_chunk_fwd(q, k, v, g, beta, S, out, scale, workspace=ws)
    torch.cuda.synchronize()
    assert L.device_error() == 0
    sl = slice(7, 8)
    o_ref, S_ref = ops.gdn_recurrent(to64(q[0, :, sl]), to64(k[0, :, sl]), to64(v[0, :, sl]), to64(g[0, :, sl]),
                                     to64(beta[0, :, sl]), to64(S0[0, sl]), scale)
    got = to64(out[0, :, sl])
    assert rel_l2(got, o_ref) < TOL["bf16"]
    assert rel_l2(got[-4096:], o_ref[-4096:]) < TOL["bf16"]      # the last chunks on their own
    assert rel_l2(to64(S[0, sl]), S_ref) < TOL["gdn_state"]


# ----------------------------------------------------------------------------- attention

def _fa_case(B, T, Hq, Hkv, dh, dtype, seed):
    n_in = 2 * Hq * dh + 2 * Hkv * dh
    P = rnd((B * T, n_in), seed, "Pfa", dtype=dtype)
    qn = rnd((dh,), seed, "qn", std=0.1, dtype=dtype) + 1
    kn = rnd((dh,), seed, "kn", std=0.1, dtype=dtype) + 1
    return P, qn, kn


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("B,T,Hq,Hkv,dh,rot,pos0", [(1, 70, 4, 1, 64, 16, 0), (2, 33, 16, 4, 256, 64, 5),
                                                    (1, 130, 16, 4, 256, 64, 0)])
def test_fa_prep_and_attention(cuda, dtype, B, T, Hq, Hkv, dh, rot, pos0):
    import looped_hybrid_attention_b200 as L
    eps, base = 1e-6, 10000.0
    cap = pos0 + T + 7
    P, qn, kn = _fa_case(B, T, Hq, Hkv, dh, dtype, seed=T)
    qo = torch.empty((B * T, Hq, dh), dtype=DT[dtype], device=cuda)
    Kc = torch.zeros((B, Hkv, cap, dh), dtype=DT[dtype], device=cuda)
    Vc = torch.zeros_like(Kc)
    if pos0:      # earlier tokens already in the slab
        Kc[:, :, :pos0] = rnd((B, Hkv, pos0, dh), 99, "Kprev", dtype=dtype).to(DT[dtype])
        Vc[:, :, :pos0] = rnd((B, Hkv, pos0, dh), 98, "Vprev", dtype=dtype).to(DT[dtype])
    L.fa_prep(P, qn, kn, qo, Kc, Vc, cap, B, T, pos0, Hq, Hkv, dh, rot, base, eps)
    tol = TOL[dtype]
    Pn = to64(P).reshape(B, T, -1)
    for b in range(B):
        q, gate, k, v = ops.fa_split_projection(Pn[b], Hq, Hkv, dh)
        rq, rk = ops.fa_qk(q, k, to64(qn), to64(kn), pos0 + np.arange(T), rot, base, eps)
        assert rel_l2(to64(qo.view(B, T, Hq, dh)[b]), rq) < tol
        assert rel_l2(to64(Kc[b, :, pos0:pos0 + T]).transpose(1, 0, 2), rk) < tol
        assert np.array_equal(to64(Vc[b, :, pos0:pos0 + T]).transpose(1, 0, 2), v)
    # attention with the gate, reading q from the compact buffer and the gate from P
    out = torch.empty((B * T, Hq * dh), dtype=DT[dtype], device=cuda)
    gate_view = P[:, Hq * dh:]
    ws = torch.empty(max(1, L.gqa_workspace_bytes(B, T, pos0 + T, Hq, dh) // 4), device=cuda)
    for workspace in (None, ws):
        L.gqa_attn(qo, Hq * dh, Kc, Vc, cap, gate_view, P.stride(0), out, B, T, pos0 + T, pos0, Hq, Hkv, dh,
                   True, workspace)
        for b in range(B):
            qb = to64(qo.view(B, T, Hq, dh)[b])
            K = to64(Kc[b, :, :pos0 + T]).transpose(1, 0, 2)
            V = to64(Vc[b, :, :pos0 + T]).transpose(1, 0, 2)
            ref = ops.attention(qb, K, V, pos0 + np.arange(T))
            _, gate, _, _ = ops.fa_split_projection(Pn[b], Hq, Hkv, dh)
            ref = ref * ops.sigmoid(gate)
            assert rel_l2(to64(out.view(B, T, Hq, dh)[b]), ref) < tol


@pytest.mark.parametrize("B,T,pos0,rot", [(1, 130, 0, 64), (2, 33, 5, 64), (1, 300, 0, 0), (1, 1100, 17, 64)])
def test_attention_fused_query_norm_and_rotary(cuda, B, T, pos0, rot):
    """gqa_attn_fused_q on the raw projection: queries QK-normed and rotated inside the attention
    kernel, keys and values from fa_prep with no q_out (K/V only).  Against the oracle's QK-norm,
    rotary and brute-force attention, and against the unfused fa_prep + gqa_attn path."""
    import looped_hybrid_attention_b200 as L
    Hq, Hkv, dh, eps, base = 16, 4, 256, 1e-6, 10000.0
    cap = pos0 + T + 3
    P, qn, kn = _fa_case(B, T, Hq, Hkv, dh, "bf16", seed=T + 1)
    Kc = torch.zeros((B, Hkv, cap, dh), dtype=torch.bfloat16, device=cuda)
    Vc = torch.zeros_like(Kc)
    if pos0:
        Kc[:, :, :pos0] = rnd((B, Hkv, pos0, dh), 97, "Kprev", dtype="bf16")
        Vc[:, :, :pos0] = rnd((B, Hkv, pos0, dh), 96, "Vprev", dtype="bf16")
    L.fa_prep(P, qn, kn, None, Kc, Vc, cap, B, T, pos0, Hq, Hkv, dh, rot, base, eps)
    out = torch.empty((B * T, Hq * dh), dtype=torch.bfloat16, device=cuda)
    gate_view = P[:, Hq * dh:]
    L.gqa_attn_fused_q(P, P.stride(0), qn, rot, base, eps, Kc, Vc, cap, gate_view, P.stride(0), out, B, T, pos0 + T,
                       pos0, Hq, Hkv, dh, True)
    # the unfused path on the same inputs
    qo = torch.empty((B * T, Hq, dh), dtype=torch.bfloat16, device=cuda)
    Kc2, Vc2 = Kc.clone(), Vc.clone()
    L.fa_prep(P, qn, kn, qo, Kc2, Vc2, cap, B, T, pos0, Hq, Hkv, dh, rot, base, eps)
    assert torch.equal(Kc, Kc2) and torch.equal(Vc, Vc2)          # the same K/V writes either way
    ref2 = torch.empty_like(out)
    L.gqa_attn(qo, Hq * dh, Kc2, Vc2, cap, gate_view, P.stride(0), ref2, B, T, pos0 + T, pos0, Hq, Hkv, dh, True)
    torch.cuda.synchronize()
    assert rel_l2(to64(out), to64(ref2)) < 4e-3
    Pn = to64(P).reshape(B, T, -1)
    for b in range(B):
        q, gate, k, v = ops.fa_split_projection(Pn[b], Hq, Hkv, dh)
        rq, rk = ops.fa_qk(q, k, to64(qn), to64(kn), pos0 + np.arange(T), rot, base, eps)
        K = np.concatenate([to64(Kc[b, :, :pos0]).transpose(1, 0, 2), rk]) if pos0 else rk
        V = np.concatenate([to64(Vc[b, :, :pos0]).transpose(1, 0, 2), v]) if pos0 else v
        ref = ops.attention(rq, K, V, pos0 + np.arange(T)) * ops.sigmoid(gate)
        assert rel_l2(to64(out.view(B, T, Hq, dh)[b]), ref) < TOL["bf16"]
    # the fused form exists for the tensor-core kernel only
    with pytest.raises(L.LoopError) as e:
        L.gqa_attn_fused_q(P, P.stride(0), qn, rot, base, eps, Kc, Vc, cap, gate_view, P.stride(0), out, B, 8,
                           pos0 + 8, pos0, Hq, Hkv, dh, True)
    assert e.value.status == 7


@pytest.mark.parametrize("dtype,dh,Hq,Hkv", [("fp32", 256, 16, 4), ("bf16", 256, 16, 4), ("bf16", 128, 8, 2),
                                              ("bf16", 64, 4, 1), ("bf16", 256, 6, 2)])
def test_decode_attention_split_k(cuda, dtype, dh, Hq, Hkv):
    """One query per sequence over a long slab: split-K partials + combine (with workspace) equal brute force."""
    import looped_hybrid_attention_b200 as L
    B, L_ctx = 4, 3000
    cap = L_ctx + 10
    q = rnd((B, Hq, dh), 30, "qd", dtype=dtype)
    Kc = rnd((B, Hkv, cap, dh), 31, "Kd", dtype=dtype)
    Vc = rnd((B, Hkv, cap, dh), 32, "Vd", dtype=dtype)
    gate = rnd((B, Hq * dh), 33, "gd", dtype=dtype)
    out = torch.empty((B, Hq * dh), dtype=DT[dtype], device=cuda)
    ws = torch.empty(L.gqa_workspace_bytes(B, 1, L_ctx, Hq, dh) // 4 + 1, device=cuda)
    for workspace in (ws, None):                    # split-K with combine, and a single pass
        L.gqa_attn(q, Hq * dh, Kc, Vc, cap, gate, Hq * dh, out, B, 1, L_ctx, L_ctx - 1, Hq, Hkv, dh, True, workspace)
        for b in range(B):
            ref = ops.attention(to64(q[b])[None], to64(Kc[b, :, :L_ctx]).transpose(1, 0, 2),
                                to64(Vc[b, :, :L_ctx]).transpose(1, 0, 2), [L_ctx - 1])
            ref = ref * ops.sigmoid(to64(gate[b]).reshape(1, Hq, dh))
            assert rel_l2(to64(out[b]).reshape(1, Hq, dh), ref) < TOL[dtype]


def test_attention_single_key_and_zero_query(cuda):
    import looped_hybrid_attention_b200 as L
    Hq, Hkv, dh, T = 4, 1, 64, 20
    Kc = rnd((1, Hkv, T, dh), 40, "K1")
    Vc = rnd((1, Hkv, T, dh), 41, "V1")
    q = torch.zeros((T, Hq, dh), device=cuda)
    out = torch.empty((T, Hq * dh), device=cuda)
    L.gqa_attn(q, Hq * dh, Kc, Vc, T, None, 0, out, 1, T, T, 0, Hq, Hkv, dh, True)
    mean = torch.cumsum(Vc[0, 0], 0) / torch.arange(1, T + 1, device=cuda)[:, None]
    assert torch.allclose(out.view(T, Hq, dh), mean[:, None, :].expand(T, Hq, dh), atol=1e-5)
    assert torch.allclose(out.view(T, Hq, dh)[0], Vc[0, 0, 0][None].expand(Hq, dh), atol=1e-6)


def test_attention_late_dominant_key_rescales_part_of_a_warp(cuda):
    """One key in the third 128-key tile is scaled up 12x, so the running row maximum of about
    a quarter of the query rows jumps by far more than the lazy-rescale threshold there while
    the other rows of the same warps keep theirs: O is rescaled for some rows of a warp only.
    Every row against brute force."""
    import looped_hybrid_attention_b200 as L
    T, Hq, Hkv, dh = 600, 16, 4, 256
    q = rnd((T, Hq, dh), 53, "qd", dtype="bf16")
    Kc = rnd((1, Hkv, T, dh), 54, "Kd")
    Kc[0, :, 300] *= 12.0
    Kc = Kc.to(torch.bfloat16)
    Vc = rnd((1, Hkv, T, dh), 55, "Vd", dtype="bf16")
    out = torch.empty((T, Hq * dh), dtype=torch.bfloat16, device=cuda)
    L.gqa_attn(q, Hq * dh, Kc, Vc, T, None, 0, out, 1, T, T, 0, Hq, Hkv, dh, True)
    torch.cuda.synchronize()
    # rows t >= 300 whose score at key 300 exceeds their maximum over keys 0..255 (the first
    # two tiles) by more than 8 in log2 units: those rescale O at the third tile
    qn, Kn = to64(q), to64(Kc[0])
    kv = np.arange(Hq) // (Hq // Hkv)
    s_late = np.einsum("thd,hd->th", qn[300:], Kn[kv, 300]) / 16.0
    s_early = np.einsum("thd,hkd->thk", qn[300:], Kn[kv, :256]) / 16.0
    jump = (s_late - s_early.max(axis=-1)) * np.log2(np.e)
    frac = float(np.mean(jump > 8.0))
    assert 0.05 < frac < 0.95, frac                  # some rows of a warp rescale, others do not
    ref = ops.attention(to64(q), to64(Kc[0]).transpose(1, 0, 2), to64(Vc[0]).transpose(1, 0, 2), np.arange(T))
    assert rel_l2(to64(out).reshape(T, Hq, dh), ref) < TOL["bf16"]
    assert L.device_error() == 0


@pytest.mark.slow
def test_attention_full_length_sampled_rows(cuda):
    """The bench's shape (T = 8192, 16q/4kv x 256, bf16): sampled query rows against brute force."""
    import looped_hybrid_attention_b200 as L
    T, Hq, Hkv, dh = 8192, 16, 4, 256
    q = rnd((T, Hq, dh), 50, "qf", dtype="bf16")
    Kc = rnd((1, Hkv, T, dh), 51, "Kf", dtype="bf16")
    Vc = rnd((1, Hkv, T, dh), 52, "Vf", dtype="bf16")
    out = torch.empty((T, Hq * dh), dtype=torch.bfloat16, device=cuda)
    L.gqa_attn(q, Hq * dh, Kc, Vc, T, None, 0, out, 1, T, T, 0, Hq, Hkv, dh, True)
    rows = np.array([0, 1, 63, 64, 127, 128, 4095, 5000, 8190, 8191])
    ref = ops.attention(to64(q[rows]), to64(Kc[0]).transpose(1, 0, 2), to64(Vc[0]).transpose(1, 0, 2), rows)
    assert rel_l2(to64(out[rows]).reshape(len(rows), Hq, dh), ref) < TOL["bf16"]



@pytest.mark.slow
def test_attention_long_context_sampled_rows(cuda):
    """The long-context prefill shape (T = 131,072, 16q/4kv x 256, bf16, gate fused): sampled
    query rows, including the last, against brute-force softmax over their causal prefix."""
    import looped_hybrid_attention_b200 as L
    T, Hq, Hkv, dh = 131072, 16, 4, 256
    gen = torch.Generator(device=cuda).manual_seed(53)
    q = torch.randn((T, Hq, dh), device=cuda, generator=gen).to(torch.bfloat16)
    Kc = torch.randn((1, Hkv, T, dh), device=cuda, generator=gen).to(torch.bfloat16)
    Vc = torch.randn((1, Hkv, T, dh), device=cuda, generator=gen).to(torch.bfloat16)
    gate = torch.randn((T, Hq * dh), device=cuda, generator=gen).to(torch.bfloat16)
    out = torch.empty((T, Hq * dh), dtype=torch.bfloat16, device=cuda)
    L.gqa_attn(q, Hq * dh, Kc, Vc, T, gate, Hq * dh, out, 1, T, T, 0, Hq, Hkv, dh, True)
    torch.cuda.synchronize()
    assert L.device_error() == 0
    rows = np.array([0, 63, 64, 65535, 65536, 100000, 131007, 131008, 131070, 131071])
    ref = ops.attention(to64(q[rows]), to64(Kc[0]).transpose(1, 0, 2), to64(Vc[0]).transpose(1, 0, 2), rows)
    ref = ref * ops.sigmoid(to64(gate[rows]).reshape(len(rows), Hq, dh))
    assert rel_l2(to64(out[rows]).reshape(len(rows), Hq, dh), ref) < TOL["bf16"]


# the projections of the 9B-shape prefill at T = 8192: (N, K, epilogue)
FULL_GEMMS = [(6176, 4096, "store"), (2048 * 2, 2048, "store"), (10240, 4096, "store"), (4096, 4096, "store"),
              (12288, 4096, "swiglu"), (4096, 12288, "add")]


@pytest.mark.slow
@pytest.mark.parametrize("N,K,epi", FULL_GEMMS)
def test_linear_full_size_sampled_rows(cuda, N, K, epi):
    """bf16 projections at M = 8192 (the prefill bench's token count): sampled rows vs fp64."""
    import looped_hybrid_attention_b200 as L
    M = 8192
    X = torch.randn((M, K), device=cuda, generator=torch.Generator(device=cuda).manual_seed(1)).to(torch.bfloat16)
    W = (0.02 * torch.randn((N, K), device=cuda, generator=torch.Generator(device=cuda).manual_seed(2))).to(torch.bfloat16)
    Y = torch.empty((M, N), dtype=torch.bfloat16, device=cuda)
    rows = np.array([0, 1, 127, 128, 129, 4000, 8063, 8064, 8190, 8191])
    xr = to64(X[rows])
    if epi == "swiglu":
        W2 = (0.02 * torch.randn((N, K), device=cuda, generator=torch.Generator(device=cuda).manual_seed(3))).to(torch.bfloat16)
        L.linear(X, W, Y, L.EPI_SWIGLU, W2=W2)
        ref = ops.silu(ops.linear(xr, to64(W))) * ops.linear(xr, to64(W2))
    elif epi == "add":
        R = torch.randn((M, N), device=cuda, generator=torch.Generator(device=cuda).manual_seed(4)).to(torch.bfloat16)
        L.linear(X, W, Y, L.EPI_ADD, R=R)
        ref = ops.linear(xr, to64(W)) + to64(R[rows])
    else:
        L.linear(X, W, Y, L.EPI_STORE)
        ref = ops.linear(xr, to64(W))
    torch.cuda.synchronize()
    assert L.device_error() == 0
    assert rel_l2(to64(Y[rows]), ref) < TOL["bf16"]
    # every row is written (no tile skipped): compare row norms against a cheap fp32 reference
    if epi == "store":
        ref_all = (X.float() @ W.float().t())
        assert rel_l2(to64(Y), to64(ref_all)) < TOL["bf16"]


def test_lm_head_shape_fp32_out(cuda):
    """M = 1..64 rows (prefill last position / decode batch) against the 248,320-row LM head, fp32 logits."""
    import looped_hybrid_attention_b200 as L
    V, d = 248320, 4096
    W = (0.02 * torch.randn((V, d), device=cuda, generator=torch.Generator(device=cuda).manual_seed(5))).to(torch.bfloat16)
    for M in (1, 64):
        X = torch.randn((M, d), device=cuda, generator=torch.Generator(device=cuda).manual_seed(6)).to(torch.bfloat16)
        Y = torch.empty((M, V), device=cuda)
        L.linear(X, W, Y, L.EPI_F32)
        cols = np.r_[0:64, 124000:124100, V - 70:V]
        ref = ops.linear(to64(X), to64(W[cols]))
        assert rel_l2(to64(Y[:, cols]), ref) < 1e-4
