"""The Gated-DeltaNet variant on the GPU ("原地套圈" investigation §01: backbone qwen3_5_text):
causal conv + SiLU on q|k|v with the conv inputs carried in the cache, value heads sharing key
heads, gated output norm -- per op and for whole stacks, against the oracle."""
import numpy as np
import pytest
import torch

import synth
from conftest import TOL, rel_l2, to64
from oracle import model as omodel
from oracle import ops

pytestmark = pytest.mark.gpu

DT = {"fp32": torch.float32, "bf16": torch.bfloat16}


def rnd(shape, seed, name, std=1.0, dtype="fp32"):
    return synth.normal(shape, std, seed, name).to(DT[dtype]).cuda()


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("B,T,Hk,Hv,dk", [(2, 70, 2, 4, 128), (1, 1, 2, 4, 128), (3, 2, 1, 2, 64), (1, 5, 4, 4, 64)])
def test_gdn_conv_prep_vs_oracle(cuda, dtype, B, T, Hk, Hv, dk):
    import looped_hybrid_attention_b200 as L
    dv, K, eps = dk, 4, 1e-6
    C = 2 * Hk * dk + Hv * dv
    n_in = C + Hv * dv + 2 * Hv
    P = rnd((B * T, n_in), 1, "Pv", dtype=dtype)
    conv_w = rnd((C, K), 2, "cw", std=0.5, dtype=dtype)
    state = rnd((B, K - 1, C), 3, "cs", dtype=dtype)
    state0 = state.clone()
    ab, bb = rnd((Hv,), 4, "ab"), rnd((Hv,), 5, "bb")
    q = torch.empty((B * T, Hv, dk), dtype=DT[dtype], device=cuda)
    k, v = torch.empty_like(q), torch.empty((B * T, Hv, dv), dtype=DT[dtype], device=cuda)
    g, beta = torch.empty((B * T, Hv), device=cuda), torch.empty((B * T, Hv), device=cuda)
    L.gdn_conv_prep(P, conv_w, state, ab, bb, q, k, v, g, beta, B, T, Hk, Hv, dk, dv, eps)
    torch.cuda.synchronize()
    tol = TOL[dtype]
    Pn = to64(P).reshape(B, T, n_in)
    rep = Hv // Hk
    for b in range(B):
        y, st = ops.causal_conv_silu(Pn[b, :, :C], to64(conv_w), to64(state0[b]))
        rq = np.repeat(ops.l2norm(y[:, :Hk * dk].reshape(T, Hk, dk), eps), rep, axis=1)
        rk = np.repeat(ops.l2norm(y[:, Hk * dk:2 * Hk * dk].reshape(T, Hk, dk), eps), rep, axis=1)
        rv = y[:, 2 * Hk * dk:].reshape(T, Hv, dv)
        sl = slice(b * T, (b + 1) * T)
        assert rel_l2(to64(q[sl]), rq) < tol and rel_l2(to64(k[sl]), rk) < tol and rel_l2(to64(v[sl]), rv) < tol
        _, _, _, _, a, bvec = ops.gdn_split_projection_v2(Pn[b], Hk, Hv, dk, dv)
        rg, rb = ops.gdn_gates(a, bvec, to64(ab), to64(bb))
        assert rel_l2(to64(g[sl]), rg) < 1e-5 and rel_l2(to64(beta[sl]), rb) < 1e-5
        assert np.array_equal(to64(state[b]), st)            # the last K-1 inputs, copied exactly


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("H,dv", [(4, 128), (3, 64)])
def test_gdn_gated_norm_vs_oracle(cuda, dtype, H, dv):
    import looped_hybrid_attention_b200 as L
    M, eps = 37, 1e-6
    o = rnd((M, H, dv), 6, "o", dtype=dtype)
    zrow = rnd((M, 2 * H * dv), 7, "z", dtype=dtype)           # z is a block inside wider rows
    w = rnd((dv,), 8, "w", std=0.2, dtype=dtype) + 1
    y = torch.empty_like(o)
    L.gdn_gated_norm(o, zrow[:, H * dv:], zrow.stride(0), w, y, M, H, dv, eps)
    ref = ops.gated_rmsnorm(to64(o), to64(zrow[:, H * dv:]).reshape(M, H, dv), to64(w), eps)
    assert rel_l2(to64(y), ref) < TOL[dtype]
    L.gdn_gated_norm(o, zrow[:, H * dv:], zrow.stride(0), w, o, M, H, dv, eps)    # in place
    assert torch.equal(o, y)


def dev_weights(w):
    return {k: v.cuda() for k, v in w.items()}


VARIANT_TINY = synth.TINY.with_(gdn_variant=1, gdn_v_heads=8, with_embedding=True, vocab=500)


def test_variant_tiny_stack_prefill_decode_fp32(cuda):
    """Tiny stack with the variant (4 key / 8 value heads x 64), fp32: two prefill segments (the
    second shorter than the conv kernel), then three decode steps, against the oracle at 1e-5;
    every GDN state and conv-input slot against the oracle's cache."""
    import looped_hybrid_attention_b200 as L
    s = VARIANT_TINY
    w = synth.make_weights(s, seed=11)
    W = omodel.Weights(w)
    B, T1, T2 = 2, 60, 2
    ids = synth.uniform_ids((B, T1 + T2 + 3), s.vocab, 11)
    ref, caches = omodel.prefill(s, W, ids[:, :T1 + T2].numpy())
    m = L.Model(s, dev_weights(w))
    c = m.cache(B, 80)
    lg = torch.empty((B, s.vocab), device=cuda)
    m.prefill(c, ids[:, :T1].contiguous().cuda(), lg)
    m.prefill(c, ids[:, T1:T1 + T2].contiguous().cuda(), lg)
    torch.cuda.synchronize()
    assert rel_l2(to64(lg), ref) < TOL["fp32"]
    nxt = torch.empty(B, dtype=torch.int32, device=cuda)
    for t in range(T1 + T2, T1 + T2 + 3):
        tok = ids[:, t].contiguous()
        ref_l, ref_n = omodel.decode_step(s, W, caches, tok.numpy())
        m.decode_step(c, tok.cuda(), lg, nxt)
        torch.cuda.synchronize()
        assert rel_l2(to64(lg), ref_l) < TOL["fp32"]
    Hv, C = s.gdn_v_heads, 2 * s.gdn_heads * s.gdn_dk + s.gdn_v_heads * s.gdn_dv
    _, state_bytes = c.nbytes()
    n_gdn = 12
    assert state_bytes == n_gdn * (B * Hv * s.gdn_dv * s.gdn_dk * 4 + B * 3 * C * 4)
    for slot in range(n_gdn):
        st = L.device_view(c.state_ptr(slot), (B, Hv, s.gdn_dv, s.gdn_dk), torch.float32)
        for b in range(B):
            assert rel_l2(to64(st[b]), caches[b]["state"][slot]) < 1e-4, slot


def test_variant_narrow_bf16_stack(cuda):
    """A narrow bf16 stack with the full-size head shapes (2 key / 4 value heads x 128, FA head 256):
    prefill of 160 tokens (tensor-core GEMMs, two-pass scan on 4 value heads) and a decode step."""
    import looped_hybrid_attention_b200 as L
    s = synth.ModelShape(d=512, ffn=1024, vocab=2048, n_layers=4, loop_start=0, loop_end=4, loop_passes=1,
                         gdn_heads=2, gdn_v_heads=4, gdn_variant=1, fa_q_heads=4, fa_kv_heads=1, dtype="bf16",
                         with_embedding=True)
    T = 160
    w = synth.make_weights(s, seed=12)
    ids = synth.uniform_ids((1, T + 1), s.vocab, 12)
    W = omodel.Weights(w)
    ref, caches = omodel.prefill(s, W, ids[:, :T].numpy())
    ref_step, _ = omodel.decode_step(s, W, caches, ids[:, T].numpy())
    m = L.Model(s, dev_weights(w))
    c = m.cache(1, T + 8)
    lg = torch.empty((1, s.vocab), device=cuda)
    m.prefill(c, ids[:, :T].contiguous().cuda(), lg)
    torch.cuda.synchronize()
    assert rel_l2(to64(lg), ref) < TOL["bf16_e2e"]
    nxt = torch.empty(1, dtype=torch.int32, device=cuda)
    m.decode_step(c, ids[:, T].contiguous().cuda(), lg, nxt)
    torch.cuda.synchronize()
    assert rel_l2(to64(lg), ref_step) < TOL["bf16_e2e"]
    assert L.device_error() == 0
