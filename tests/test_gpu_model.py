"""Model-level parity: the looped stack through loop_forward_hidden / loop_prefill / loop_decode_step vs the oracle."""
import numpy as np
import pytest
import torch

import synth
from conftest import TOL, rel_l2, to64
from oracle import model as omodel
from oracle import schedule as osched

pytestmark = pytest.mark.gpu

TINY_LM = synth.TINY.with_(with_embedding=True, vocab=1000)


def dev_weights(w):
    return {k: v.cuda() for k, v in w.items()}


def test_tiny_stack_fp32_vs_oracle(cuda):
    """Tiny looped stack (12 stored layers, 16 executions, fp32), batch 1, seq 256, inputs N(0,1)."""
    import looped_hybrid_attention_b200 as L
    s = synth.TINY
    w = synth.make_weights(s, seed=0)
    h = synth.normal((1, 256, s.d), 1.0, 0, "hidden")
    ref, caches = omodel.forward_hidden(s, omodel.Weights(w), h)
    m = L.Model(s, dev_weights(w))
    c = m.cache(1, 256)
    out = torch.empty((1, 256, s.d), device=cuda)
    m.forward_hidden(c, h.cuda(), out)
    torch.cuda.synchronize()
    assert rel_l2(to64(out), ref) < TOL["fp32"]
    assert c.length == 256
    # per-execution GDN states: every slot holds what the oracle's execution of that slot left
    for slot in range(12):
        st = L.device_view(c.state_ptr(slot), (1, s.gdn_heads, s.gdn_dv, s.gdn_dk), torch.float32)
        assert rel_l2(to64(st[0]), caches[0]["state"][slot]) < 1e-4


def test_tiny_kv_slabs_per_execution(cuda):
    """Slot s of the cache holds the normed+rotated keys of FA execution s (bit-exact slot indexing)."""
    import looped_hybrid_attention_b200 as L
    s = synth.TINY
    w = synth.make_weights(s, seed=1)
    T = 50
    h = synth.normal((1, T, s.d), 1.0, 1, "hidden")
    _, caches = omodel.forward_hidden(s, omodel.Weights(w), h)
    m = L.Model(s, dev_weights(w))
    c = m.cache(1, 64)
    out = torch.empty((1, T, s.d), device=cuda)
    m.forward_hidden(c, h.cuda(), out)
    torch.cuda.synchronize()
    n_fa = osched.counts(s)[1]
    errs = np.zeros((n_fa, n_fa))
    for slot in range(n_fa):
        kp, vp = c.kv_ptrs(slot)
        K = L.device_view(kp, (1, s.fa_kv_heads, 64, s.fa_head_dim), torch.float32)
        got = to64(K[0, :, :T]).transpose(1, 0, 2)
        for o in range(n_fa):
            errs[slot, o] = rel_l2(got, caches[0]["kv"][o][0])
    # the diagonal matches, every other pairing does not
    assert np.all(np.diag(errs) < 1e-5)
    assert np.all(errs[~np.eye(n_fa, dtype=bool)] > 1e-2)


def test_tiny_prefill_decode_fp32_vs_oracle(cuda):
    import looped_hybrid_attention_b200 as L
    s = TINY_LM
    w = synth.make_weights(s, seed=3)
    W = omodel.Weights(w)
    B, T = 2, 40
    ids = synth.uniform_ids((B, T + 3), s.vocab, 3)
    ref_logits, caches = omodel.prefill(s, W, ids[:, :T].numpy())
    m = L.Model(s, dev_weights(w))
    c = m.cache(B, 64)
    lg = torch.empty((B, s.vocab), device=cuda)
    m.prefill(c, ids[:, :T].contiguous().cuda(), lg)
    torch.cuda.synchronize()
    assert rel_l2(to64(lg), ref_logits) < TOL["fp32"]
    nxt = torch.empty(B, dtype=torch.int32, device=cuda)
    for t in range(T, T + 3):
        tok = ids[:, t].contiguous()
        ref_l, ref_n = omodel.decode_step(s, W, caches, tok.numpy())
        m.decode_step(c, tok.cuda(), lg, nxt)
        torch.cuda.synchronize()
        assert rel_l2(to64(lg), ref_l) < TOL["fp32"]
        srt = np.sort(ref_l, axis=1)
        clear = (srt[:, -1] - srt[:, -2]) > 1e-3 * np.abs(srt[:, -1])
        assert np.array_equal(nxt.cpu().numpy()[clear], ref_n[clear])
    assert c.length == T + 3


def test_tiny_segmented_prefill(cuda):
    """Two prefill segments (GDN states and KV carried in the cache) equal the oracle's one-shot prefill."""
    import looped_hybrid_attention_b200 as L
    s = TINY_LM
    w = synth.make_weights(s, seed=4)
    ids = synth.uniform_ids((1, 150), s.vocab, 4)
    ref, _ = omodel.prefill(s, omodel.Weights(w), ids.numpy())
    m = L.Model(s, dev_weights(w))
    c = m.cache(1, 160)
    lg = torch.empty((1, s.vocab), device=cuda)
    m.prefill(c, ids[:, :97].contiguous().cuda(), lg)
    m.prefill(c, ids[:, 97:].contiguous().cuda(), lg)
    torch.cuda.synchronize()
    assert rel_l2(to64(lg), ref) < TOL["fp32"]
    with pytest.raises(L.LoopError) as e:
        m.prefill(c, ids[:, :20].contiguous().cuda(), lg)      # 150 + 20 > 160
    assert e.value.status == 5


def test_group_bf16_vs_oracle(cuda):
    """One full-width group (3 GDN 16x128 + 1 GQA 16q/4kv x 256, d 4096, FFN 12288, mHC), bf16, ragged T."""
    import looped_hybrid_attention_b200 as L
    s = synth.GROUP
    T = 300
    w = synth.make_weights(s, seed=0)
    h = synth.normal((1, T, s.d), 1.0, 0, "hidden").to(torch.bfloat16)
    ref, _ = omodel.forward_hidden(s, omodel.Weights(w), h)
    m = L.Model(s, dev_weights(w))
    c = m.cache(1, T)
    out = torch.empty((1, T, s.d), dtype=torch.bfloat16, device=cuda)
    m.forward_hidden(c, h.cuda(), out)
    torch.cuda.synchronize()
    assert rel_l2(to64(out), ref) < TOL["bf16_e2e"]


def test_tiny_stack_long_sequence_fp32(cuda):
    """1100 tokens: the prefill-sized mHC path (4 tokens per warp, transposed routing maps) and many GDN chunks."""
    import looped_hybrid_attention_b200 as L
    s = synth.TINY
    w = synth.make_weights(s, seed=5)
    T = 1100
    h = synth.normal((1, T, s.d), 1.0, 5, "hidden")
    ref, _ = omodel.forward_hidden(s, omodel.Weights(w), h)
    m = L.Model(s, dev_weights(w))
    c = m.cache(1, T)
    out = torch.empty((1, T, s.d), device=cuda)
    m.forward_hidden(c, h.cuda(), out)
    torch.cuda.synchronize()
    assert rel_l2(to64(out), ref) < TOL["fp32"]


@pytest.mark.slow
def test_full_stack_long_context_prefix(cuda):
    """The full 9B-shape stack (56 executions, bf16) over a 131,072-token input in one call.

    The stack is causal and every kernel's arithmetic for a row depends only on that row's
    prefix (fixed chunk and tile boundaries), so the first 8,192 output rows must equal,
    bit for bit, a separate 8,192-token call; the KV slab of every full-attention execution
    holds 131,072 written positions, and every output is finite."""
    import looped_hybrid_attention_b200 as L
    s = synth.FULL
    T, T0 = 131072, 8192
    w = synth.make_weights(s, seed=0, device=cuda)
    gen = torch.Generator(device=cuda).manual_seed(9)
    h = torch.randn((1, T, s.d), device=cuda, generator=gen).to(torch.bfloat16)
    m = L.Model(s, w)
    c = m.cache(1, T)
    out = torch.empty_like(h)
    m.forward_hidden(c, h, out)
    torch.cuda.synchronize()
    assert L.device_error() == 0
    assert c.length == T
    assert bool(torch.isfinite(out).all())
    kv_bytes, _ = c.nbytes()
    assert kv_bytes == 14 * 4096 * T            # 4 KB per token per full-attention execution
    last_k = L.device_view(c.kv_ptrs(13)[0], (1, s.fa_kv_heads, T, s.fa_head_dim), torch.bfloat16)
    assert bool((last_k[0, :, -1].abs().sum(dim=-1) > 0).all())   # the last position was written
    del c
    c0 = m.cache(1, T0)
    out0 = torch.empty((1, T0, s.d), dtype=torch.bfloat16, device=cuda)
    m.forward_hidden(c0, h[:, :T0].contiguous(), out0)
    torch.cuda.synchronize()
    assert torch.equal(out[:, :T0], out0)
