"""Pins of the oracle's whole-model forward: B(B(h)) weight sharing, mHC special case, cache semantics, causality."""
import numpy as np
import pytest
import torch

import synth
from oracle import model, ops, schedule

# a tiny shape with an embedding and LM head, for prefill/decode tests
TINY_LM = synth.TINY.with_(with_embedding=True, vocab=97)


@pytest.fixture(scope="module")
def tiny_w():
    return model.Weights(synth.make_weights(synth.TINY, seed=0))


@pytest.fixture(scope="module")
def tiny_lm_w():
    return model.Weights(synth.make_weights(TINY_LM, seed=3))


def test_looped_equals_unrolled_stack_with_copied_weights():
    """B(B(h)): the looped forward equals an unrolled stack whose layers are explicit weight copies."""
    s = synth.TINY
    w = synth.make_weights(s, seed=1)
    layers = schedule.execution_layers(s.n_layers, s.loop_start, s.loop_end, s.loop_passes)
    n = len(layers)
    unrolled = s.with_(n_layers=n, loop_start=s.loop_start, loop_end=s.loop_start + (s.loop_end - s.loop_start) * s.loop_passes,
                       loop_passes=1)
    wu = {}
    for e, l in enumerate(layers):
        for k, t in w.items():
            if k.startswith(f"layers.{l}."):
                wu[k.replace(f"layers.{l}.", f"layers.{e}.", 1)] = t.clone()
    # kinds line up because the loop block is whole groups
    assert [schedule.layer_kind(e, s.group) for e in range(n)] == [schedule.layer_kind(l, s.group) for l in layers]
    h = synth.normal((1, 40, s.d), 1.0, 0, "h")
    a, _ = model.forward_hidden(s, model.Weights(w), h)
    b, _ = model.forward_hidden(unrolled, model.Weights(wu), h)
    assert np.array_equal(a, b)
    # a second pass is not a no-op: one pass gives a different result
    c, _ = model.forward_hidden(s.with_(loop_passes=1), model.Weights(w), h)
    assert not np.allclose(a, c, atol=1e-3)


def test_zero_routing_mhc_equals_plain_residual_stack():
    """W_r = 0, b_r = 0: H_pre = (1/2,1/2), H_post = (1,1), H_res = 1/2 -> streams stay equal -> plain residual."""
    s = synth.TINY
    w = synth.make_weights(s, seed=2)
    for k in list(w):
        if "mhc_" in k:
            w[k] = torch.zeros_like(w[k])
    W = model.Weights(w)
    h = synth.normal((1, 24, s.d), 1.0, 0, "h2")
    out, _ = model.forward_hidden(s, W, h)
    hp = ops.f64(h[0])
    cache = model.new_cache()
    for e, l, kind, slot, _ in schedule.table(s):
        hp = hp + model.layer_branch(s, W, l, kind, slot, hp, cache, 0)
    assert np.allclose(out[0], hp, rtol=1e-12, atol=1e-12)


def test_decode_after_prefill_equals_longer_prefill(tiny_lm_w):
    s = TINY_LM
    ids = synth.uniform_ids((2, 19), s.vocab, 0)
    logits_T, caches = model.prefill(s, tiny_lm_w, ids[:, :18].numpy())
    l1, nxt = model.decode_step(s, tiny_lm_w, caches, ids[:, 18].numpy())
    l2, _ = model.prefill(s, tiny_lm_w, ids.numpy())
    assert np.allclose(l1, l2, rtol=1e-10, atol=1e-10)
    assert np.array_equal(nxt, np.argmax(l2, axis=-1))
    assert all(c["len"] == 19 for c in caches)
    # each FA execution cached its own K/V for all 19 tokens; GDN states are constant-size
    assert all(caches[0]["kv"][slot][0].shape == (19, s.fa_kv_heads, s.fa_head_dim) for slot in range(4))
    assert all(caches[0]["state"][slot].shape == (s.gdn_heads, s.gdn_dv, s.gdn_dk) for slot in range(12))


def test_causality(tiny_w):
    s = synth.TINY
    h = synth.normal((1, 30, s.d), 1.0, 0, "h3").numpy()
    h2 = h.copy()
    h2[0, 20:] = np.random.default_rng(0).normal(size=(10, s.d))
    a, _ = model.forward_hidden(s, tiny_w, h)
    b, _ = model.forward_hidden(s, tiny_w, h2)
    assert np.allclose(a[0, :20], b[0, :20], atol=1e-12)
    assert not np.allclose(a[0, 20:], b[0, 20:], atol=1e-3)


def test_segmented_prefill_equals_one_shot(tiny_w):
    """Prefill in two segments (state and KV carried over) equals one pass over the whole sequence."""
    s = synth.TINY
    h = synth.normal((1, 50, s.d), 1.0, 0, "h4").numpy()
    full, _ = model.forward_hidden(s, tiny_w, h)
    caches = [model.new_cache()]
    a, caches = model.forward_hidden(s, tiny_w, h[:, :33], caches)
    b, caches = model.forward_hidden(s, tiny_w, h[:, 33:], caches)
    assert np.allclose(np.concatenate([a, b], axis=1), full, rtol=1e-10, atol=1e-10)


def test_taps_cover_every_execution(tiny_w):
    s = synth.TINY
    taps = []
    out, _ = model.forward_hidden(s, tiny_w, synth.normal((1, 8, s.d), 1.0, 0, "h5"), taps=taps)
    assert len(taps) == schedule.counts(s)[0]
    assert np.allclose(taps[-1], out[0])
