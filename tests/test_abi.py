"""The C-ABI library loads, exports every declared symbol, and its host-side logic matches the oracle (no GPU)."""
import ctypes

import pytest

import synth
from oracle import schedule as osched

L = pytest.importorskip("looped_hybrid_attention_b200")


def test_every_declared_function_is_exported():
    names = L.header_functions()
    assert len(names) >= 25
    for n in names:
        assert hasattr(L._lib, n), f"{n} declared in include/loop.h but not exported"
    for required in ("loop_model_create", "loop_prefill", "loop_decode_step", "gdn_chunk_fwd", "gdn_step",
                     "gqa_attn", "mhc_route_mix", "sinkhorn_fp32"):
        assert required in names


@pytest.mark.parametrize("shape", [synth.FULL, synth.TINY, synth.GROUP, synth.FULL.with_(loop_passes=3),
                                   synth.FULL.with_(loop_passes=1), synth.TINY.with_(loop_passes=0)])
def test_schedule_and_slots_bit_exact_vs_oracle(shape):
    lib = L.schedule(shape)
    ora = [(e, l, 1 if k == "fa" else 0, slot, int(il)) for e, l, k, slot, il in osched.table(shape)]
    assert lib == ora


def test_schedule_counts_full():
    cfg = L.make_config(synth.FULL)
    n, fa, gdn = ctypes.c_int(), ctypes.c_int(), ctypes.c_int()
    L.check(L._lib.loop_schedule(ctypes.byref(cfg), None, 0, ctypes.byref(n), ctypes.byref(fa), ctypes.byref(gdn)))
    assert (n.value, fa.value, gdn.value) == (56, 14, 42)
    buf = (ctypes.c_int32 * 10)()
    assert L._lib.loop_schedule(ctypes.byref(cfg), buf, 2, ctypes.byref(n), None, None) == 5   # CAPACITY


def _fake_weights(shape):
    """Non-null fake addresses: model creation only validates and copies pointers (no device access)."""
    fake = {}
    for i, (name, _, _) in enumerate(synth.weight_names(shape)):
        class T:
            def __init__(self, a):
                self.a = a

            def data_ptr(self):
                return self.a
        fake[name] = T(0x10000 + 256 * i)
    return fake


def test_model_create_validates_without_gpu():
    m = L.Model(synth.TINY, _fake_weights(synth.TINY))
    m.close()
    bad = _fake_weights(synth.TINY)
    del bad["layers.5.mhc_w_r"]
    with pytest.raises(L.LoopError) as e:
        L.Model(synth.TINY, bad)
    assert e.value.status == 1 and "layer 5" in str(e.value)
    with pytest.raises(L.LoopError) as e:
        L.Model(synth.TINY.with_(gdn_dk=96, gdn_dv=96), _fake_weights(synth.TINY))
    assert e.value.status == 7
    with pytest.raises(L.LoopError) as e:
        L.Model(synth.TINY.with_(mhc_streams=4), _fake_weights(synth.TINY))
    assert e.value.status == 7
    with pytest.raises(L.LoopError) as e:
        L.Model(synth.TINY.with_(loop_end=20), _fake_weights(synth.TINY))
    assert e.value.status == 1


def test_per_op_argument_errors_without_gpu():
    P = ctypes.c_void_p(0x1000)
    # unsupported head size -> UNSUPPORTED, nothing launched
    st = L._lib.gdn_chunk_fwd(P, P, P, P, P, P, P, 1, 64, 2, 96, 96, 64, 1.0, None, 1, None)
    assert st == 7
    st = L._lib.gdn_chunk_fwd(P, P, P, P, P, P, P, 1, 64, 2, 128, 128, 32, 1.0, None, 1, None)
    assert st == 7 and "chunk" in L.last_error()
    st = L._lib.gqa_attn(P, 4096, P, P, 10, None, 0, P, 1, 20, 10, 0, 16, 4, 256, 1, None, 1, None)
    assert st == 2                                       # kv_cap < Tkv ... causal overrun -> SHAPE
    st = L._lib.sinkhorn_fp32(P, P, 4, 9, 20, None)
    assert st == 1
    st = L._lib.mhc_route_mix(1, P, None, None, P, P, P, P, None, P, 4, 256, 1e-6, 20, 1, None)
    assert st == 1 and "F" in L.last_error()
    st = L._lib.fa_prep(P, 10240, P, P, P, P, P, 100, 1, 64, 50, 16, 4, 256, 64, 1e4, 1e-6, 1, None)
    assert st == 5                                       # positions past the slab -> CAPACITY
    st = L._lib.loop_linear(P, 100, P, None, None, 0, P, 64, 4, 64, 100, 0, None, 1, None)
    assert st == 2                                       # bf16 needs K % 8 == 0


def test_newer_entry_points_argument_errors_without_gpu():
    """Argument checks of the taps, the GDN variant ops, the fused GDN input projection and the
    fused-query attention: each bad call returns its status before anything is launched."""
    P = ctypes.c_void_p(0x1000)
    # gdn_conv_prep: conv taps other than 4, value heads not a multiple of key heads -> UNSUPPORTED;
    # a projection row narrower than q|k|v|z|a|b -> SHAPE; an empty batch is a no-op
    args = lambda ld, Hk, Hv, conv: (P, ld, P, P, P, P, P, P, P, P, P, 2, 5, Hk, Hv, 128, 128, conv, 1e-6, 1, None)
    width = 2 * 2 * 128 + 2 * 4 * 128 + 2 * 4
    assert L._lib.gdn_conv_prep(*args(width, 2, 4, 3)) == 7
    assert L._lib.gdn_conv_prep(*args(width, 3, 4, 4)) == 7
    assert L._lib.gdn_conv_prep(*args(width - 1, 2, 4, 4)) == 2
    assert L._lib.gdn_conv_prep(P, width, P, P, P, P, P, P, P, P, P, 0, 5, 2, 4, 128, 128, 4, 1e-6, 1, None) == 0
    # gdn_gated_norm: dv not a multiple of 32 -> UNSUPPORTED; z rows narrower than H*dv -> SHAPE
    assert L._lib.gdn_gated_norm(P, P, 4 * 48, P, P, 10, 4, 48, 1e-6, 1, None) == 7
    assert L._lib.gdn_gated_norm(P, P, 4 * 128 - 1, P, P, 10, 4, 128, 1e-6, 1, None) == 2
    assert L._lib.gdn_gated_norm(None, None, 0, None, None, 0, 4, 128, 1e-6, 1, None) == 0
    # gdn_in_proj: built for bf16 batches of more than 128 rows with 128-dim heads
    proj = lambda M, ldx, H, dt: (P, ldx, P, P, P, P, P, P, P, P, M, 4096, H, 128, 128, 1e-6, dt, None)
    assert L._lib.gdn_in_proj(*proj(128, 4096, 16, 1)) == 7
    assert L._lib.gdn_in_proj(*proj(8192, 4096, 16, 0)) == 7
    assert L._lib.gdn_in_proj(*proj(8192, 4096, 15, 1)) == 7
    assert L._lib.gdn_in_proj(*proj(8192, 4000, 16, 1)) == 2
    # the bounded-wait self-test refuses a cycle limit outside (0, 4e9] before launching
    assert L._lib.loop_wait_selftest(0, None) == 1
    assert L._lib.loop_wait_selftest(5_000_000_000, None) == 1
    # gqa_attn_fused_q: the query norm gain is required; rotary dims even and at most dh / 2
    fq = lambda qn, rot: (P, 4096, qn, rot, 1e4, 1e-6, P, P, 64, P, 4096, P, 1, 64, 64, 0, 16, 4, 256, 1, 1, None)
    assert L._lib.gqa_attn_fused_q(*fq(None, 64)) == 1
    assert L._lib.gqa_attn_fused_q(*fq(P, 63)) == 1
    assert L._lib.gqa_attn_fused_q(*fq(P, 130)) == 1


def test_set_taps_validation_without_gpu():
    """Tap executions must lie in [0, executions) and be distinct; n = 0 clears the taps."""
    m = L.Model(synth.TINY, _fake_weights(synth.TINY))
    try:
        n_exec = len(L.schedule(synth.TINY))
        ex = lambda *e: (ctypes.c_int32 * len(e))(*e)
        ps = lambda n: (ctypes.c_void_p * n)(*([0x2000] * n))
        assert L._lib.loop_set_taps(m.handle, 2, ex(3, n_exec - 1), ps(2), 64) == 0
        assert L._lib.loop_set_taps(m.handle, 1, ex(n_exec), ps(1), 64) == 1
        assert "outside" in L.last_error()
        assert L._lib.loop_set_taps(m.handle, 2, ex(3, 3), ps(2), 64) == 1
        assert "twice" in L.last_error()
        assert L._lib.loop_set_taps(m.handle, 1, ex(3), (ctypes.c_void_p * 1)(None), 64) == 1
        assert L._lib.loop_set_taps(m.handle, 1, ex(3), ps(1), -1) == 1
        assert L._lib.loop_set_taps(m.handle, 0, None, None, 0) == 0
    finally:
        m.close()
