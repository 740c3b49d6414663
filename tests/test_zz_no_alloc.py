"""gqa_attn_noalloc: the attention entry point that allocates no device memory.

It is meant for callers that cannot allocate a workspace (a runtime that has given all
free device memory to its own pool, or a loop that must not take the synchronisation of
cudaMalloc / cudaFree).  Its split-K scratch is a fixed array inside the library.  It
runs the same kernels with the same split plan as gqa_attn given a workspace, so its
result must equal that entry point's bit for bit, call after call, and it must leave the
device's free memory unchanged.  This file is collected last so that a failure here
comes after every other test has run.
"""
import numpy as np
import pytest
import torch

import synth
from conftest import TOL, rel_l2, to64
from oracle import ops

pytestmark = pytest.mark.gpu


def _decode_case(B, Hq, Hkv, dh, cap, seed):
    g = lambda shape, name: synth.normal(shape, 1.0, seed, name).to(torch.bfloat16).cuda()
    return g((B, Hq, dh), "q"), g((B, Hkv, cap, dh), "K"), g((B, Hkv, cap, dh), "V"), g((B, Hq * dh), "gate")


def _workspace_ref(L, q, K, V, gate, cap, B, Tq, L_ctx, q_off, Hq, Hkv, dh, cuda):
    ws = torch.empty(L.gqa_workspace_bytes(B, Tq, L_ctx, Hq, dh) // 4 + 1, device=cuda)
    ref = torch.empty((B * Tq, Hq * dh), dtype=torch.bfloat16, device=cuda)
    L.gqa_attn(q, Hq * dh, K, V, cap, gate, Hq * dh, ref, B, Tq, L_ctx, q_off, Hq, Hkv, dh, True, ws)
    return ref


def test_noalloc_equals_workspace_entry_point_twice(cuda):
    """Decode-shaped split-K attention, two calls in a row (the longer context first, so the
    second call's fewer splits leave stale partials of the first in the scratch), each equal
    to gqa_attn with a workspace bit for bit; one batch row also against the oracle."""
    import looped_hybrid_attention_b200 as L
    B, Hq, Hkv, dh = 8, 16, 4, 256
    for call, L_ctx in enumerate((4100, 3000)):
        cap = L_ctx + 16
        q, K, V, gate = _decode_case(B, Hq, Hkv, dh, cap, seed=100 + call)
        ref = _workspace_ref(L, q, K, V, gate, cap, B, 1, L_ctx, L_ctx - 1, Hq, Hkv, dh, cuda)
        out = torch.full_like(ref, float("nan"))
        L.gqa_attn_noalloc(q, Hq * dh, K, V, cap, gate, Hq * dh, out, B, 1, L_ctx, L_ctx - 1, Hq, Hkv, dh, True)
        torch.cuda.synchronize()
        assert torch.equal(out, ref)
        b = 3
        o = ops.attention(to64(q[b])[None], to64(K[b, :, :L_ctx]).transpose(1, 0, 2),
                          to64(V[b, :, :L_ctx]).transpose(1, 0, 2), [L_ctx - 1])
        o = o.reshape(Hq * dh) * ops.sigmoid(to64(gate[b]))
        assert rel_l2(to64(out[b]), o) < TOL["bf16"]


def test_noalloc_prefill_needs_no_scratch(cuda):
    """Multi-token bf16 queries run the tensor-core kernel, which keeps no partials, so a
    prefill of 3,000 tokens is accepted even though the workspace bound for it is larger
    than the built-in scratch."""
    import looped_hybrid_attention_b200 as L
    B, T, Hq, Hkv, dh = 1, 3000, 16, 4, 256
    assert L.gqa_workspace_bytes(B, T, T, Hq, dh) > 32 << 20
    g = lambda shape, name: synth.normal(shape, 1.0, 7, name).to(torch.bfloat16).cuda()
    q, K, V, gate = g((B * T, Hq * dh), "qp"), g((B, Hkv, T, dh), "Kp"), g((B, Hkv, T, dh), "Vp"), g((B * T, Hq * dh), "gp")
    ref = _workspace_ref(L, q, K, V, gate, T, B, T, T, 0, Hq, Hkv, dh, cuda)
    out = torch.empty_like(ref)
    L.gqa_attn_noalloc(q, Hq * dh, K, V, T, gate, Hq * dh, out, B, T, T, 0, Hq, Hkv, dh, True)
    torch.cuda.synchronize()
    assert torch.equal(out, ref)


def test_noalloc_leaves_device_memory_unchanged(cuda):
    import looped_hybrid_attention_b200 as L
    B, Hq, Hkv, dh, L_ctx = 8, 16, 4, 256, 2048
    q, K, V, gate = _decode_case(B, Hq, Hkv, dh, L_ctx, seed=5)
    out = torch.empty((B, Hq * dh), dtype=torch.bfloat16, device=cuda)
    L.gqa_attn_noalloc(q, Hq * dh, K, V, L_ctx, gate, Hq * dh, out, B, 1, L_ctx, L_ctx - 1, Hq, Hkv, dh, True)
    torch.cuda.synchronize()
    free0, alloc0 = torch.cuda.mem_get_info()[0], torch.cuda.memory_allocated()
    for _ in range(3):
        L.gqa_attn_noalloc(q, Hq * dh, K, V, L_ctx, gate, Hq * dh, out, B, 1, L_ctx, L_ctx - 1, Hq, Hkv, dh, True)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
    assert torch.cuda.memory_allocated() == alloc0


def test_noalloc_rejects_problems_beyond_its_scratch(cuda):
    """32 q heads per KV head take the row kernel; 1,100 single-token rows over 8,192 keys
    split the keys in two, and their partials (1100 x 32 x 2 x 258 x 4 B = 72.6 MB) do not fit."""
    import looped_hybrid_attention_b200 as L
    B, Hq, Hkv, dh, L_ctx = 1100, 32, 1, 256, 8192
    q = torch.zeros((16,), dtype=torch.bfloat16, device=cuda)   # never read: rejected before launch
    with pytest.raises(L.LoopError) as e:
        L.gqa_attn_noalloc(q, Hq * dh, q, q, L_ctx, None, 0, q, B, 1, L_ctx, L_ctx - 1, Hq, Hkv, dh, True)
    assert e.value.status == 5 and "32 MiB" in str(e.value) and "72652800" in str(e.value)
