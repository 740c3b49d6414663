"""gqa_attn_noalloc: the attention entry point that allocates no device memory.

It is meant for callers that cannot allocate a workspace (a runtime that has given all
free device memory to its own pool, or a loop that must not take the synchronisation of
cudaMalloc / cudaFree).  Its split-K scratch is a fixed array inside the library; its
result must equal the workspace entry point's, call after call.  This file is collected
last so that a failure here comes after every other test has run.
"""
import numpy as np
import pytest
import torch

import synth
from conftest import TOL, rel_l2, to64

pytestmark = pytest.mark.gpu


def _case(B, Hq, Hkv, dh, L_ctx, cap, seed):
    g = lambda shape, name: synth.normal(shape, 1.0, seed, name).to(torch.bfloat16).cuda()
    return g((B, Hq, dh), "q"), g((B, Hkv, cap, dh), "K"), g((B, Hkv, cap, dh), "V"), g((B, Hq * dh), "gate")


def test_noalloc_equals_workspace_entry_point_twice(cuda):
    """Decode-shaped split-K attention, two different calls in a row, against gqa_attn with a workspace."""
    import looped_hybrid_attention_b200 as L
    B, Hq, Hkv, dh = 8, 16, 4, 256
    for call, L_ctx in enumerate((3000, 4100)):
        cap = L_ctx + 16
        q, K, V, gate = _case(B, Hq, Hkv, dh, L_ctx, cap, seed=100 + call)
        ws = torch.empty(L.gqa_workspace_bytes(B, 1, L_ctx, Hq, dh) // 4 + 1, device=cuda)
        ref = torch.empty((B, Hq * dh), dtype=torch.bfloat16, device=cuda)
        L.gqa_attn(q, Hq * dh, K, V, cap, gate, Hq * dh, ref, B, 1, L_ctx, L_ctx - 1, Hq, Hkv, dh, True, ws)
        out = torch.empty_like(ref)
        L.gqa_attn_noalloc(q, Hq * dh, K, V, cap, gate, Hq * dh, out, B, 1, L_ctx, L_ctx - 1, Hq, Hkv, dh, True)
        torch.cuda.synchronize()
        assert rel_l2(to64(out), to64(ref)) <= TOL["bf16"]
        assert torch.isfinite(out.float()).all()


def test_noalloc_rejects_problems_beyond_its_scratch(cuda):
    import looped_hybrid_attention_b200 as L
    B, Hq, Hkv, dh, L_ctx = 2048, 16, 4, 256, 8192     # needs far more than 32 MiB of partials
    assert L.gqa_workspace_bytes(B, 1, L_ctx, Hq, dh) > 32 << 20
    q = torch.zeros((16,), dtype=torch.bfloat16, device=cuda)   # never read: rejected before launch
    with pytest.raises(L.LoopError) as e:
        L.gqa_attn_noalloc(q, Hq * dh, q, q, L_ctx, None, 0, q, B, 1, L_ctx, L_ctx - 1, Hq, Hkv, dh, True)
    assert e.value.status == 5 and "32 MiB" in str(e.value)
