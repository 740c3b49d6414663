"""Parameter and KV-cache accounting (oracle, test infrastructure only).

[teardown] §二: vocab 248,320 x hidden 4096 -> the embedding alone is about 1.02 B
parameters.  [teardown] §四: one full-attention execution stores, per token,
4 KV heads x 256 dims x (K and V) x 2 bytes (BF16) = 4 KB; 14 such executions
make 56 KB per token (about 7.2 GB at 128K tokens, 14.4 GB at 256K).
"""
from __future__ import annotations

from . import schedule


def layer_params(shape, kind):
    """Parameters of one stored layer (norm gains, projections, FFN; mHC counted separately)."""
    s = shape
    ffn = 3 * s.ffn * s.d + s.d                                    # gate, up, down + ffn norm
    if kind == "gdn":
        H, dk, dv = s.gdn_heads, s.gdn_dk, s.gdn_dv
        mixer = (2 * H * dk + H * dv + 2 * H) * s.d + 2 * H + H * dv * s.d
    else:
        Hq, Hkv, dh = s.fa_q_heads, s.fa_kv_heads, s.fa_head_dim
        mixer = (2 * Hq * dh + 2 * Hkv * dh) * s.d + 2 * dh + Hq * dh * s.d
    return s.d + mixer + ffn                                         # + attn norm


def mhc_params(shape):
    """Routing map [streams*d, 8] + bias [8] of one looped layer."""
    return shape.mhc_streams * shape.d * 8 + 8


def embedding_params(shape):
    return shape.vocab * shape.d


def total_params(shape, tied=False):
    s = shape
    n = sum(layer_params(s, schedule.layer_kind(l, s.group)) for l in range(s.n_layers))
    n += (s.loop_end - s.loop_start) * mhc_params(s)
    if s.with_embedding:
        n += embedding_params(s) * (1 if tied else 2) + s.d           # + final norm
    return n


def executed_params(shape):
    """Layer parameters touched per token, counted per execution (the loop block twice)."""
    s = shape
    rows = schedule.table(s)
    return sum(layer_params(s, r[2]) + (mhc_params(s) if r[4] else 0) for r in rows)


def kv_bytes_per_token_per_fa_exec(shape, bytes_per_elem=2):
    return shape.fa_kv_heads * shape.fa_head_dim * 2 * bytes_per_elem


def kv_bytes_per_token(shape, bytes_per_elem=2):
    _, n_fa, _ = schedule.counts(shape)
    return n_fa * kv_bytes_per_token_per_fa_exec(shape, bytes_per_elem)


def gdn_state_bytes_per_sequence(shape, bytes_per_elem=4):
    _, _, n_gdn = schedule.counts(shape)
    return n_gdn * shape.gdn_heads * shape.gdn_dk * shape.gdn_dv * bytes_per_elem
