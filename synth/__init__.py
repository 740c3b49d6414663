"""Seeded synthetic workloads: model shapes, random-init weights and inputs.

This module is the only code shared by the CPU oracle tests and the CUDA path.
It holds none of the decoder's arithmetic: it only names shapes and draws
seeded random numbers (torch generators, one independent stream per tensor,
keyed by a hash of the seed and the tensor's name).

Shapes follow the SenseNova-Loop-9B-Preview pages: hidden 4096, SwiGLU FFN
12288, vocab 248,320, 32 stored layers run as 4 + 24x2 + 4 = 56 executions,
groups of 3 Gated-DeltaNet + 1 GQA layer (16 q / 4 KV heads, head dim 256,
rotary on 0.25 of the head dims), two-stream mHC with 20 Sinkhorn iterations.
The GDN head sizes (16 heads, dk = dv = 128) are this build's reading; the
pages leave them open.
"""
from __future__ import annotations

import hashlib
from dataclasses import dataclass, asdict, replace

import torch

__all__ = [
    "ModelShape", "TINY", "GROUP", "FULL", "stream_seed", "normal", "uniform_ids",
    "make_weights", "layer_kinds", "weight_names",
]


@dataclass(frozen=True)
class ModelShape:
    """Dimensions of a looped hybrid decoder (no arithmetic here)."""
    d: int = 4096                 # hidden size
    ffn: int = 12288              # SwiGLU intermediate size
    vocab: int = 248320
    n_layers: int = 32            # stored decoder layers
    loop_start: int = 4           # first looped layer (inclusive)
    loop_end: int = 28            # last looped layer (exclusive)
    loop_passes: int = 2
    group: int = 4                # layers per hybrid group: (group-1) GDN + 1 FA
    gdn_heads: int = 16
    gdn_dk: int = 128
    gdn_dv: int = 128
    fa_q_heads: int = 16
    fa_kv_heads: int = 4
    fa_head_dim: int = 256
    rotary_dims: int = 64         # 0.25 of the head dim
    mhc_streams: int = 2
    sinkhorn_iters: int = 20
    gdn_chunk: int = 64
    eps: float = 1e-6
    rope_base: float = 10000.0
    dtype: str = "bf16"           # storage dtype of weights and activations
    with_embedding: bool = True   # False: hidden-state in/out (tiny and group configs)
    gdn_variant: int = 0          # 0: plain GDN; 1: short causal conv on q|k|v + gated output norm
    gdn_v_heads: int = 0          # value heads of the variant (0: gdn_heads); a multiple of gdn_heads
    gdn_conv: int = 4             # conv kernel size of the variant

    def as_dict(self):
        return asdict(self)

    def with_(self, **kw) -> "ModelShape":
        return replace(self, **kw)


# Tiny looped stack: 12 stored layers run as 4 + 4x2 + 4 = 16 executions, fp32.
TINY = ModelShape(d=256, ffn=768, vocab=1000, n_layers=12, loop_start=4, loop_end=8,
                  gdn_heads=4, gdn_dk=64, gdn_dv=64, fa_q_heads=4, fa_kv_heads=1,
                  fa_head_dim=64, rotary_dims=16, dtype="fp32", with_embedding=False)

# One full-width four-layer group, all four layers inside the two-stream mHC.
GROUP = ModelShape(n_layers=4, loop_start=0, loop_end=4, loop_passes=1,
                   dtype="bf16", with_embedding=False)

# The full 9B-shape stack.
FULL = ModelShape()


def layer_kinds(shape: ModelShape):
    """'fa' for the last layer of every group, 'gdn' otherwise (stored-layer order)."""
    return ["fa" if (l % shape.group) == shape.group - 1 else "gdn" for l in range(shape.n_layers)]


def stream_seed(seed: int, name: str) -> int:
    h = hashlib.sha256(f"{seed}/{name}".encode()).digest()
    return int.from_bytes(h[:8], "little") & ((1 << 62) - 1)


def _gen(seed: int, name: str, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(stream_seed(seed, name))
    return g


def normal(shape, std: float, seed: int, name: str, device="cpu", mean: float = 0.0) -> torch.Tensor:
    """fp32 N(mean, std^2) tensor from the stream (seed, name)."""
    t = torch.randn(tuple(shape), generator=_gen(seed, name, device), device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    if mean != 0.0:
        t.add_(mean)
    return t


def uniform_ids(shape, vocab: int, seed: int, name: str = "ids", device="cpu") -> torch.Tensor:
    """int32 token ids uniform over [0, vocab)."""
    return torch.randint(0, vocab, tuple(shape), generator=_gen(seed, name, device),
                         device=device, dtype=torch.int64).to(torch.int32)


def _store(t: torch.Tensor, dtype: str) -> torch.Tensor:
    """Round to the storage dtype (bf16 configs keep bf16 tensors)."""
    return t.to(torch.bfloat16) if dtype == "bf16" else t


def weight_names(shape: ModelShape):
    """Names and shapes of every tensor of the model, in a fixed order.

    Row-major, nn.Linear convention: a projection weight is [out, in].
    GDN input projection rows: q (H*dk) | k (H*dk) | v (H*dv) | a (H) | b (H); for the
    variant (gdn_variant 1): q, k (Hk = gdn_heads) | v, z (Hv = gdn_v_heads) | a, b (Hv),
    conv weights [2*Hk*dk + Hv*dv, gdn_conv] and an output-norm gain [dv].
    FA input projection rows:  q (Hq*dh) | gate (Hq*dh) | k (Hkv*dh) | v (Hkv*dh).
    mHC routing map w_r is [streams*d, 8] fp32; b_r is [8] fp32.
    """
    s = shape
    out = []
    if s.with_embedding:
        out.append(("embed", (s.vocab, s.d), "store"))
    for l, kind in enumerate(layer_kinds(s)):
        p = f"layers.{l}."
        out.append((p + "attn_norm", (s.d,), "gain"))
        if kind == "gdn" and s.gdn_variant == 1:
            Hk, Hv, dk, dv = s.gdn_heads, s.gdn_v_heads or s.gdn_heads, s.gdn_dk, s.gdn_dv
            out.append((p + "gdn_w_in", (2 * Hk * dk + 2 * Hv * dv + 2 * Hv, s.d), "store"))
            out.append((p + "gdn_conv_w", (2 * Hk * dk + Hv * dv, s.gdn_conv), "store"))
            out.append((p + "gdn_a_bias", (Hv,), "fp32"))
            out.append((p + "gdn_b_bias", (Hv,), "fp32"))
            out.append((p + "gdn_o_norm", (dv,), "gain"))
            out.append((p + "gdn_w_out", (s.d, Hv * dv), "store"))
        elif kind == "gdn":
            H, dk, dv = s.gdn_heads, s.gdn_dk, s.gdn_dv
            out.append((p + "gdn_w_in", (2 * H * dk + H * dv + 2 * H, s.d), "store"))
            out.append((p + "gdn_a_bias", (H,), "fp32"))
            out.append((p + "gdn_b_bias", (H,), "fp32"))
            out.append((p + "gdn_w_out", (s.d, H * dv), "store"))
        else:
            Hq, Hkv, dh = s.fa_q_heads, s.fa_kv_heads, s.fa_head_dim
            out.append((p + "fa_w_in", (2 * Hq * dh + 2 * Hkv * dh, s.d), "store"))
            out.append((p + "fa_q_norm", (dh,), "gain"))
            out.append((p + "fa_k_norm", (dh,), "gain"))
            out.append((p + "fa_w_out", (s.d, Hq * dh), "store"))
        out.append((p + "ffn_norm", (s.d,), "gain"))
        out.append((p + "ffn_w_gate", (s.ffn, s.d), "store"))
        out.append((p + "ffn_w_up", (s.ffn, s.d), "store"))
        out.append((p + "ffn_w_down", (s.d, s.ffn), "store"))
        if s.loop_start <= l < s.loop_end:
            out.append((p + "mhc_w_r", (s.mhc_streams * s.d, 8), "fp32"))
            out.append((p + "mhc_b_r", (8,), "fp32"))
    if s.with_embedding:
        out.append(("final_norm", (s.d,), "gain"))
        out.append(("lm_head", (s.vocab, s.d), "store"))
    return out


def make_weights(shape: ModelShape, seed: int = 0, device="cpu", std: float = 0.02,
                 gain_std: float = 0.02, names=None):
    """Random-init weights: every tensor N(0, std^2); norm gains 1 + N(0, gain_std^2).

    Projection weights and the embedding are rounded to the storage dtype
    (bf16 for bf16 configs); biases and the mHC routing map stay fp32 (the
    pages keep the mHC routing parameters in FP32).  `names` restricts the
    draw to a subset (each tensor has its own stream, so a subset draws the
    same values as the full set).
    """
    w = {}
    for name, shp, kind in weight_names(shape):
        if names is not None and name not in names:
            continue
        if kind == "gain":
            t = normal(shp, gain_std, seed, name, device, mean=1.0)
            w[name] = _store(t, shape.dtype)
        elif kind == "fp32":
            w[name] = normal(shp, std, seed, name, device)
        else:
            w[name] = _store(normal(shp, std, seed, name, device), shape.dtype)
    return w
