"""Time one kernel of the library at a chosen shape (CUDA events), e.g. for ncu captures.

  python -m looped_hybrid_attention_b200.kernel_bench gemm --M 8192 --N 12288 --K 4096 --epi swiglu
  python -m looped_hybrid_attention_b200.kernel_bench gdn --T 8192 --H 16
  python -m looped_hybrid_attention_b200.kernel_bench attn --T 8192
  python -m looped_hybrid_attention_b200.kernel_bench mhc --T 8192
  python -m looped_hybrid_attention_b200.kernel_bench decode --B 16 --T 32768
  python -m looped_hybrid_attention_b200.kernel_bench group --T 8192   (one full-width layer group in the model flow)
  python -m looped_hybrid_attention_b200.kernel_bench gdnstep --B 64   (recurrent GDN step, 16 heads x 128)
  python -m looped_hybrid_attention_b200.kernel_bench rmsnorm --M 8192 (d 4096, with the residual sum)
  python -m looped_hybrid_attention_b200.kernel_bench gdnprep --M 8192 (GDN input preparation, 16 heads)
  python -m looped_hybrid_attention_b200.kernel_bench faprep --T 8192  (QK-norm, rotary, K/V slab write)

Inputs are random bf16 tensors created on the device (larger than L2 at the default
sizes); the printed rate uses the same algorithmic flop/byte counts as bench.py.
"""
from __future__ import annotations

import argparse
import json

import torch

import looped_hybrid_attention_b200 as L


def timed(fn, warmup, iters):
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(iters):
        fn()
    b.record()
    torch.cuda.synchronize()
    return a.elapsed_time(b) / iters


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("op", choices=["gemm", "gdn", "attn", "decode", "mhc", "group", "gdnstep", "rmsnorm", "gdnprep",
                                   "faprep"])
    ap.add_argument("--M", type=int, default=8192)
    ap.add_argument("--N", type=int, default=12288)
    ap.add_argument("--K", type=int, default=4096)
    ap.add_argument("--epi", choices=["store", "add", "swiglu", "f32", "gdn"], default="swiglu",
                    help="gdn: the GDN input projection with its preparation in the epilogue (N = 3*H*128 + 2*H)")
    ap.add_argument("--T", type=int, default=8192)
    ap.add_argument("--H", type=int, default=16)
    ap.add_argument("--B", type=int, default=1)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--iters", type=int, default=10)
    ap.add_argument("--no-ws", action="store_true", help="gemm: no partial-sum workspace (whole tiles per CTA)")
    ap.add_argument("--rotate", type=int, default=1,
                    help="gemm: cycle through this many weight copies (more than L2 holds: cold weights)")
    ap.add_argument("--graph", action="store_true",
                    help="gemm: time a CUDA graph of the launches (no host issue cost in the timing)")
    a = ap.parse_args()
    dev = torch.device("cuda")
    g = torch.Generator(device=dev).manual_seed(0)
    bf = torch.bfloat16
    r = lambda *s, std=1.0: (std * torch.randn(*s, device=dev, generator=g)).to(bf)
    res = {"op": a.op}
    if a.op == "gemm" and a.epi == "gdn":
        H = a.N // 386 if a.N % 386 == 0 else 16            # N = 3*H*128 + 2*H
        N = 3 * H * 128 + 2 * H
        X, W = r(a.M, a.K), r(N, a.K, std=0.02)
        q = torch.empty((a.M, H, 128), device=dev, dtype=bf)
        k, v = torch.empty_like(q), torch.empty_like(q)
        gg, beta = torch.empty((a.M, H), device=dev), torch.empty((a.M, H), device=dev)
        ab, bb = torch.zeros(H, device=dev), torch.zeros(H, device=dev)
        ms = timed(lambda: L.gdn_in_proj(X, W, ab, bb, q, k, v, gg, beta, H, 128, 128, 1e-6), a.warmup, a.iters)
        flops = 2.0 * a.M * N * a.K
        byts = 2.0 * (a.M * a.K + N * a.K) + 2.0 * a.M * 3 * H * 128 + 8.0 * a.M * H
        res.update(shape=[a.M, N, a.K], epi="gdn", ms=ms, tflops=flops / ms / 1e9, gbs=byts / ms / 1e6)
    elif a.op == "gemm":
        X = r(a.M, a.K)
        Ws = [r(a.N, a.K, std=0.02) for _ in range(a.rotate)]
        W2s = [r(a.N, a.K, std=0.02) if a.epi == "swiglu" else None for _ in range(a.rotate)]
        R = r(a.M, a.N) if a.epi == "add" else None
        Y = torch.empty((a.M, a.N), device=dev, dtype=torch.float32 if a.epi == "f32" else bf)
        epi = {"store": L.EPI_STORE, "add": L.EPI_ADD, "swiglu": L.EPI_SWIGLU, "f32": L.EPI_F32}[a.epi]
        # zero-filled partial-sum workspace for few rows (M <= 128), as the runtime gives it
        nws = L.linear_workspace_bytes(a.M, a.N, a.K, epi)
        ws = torch.zeros(nws // 4 + 1, device=dev) if nws and not a.no_ws else None
        it = [0]

        def call():
            i = it[0] % a.rotate
            it[0] += 1
            L.linear(X, Ws[i], Y, epi, W2=W2s[i], R=R, workspace=ws)

        if a.graph:
            for _ in range(a.warmup):
                call()
            torch.cuda.synchronize()
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph):
                for _ in range(a.iters):
                    call()
            ms = timed(graph.replay, 2, 1) / a.iters
        else:
            ms = timed(call, a.warmup, a.iters)
        nmat = 2 if a.epi == "swiglu" else 1
        flops = 2.0 * a.M * a.N * a.K * nmat
        byts = 2.0 * (a.M * a.K + nmat * a.N * a.K) + Y.element_size() * a.M * a.N * (2 if a.epi == "add" else 1)
        res.update(shape=[a.M, a.N, a.K], epi=a.epi, ms=ms, tflops=flops / ms / 1e9, gbs=byts / ms / 1e6)
    elif a.op == "gdn":
        B, T, H, dk = a.B, a.T, a.H, 128
        q = torch.nn.functional.normalize(torch.randn(B, T, H, dk, device=dev, generator=g), dim=-1).to(bf)
        k = torch.nn.functional.normalize(torch.randn(B, T, H, dk, device=dev, generator=g), dim=-1).to(bf)
        v = r(B, T, H, dk)
        gg = -torch.nn.functional.softplus(torch.randn(B, T, H, device=dev, generator=g))
        beta = torch.sigmoid(torch.randn(B, T, H, device=dev, generator=g))
        S = torch.zeros(B, H, dk, dk, device=dev)
        out = torch.empty_like(v)
        ws = torch.empty(L.gdn_workspace_bytes(B, T, H, dk, dk) // 4, device=dev)
        ms = timed(lambda: L.gdn_chunk_fwd(q, k, v, gg, beta, S, out, dk ** -0.5, workspace=ws), a.warmup, a.iters)
        byts = B * T * H * (4 * dk * 2 + 8) + 8 * B * H * dk * dk
        res.update(shape=[B, T, H, dk], ms=ms, gbs=byts / ms / 1e6)
    elif a.op == "attn":
        B, T, Hq, Hkv, dh = a.B, a.T, 16, 4, 256
        q, gate = r(B * T, Hq, dh), r(B * T, Hq * dh)
        K, V = r(B, Hkv, T, dh), r(B, Hkv, T, dh)
        out = torch.empty((B * T, Hq * dh), device=dev, dtype=bf)
        ms = timed(lambda: L.gqa_attn(q, Hq * dh, K, V, T, gate, Hq * dh, out, B, T, T, 0, Hq, Hkv, dh, True),
                   a.warmup, a.iters)
        flops = 4.0 * Hq * dh * B * T * (T + 1) / 2
        res.update(shape=[B, T, Hq, Hkv, dh], ms=ms, tflops=flops / ms / 1e9)
    elif a.op == "decode":
        B, T, Hq, Hkv, dh = a.B, a.T, 16, 4, 256
        q, gate = r(B, Hq * dh), r(B, Hq * dh)
        K, V = r(B, Hkv, T, dh), r(B, Hkv, T, dh)
        out = torch.empty((B, Hq * dh), device=dev, dtype=bf)
        ws = torch.empty(L.gqa_workspace_bytes(B, 1, T, Hq, dh) // 4 + 1, device=dev)
        ms = timed(lambda: L.gqa_attn(q, Hq * dh, K, V, T, gate, Hq * dh, out, B, 1, T, T - 1, Hq, Hkv, dh, True, ws),
                   a.warmup, a.iters)
        res.update(shape=[B, T, Hq, Hkv, dh], ms=ms, gbs=B * Hkv * T * dh * 2 * 2 / ms / 1e6)
    elif a.op == "gdnstep":
        B, H, dk = a.B, a.H, 128
        q = torch.nn.functional.normalize(torch.randn(B, H, dk, device=dev, generator=g), dim=-1).to(bf)
        k = torch.nn.functional.normalize(torch.randn(B, H, dk, device=dev, generator=g), dim=-1).to(bf)
        v = r(B, H, dk)
        gg = -torch.nn.functional.softplus(torch.randn(B, H, device=dev, generator=g))
        beta = torch.sigmoid(torch.randn(B, H, device=dev, generator=g))
        S = 0.1 * torch.randn(B, H, dk, dk, device=dev, generator=g)
        out = torch.empty_like(v)
        ms = timed(lambda: L.gdn_step(q, k, v, gg, beta, S, out, dk ** -0.5), a.warmup, a.iters)
        byts = 8.0 * B * H * dk * dk + B * H * (4 * dk * 2 + 8)
        res.update(shape=[B, H, dk], ms=ms, gbs=byts / ms / 1e6)
    elif a.op == "rmsnorm":
        M, d = a.M, 4096
        x, rr, w = r(M, d), r(M, d), r(d)
        y, sm = torch.empty_like(x), torch.empty_like(x)
        ms = timed(lambda: L.rmsnorm(x, w, y, 1e-6, r=rr, sum_out=sm), a.warmup, a.iters)
        ms_add = timed(lambda: L.rmsnorm(x, w, y, 1e-6, r=rr), a.warmup, a.iters)
        ms_plain = timed(lambda: L.rmsnorm(x, w, y, 1e-6), a.warmup, a.iters)
        res.update(shape=[M, d], ms=ms, gbs=2.0 * 4 * M * d / ms / 1e6,
                   add_no_sum_ms=ms_add, add_no_sum_gbs=2.0 * 3 * M * d / ms_add / 1e6,
                   plain_ms=ms_plain, plain_gbs=2.0 * 2 * M * d / ms_plain / 1e6)
    elif a.op == "gdnprep":
        M, H, dk = a.M, a.H, 128
        n_in = 3 * H * dk + 2 * H
        P = r(M, n_in)
        ab, bb = torch.zeros(H, device=dev), torch.zeros(H, device=dev)
        q = torch.empty((M, H, dk), device=dev, dtype=bf)
        k, v = torch.empty_like(q), torch.empty_like(q)
        gg, beta = torch.empty((M, H), device=dev), torch.empty((M, H), device=dev)
        ms = timed(lambda: L.gdn_prep(P, ab, bb, q, k, v, gg, beta, H, dk, dk, 1e-6), a.warmup, a.iters)
        res.update(shape=[M, H, dk], ms=ms, gbs=(2.0 * M * n_in + 2.0 * 3 * M * H * dk + 8.0 * M * H) / ms / 1e6)
    elif a.op == "faprep":
        T, Hq, Hkv, dh = a.T, 16, 4, 256
        P = r(T, 2 * Hq * dh + 2 * Hkv * dh)
        qn, kn = r(dh), r(dh)
        qo = torch.empty((T, Hq, dh), device=dev, dtype=bf)
        K, V = torch.empty((1, Hkv, T, dh), device=dev, dtype=bf), torch.empty((1, Hkv, T, dh), device=dev, dtype=bf)
        ms = timed(lambda: L.fa_prep(P, qn, kn, qo, K, V, T, 1, T, 0, Hq, Hkv, dh, 64, 10000.0, 1e-6),
                   a.warmup, a.iters)
        ms_kv = timed(lambda: L.fa_prep(P, qn, kn, None, K, V, T, 1, T, 0, Hq, Hkv, dh, 64, 10000.0, 1e-6),
                      a.warmup, a.iters)
        res.update(shape=[T, Hq, Hkv, dh], ms=ms, gbs=2.0 * T * (Hq + 2 * Hkv) * dh * 2 / ms / 1e6,
                   kv_only_ms=ms_kv, kv_only_gbs=2.0 * T * (2 * Hkv) * dh * 2 / ms_kv / 1e6)
    elif a.op == "group":
        import synth
        shape = synth.GROUP
        w = synth.make_weights(shape, seed=0, device=dev)
        m = L.Model(shape, w)
        c = m.cache(a.B, a.T)
        h = torch.randn((a.B, a.T, shape.d), device=dev, generator=g).to(bf)
        out = torch.empty_like(h)

        def run():
            c.reset()
            m.forward_hidden(c, h, out)
        ms = timed(run, a.warmup, a.iters)
        m.profile(True)
        run()
        torch.cuda.synchronize()
        prof = {k: [v["launches"], round(v["ms"], 4)] for k, v in m.profile_read().items() if v["launches"]}
        m.profile(False)
        res.update(shape=[a.B, a.T], ms=ms, tokens_per_s=a.B * a.T / ms * 1e3, per_kernel_ms=prof)
    else:
        N, d = a.B * a.T, 4096
        X, F = r(N, 2, d), r(N, d)
        w_r = 0.02 * torch.randn(2 * d, 8, device=dev, generator=g)
        b_r = torch.zeros(8, device=dev)
        c_in = torch.tensor([0.5, 0.5, 1, 1, 0.6, 0.4, 0.4, 0.6], device=dev).repeat(N, 1)
        c_out = torch.empty_like(c_in)
        x_in = torch.empty((N, d), device=dev, dtype=bf)
        ms = timed(lambda: L.mhc_route_mix(L.MHC_MIX, X, F, c_in, w_r, b_r, X, x_in, None, c_out, N, d, 1e-6, 20,
                                           L.BF16), a.warmup, a.iters)
        h = torch.empty((N, d), device=dev, dtype=bf)
        ms_m = timed(lambda: L.mhc_route_mix(L.MHC_MERGE, X, F, c_in, None, None, None, None, h, None, N, d, 1e-6, 20,
                                             L.BF16), a.warmup, a.iters)
        res.update(shape=[N, d], ms=ms, gbs=N * (2 * 6 * d + 64) / ms / 1e6,
                   merge_ms=ms_m, merge_gbs=N * (2 * 4 * d + 32) / ms_m / 1e6)
    assert L.device_error() == 0
    print(json.dumps(res))


if __name__ == "__main__":
    main()
