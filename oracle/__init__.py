"""CPU oracle for the looped hybrid decoder forward pass -- TEST INFRASTRUCTURE ONLY.

Plain, slow, obviously-correct numpy code in float64.  It defines what the
CUDA path must compute and is used only by `tests/`, by `__graft_entry__.smoke()`
and by the CPU-baseline leg of `bench.py`.  The product path never imports it,
and it imports nothing from the product package (only the seeded generators in
`synth`).

Sources, cited by page and section throughout:
  [teardown]  "Loop-9B 拆解" engineering teardown, hncyxsy.com/news/268323,
              sections 一 (release) … 八 (outlook); §二 loop schedule and
              parameter/FLOP accounting, §三 hybrid attention, §四 KV memory,
              §五 mHC + Sinkhorn, §六 minimal repro.
  [wiki]      "SenseNova-Loop-9B 是什么？", yuliuswiki.com/sensenova-loop-9b,
              §二 (loop + mHC), §三 (spec list).
  [probe]     "商汤9B新模型竟反杀27B?…原地套圈的秘密", yeyulingfeng.com/a/1332585.html,
              §01 (config), §02 (mHC, FP32 routing, Sinkhorn-Knopp),
              §03 (draft-model probe points at execution indices).

Modules:
  schedule    execution order and cache-slot tables
  ops         each operation of a layer (norms, GDN recurrence, attention, RoPE,
              Sinkhorn, mHC routing/mixing, FFN, LM head, argmax)
  gdn_chunked the chunked (UT-transform) re-association of the GDN recurrence,
              used only as a cross-check of the algebra the GPU scan uses
  model       whole-model forward: hidden-state stacks, prefill, decode step
  accounting  parameter count and KV-cache bytes

Parity status: every function here is pinned by a test in tests/test_oracle_*.py
against values the pages print, closed forms, library routines or brute force,
except the end-to-end model on trained weights (no weights exist here) --
"parity unpinned" for quality metrics only.
"""
from . import schedule, ops, gdn_chunked, model, accounting  # noqa: F401
