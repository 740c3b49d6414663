"""Execution schedule of the looped decoder (oracle, test infrastructure only).

[teardown] §二 and [wiki] §二: 32 stored layers; layers 0-3 run once, the block
4-27 runs twice with the same weights (B(B(h)), the second pass takes the first
pass's output), then layers 28-31 and the head: 4 + 24*2 + 4 = 56 executions.
[teardown] §三 and [wiki] §二: every group of four layers is three Gated-DeltaNet
layers followed by one full-attention layer; the loop block is six whole groups,
so both passes see the same pattern; 14 full-attention and 42 linear-attention
executions.  [teardown] §四: each pass keeps its own attention KV and GDN state,
so caches are counted per execution, not per stored layer.
[probe] §03: the draft-model probes sit at execution indices [3, 27, 51, 53, 54]
(end of the head, end of pass 1, end of pass 2, tail).
"""
from __future__ import annotations


def n_executions(n_layers, loop_start, loop_end, loop_passes):
    """Head + loop_passes x loop block + tail ([teardown] §二: 4 + 24*2 + 4)."""
    return loop_start + (loop_end - loop_start) * loop_passes + (n_layers - loop_end)


def execution_layers(n_layers, loop_start, loop_end, loop_passes):
    """Stored-layer index run by each execution, in execution order."""
    order = list(range(loop_start))
    for _ in range(loop_passes):
        order += list(range(loop_start, loop_end))
    order += list(range(loop_end, n_layers))
    return order


def layer_kind(layer, group):
    """'fa' for the last layer of each group, 'gdn' for the others ([teardown] §三)."""
    return "fa" if layer % group == group - 1 else "gdn"


def table(shape):
    """One row per execution: (execution, layer, kind, slot, in_loop).

    slot is the ordinal of this execution among executions of the same kind:
    the FA executions take KV slabs 0..n_fa-1 and the GDN executions take
    states 0..n_gdn-1, in execution order ([teardown] §四: per-execution caches).
    in_loop marks executions wrapped by the two-stream mHC residual ([wiki] §二:
    mHC is introduced in the loop segment).
    """
    s = shape
    layers = execution_layers(s.n_layers, s.loop_start, s.loop_end, s.loop_passes)
    rows, n_fa, n_gdn = [], 0, 0
    for e, l in enumerate(layers):
        kind = layer_kind(l, s.group)
        if kind == "fa":
            slot, n_fa = n_fa, n_fa + 1
        else:
            slot, n_gdn = n_gdn, n_gdn + 1
        in_loop = s.loop_start <= l < s.loop_end and s.loop_start <= e < s.loop_start + (s.loop_end - s.loop_start) * s.loop_passes
        rows.append((e, l, kind, slot, in_loop))
    return rows


def counts(shape):
    """(n_executions, n_fa_executions, n_gdn_executions)."""
    t = table(shape)
    n_fa = sum(1 for r in t if r[2] == "fa")
    return len(t), n_fa, len(t) - n_fa
