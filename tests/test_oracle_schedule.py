"""Pins of the oracle's schedule and accounting against the numbers the pages print."""
import numpy as np
import pytest

import synth
from oracle import accounting, schedule


def test_execution_count_and_order(golden):
    s = synth.FULL
    assert s.n_layers == golden["stored_layers"]["value"]
    n, n_fa, n_gdn = schedule.counts(s)
    assert n == golden["executions"]["value"] == 4 + 24 * 2 + 4
    assert n_fa == golden["fa_executions"]["value"]
    assert n_gdn == golden["gdn_executions"]["value"]
    layers = schedule.execution_layers(s.n_layers, s.loop_start, s.loop_end, s.loop_passes)
    assert layers[:4] == [0, 1, 2, 3]
    assert layers[4:28] == list(range(4, 28)) and layers[28:52] == list(range(4, 28))
    assert layers[52:] == [28, 29, 30, 31]


def test_group_pattern(golden):
    s = synth.FULL
    pat = golden["group"]["value"]
    for l in range(s.n_layers):
        assert schedule.layer_kind(l, s.group) == pat[l % 4]
    # the loop block is six whole groups, so both passes see the same pattern
    t = schedule.table(s)
    assert [r[2] for r in t[4:28]] == [r[2] for r in t[28:52]]
    assert (s.loop_end - s.loop_start) % s.group == 0


def test_probe_indices(golden):
    """Probe points [3, 27, 51, 53, 54]: end of head, end of pass 1, end of pass 2, tail."""
    s = synth.FULL
    t = schedule.table(s)
    e3, e27, e51, e53, e54 = (t[i] for i in golden["probe_exec_indices"]["value"])
    assert e3[1] == 3 and not e3[4] and t[4][4]            # last head execution, next enters the loop
    assert e27[1] == 27 and e27[4] and t[28][1] == 4        # pass 1 ends at layer 27, pass 2 restarts at 4
    assert e51[1] == 27 and e51[4] and not t[52][4]         # pass 2 ends, the loop block is left
    assert (e53[1], e54[1]) == (29, 30) and not e53[4]


def test_slots_per_execution():
    s = synth.FULL
    t = schedule.table(s)
    fa = [r for r in t if r[2] == "fa"]
    assert [r[0] for r in fa] == list(range(3, 56, 4))
    assert [r[3] for r in fa] == list(range(14))
    gdn = [r for r in t if r[2] == "gdn"]
    assert [r[3] for r in gdn] == list(range(42))
    # the two passes of one stored layer get different slots (own cache per execution)
    assert t[7][1] == t[31][1] == 7 and t[7][3] != t[31][3]


def test_loop_passes_generalise(golden):
    s3 = synth.FULL.with_(loop_passes=3)
    g = golden["loop_passes_3_executions_printed"]
    assert schedule.counts(s3)[0] == g["arithmetic"] != g["value"]
    assert schedule.counts(synth.FULL.with_(loop_passes=1))[0] == 32
    assert schedule.counts(synth.TINY)[0] == 4 + 4 * 2 + 4


def test_embedding_params(golden):
    s = synth.FULL
    n = accounting.embedding_params(s)
    assert n == 248320 * 4096 == 1_017_118_720
    assert round(n / 1e9, 2) == golden["embedding_params_approx"]["value"]


def test_kv_accounting(golden):
    s = synth.FULL
    per = accounting.kv_bytes_per_token_per_fa_exec(s)
    assert per == 4 * 256 * 2 * 2 == 4096 == golden["kv_bytes_per_token_per_fa_exec_approx_kb"]["value"] * 1024
    tot = accounting.kv_bytes_per_token(s)
    assert tot == 14 * 4096 == golden["kv_bytes_per_token_total_approx_kb"]["value"] * 1024
    # the page rounds 56 KB x 128K with decimal units; the exact bytes are within 5 %
    assert abs(tot * 131072 / 1e9 - golden["kv_128k_gb_approx"]["value"]) / 7.2 < 0.05
    assert abs(tot * 262144 / 1e9 - golden["kv_256k_gb_approx"]["value"]) / 14.4 < 0.05
    assert tot * 131072 == 7_516_192_768


def test_param_totals_are_in_the_pages_range(golden):
    s = synth.FULL
    tot = accounting.total_params(s)
    # the pages fix no GDN widths; with 16 x 128 heads the stack lands below the printed ~9B
    assert 7.5e9 < tot < golden["params_total_approx"]["value"] * 1.05
    # BF16 weights ~ 18 GB ([teardown] §四) within the same uncertainty
    assert 14e9 < 2 * tot < golden["weights_gb_bf16_approx"]["value"] * 1e9 * 1.05
    # executed parameters exceed stored ones by the 24 looped layers (the "inference-equivalent" size)
    assert accounting.executed_params(s) > accounting.total_params(s) - 2 * accounting.embedding_params(s)


def test_layer_param_counts_closed_form():
    s = synth.FULL
    gdn = accounting.layer_params(s, "gdn")
    fa = accounting.layer_params(s, "fa")
    ffn = 3 * 4096 * 12288
    assert gdn == 4096 + (3 * 2048 + 32) * 4096 + 32 + 2048 * 4096 + ffn + 4096
    assert fa == 4096 + 10240 * 4096 + 512 + 4096 * 4096 + ffn + 4096
    assert accounting.mhc_params(s) == 2 * 4096 * 8 + 8
