"""Host logic of the attention trace summary (block_sparse_attention_ibcs_b200.trace) on a
synthetic trace whose events sit at known offsets from each tile's copy start."""

import pytest

from block_sparse_attention_ibcs_b200.trace import EVENTS_PER_SLOT, SLOTS, TILES, summarize

OFFSETS = {0: 0, 1: 1500, 2: 3800, 3: 5400, 4: 2700, 5: 3500, 6: 4000, 7: 7400, 8: 3200,
           9: 3700, 10: 5550, 12: 3850, 13: 5560, 14: 5570, 15: 5540}


def _trace(T, period, start, drain):
    tr = [0] * (SLOTS * EVENTS_PER_SLOT * TILES)
    for slot in range(SLOTS):
        base = start + 1000 * slot
        for t in range(min(T, TILES)):
            for e, off in OFFSETS.items():
                tr[(slot * EVENTS_PER_SLOT + e) * TILES + t] = base + t * period + off
        if T <= TILES:  # the CTA's end, recorded in tile slot 0 of event 11
            tr[(slot * EVENTS_PER_SLOT + 11) * TILES] = base + (T - 1) * period + OFFSETS[7] + drain
    return tr


def test_summary_recovers_offsets_period_fill_and_drain():
    T, period, drain = 64, 2500, 2450
    s = summarize(_trace(T, period, 10**12, drain), T)
    for slot in range(SLOTS):
        d = s[f"cta_slot{slot}"]
        assert d["period"] == period
        assert d["copy_issued"] == 1500 and d["k_landed"] == 2700 and d["pv_issued"] == 7400
        assert d["v_landed"] == 3850 and d["p_stored_w3"] == 5540
        assert d["fill_to_first_qk"] == 3500 and d["fill_to_first_s"] == 3700
        assert d["drain_last_pv_to_end"] == drain
        span = (T - 1) * period + OFFSETS[7] + drain
        assert d["cta_cycles"] == span
        assert d["outside_steady_frac"] == round(1 - period * T / span, 4)


def test_summary_of_blocks_longer_than_the_trace_has_no_drain():
    d = summarize(_trace(200, 2000, 5, 0), 200)["cta_slot0"]
    assert d["period"] == 2000 and "drain_last_pv_to_end" not in d


def test_summary_needs_a_steady_window():
    with pytest.raises(ValueError):
        summarize(_trace(10, 2000, 5, 0), 10)
