"""Per-op breakdown of the device trace, on synthetic schedule and stamp arrays (no GPU)."""
import numpy as np
import pytest

from decode_persistent_block_b200.trace import op_breakdown, per_sm_duration


def _put(sched, tr, sm, i, op, layer, stamps_us):
    sched[sm, i, 0] = op
    sched[sm, i, 1] = layer
    tr[sm, i, :] = np.asarray(stamps_us, dtype=np.float64) * 1000 + 1_000_000  # ns, offset like globaltimer


def test_phases_of_a_two_op_step():
    sched = np.zeros((2, 2, 16), np.int32)
    tr = np.zeros((2, 2, 8), np.uint64)
    # QKV on both blocks: start, dep, ready, first, main, end, ld_first, ld_last (µs)
    _put(sched, tr, 0, 0, 1, 0, [0, 1, 2, 3, 5, 6, 0.5, 0.6])
    _put(sched, tr, 1, 0, 1, 0, [0, 1, 2, 3, 6, 8, 0.5, 0.7])
    # LM head on both: its dependency is met 1 µs / 2 µs after QKV's last end (8 µs)
    _put(sched, tr, 0, 1, 6, 1, [6, 9, 10, 11, 20, 21, 4, 15])
    _put(sched, tr, 1, 1, 6, 1, [8, 10, 11, 12, 22, 25, 5, 16])
    bd = op_breakdown(sched, tr)
    assert list(bd) == ["QKV", "LM"]
    q, lm = bd["QKV"], bd["LM"]
    assert np.isnan(q["phase"]) and np.isnan(q["hop"])  # the first op has no predecessor
    assert q["ready"] == pytest.approx(1.0) and q["first"] == pytest.approx(1.0)
    assert q["main"] == pytest.approx(2.5) and q["epi"] == pytest.approx(1.5) and q["spread"] == pytest.approx(2.0)
    assert lm["phase"] == pytest.approx(25 - 8) and lm["hop"] == pytest.approx(1.5)
    assert lm["ld_lead"] == pytest.approx((5 + 5) / 2) and lm["ld_last"] == pytest.approx((6 + 6) / 2)
    assert lm["spread"] == pytest.approx(4.0)


def test_per_sm_duration_and_missing_stamps():
    sched = np.zeros((3, 1, 16), np.int32)
    tr = np.zeros((3, 1, 8), np.uint64)
    _put(sched, tr, 0, 0, 9, 0, [0, 1, 2, 3, 10, 12, 0, 5])
    _put(sched, tr, 1, 0, 9, 1, [0, 2, 2, 3, 10, 20, 0, 5])
    _put(sched, tr, 2, 0, 9, 0, [0, 1, 2, 3, 10, 12, 0, 5])
    tr[2, 0, 1] = 0  # dependency stamp missing: not counted
    d = per_sm_duration(sched, tr, "FFN", 2)
    assert d[0, 0] == pytest.approx(11.0) and np.isnan(d[0, 1])
    assert d[1, 1] == pytest.approx(18.0) and np.isnan(d[1, 0])
    assert np.isnan(d[2]).all()
