"""Per-SM speed from the device trace, on synthetic schedule and trace arrays (no GPU)."""
import numpy as np
import pytest

from decode_persistent_block_b200.calibrate import sm_speed_from_trace

W_OP, W_BEGIN, W_END = 0, 3, 4
OP_LM, OP_FFN, OP_QKV = 6, 9, 1


def _arrays(n_sm=3, max_instr=4):
    return np.zeros((n_sm, max_instr, 16), np.int32), np.zeros((n_sm, max_instr, 8), np.uint64)


def _put(sched, trace, sm, i, op, rows, t_dep, t_end):
    sched[sm, i, W_OP] = op
    sched[sm, i, W_BEGIN] = 100
    sched[sm, i, W_END] = 100 + rows
    trace[sm, i, 1] = t_dep
    trace[sm, i, 5] = t_end


def test_bytes_and_time_count_only_ffn_and_lm_rows():
    H = 2048
    sched, trace = _arrays()
    _put(sched, trace, 0, 0, OP_QKV, 50, 1000, 2000)      # not counted
    _put(sched, trace, 0, 1, OP_FFN, 10, 3000, 13000)     # 10 rows x (up, gate, down^T) x 2H bytes
    _put(sched, trace, 0, 2, OP_LM, 7, 20000, 27000)      # 7 rows x 2H bytes
    _put(sched, trace, 1, 0, OP_FFN, 4, 5000, 9000)
    _put(sched, trace, 1, 1, OP_LM, 3, 0, 8000)           # dependency stamp missing: skipped
    nbytes, ns = sm_speed_from_trace(sched, trace, H)
    assert nbytes[0] == 10 * 3 * 2 * H + 7 * 2 * H and ns[0] == 10000 + 7000
    assert nbytes[1] == 4 * 3 * 2 * H and ns[1] == 4000
    assert nbytes[2] == 0 and ns[2] == 0


def test_equal_rates_give_equal_speed_and_half_rate_gives_half():
    sched, trace = _arrays(n_sm=2)
    _put(sched, trace, 0, 0, OP_FFN, 8, 1000, 9000)
    _put(sched, trace, 1, 0, OP_FFN, 8, 1000, 17000)
    nbytes, ns = sm_speed_from_trace(sched, trace, 64)
    r = nbytes / ns
    assert r[0] == pytest.approx(2 * r[1])
