"""Failure detection without a GPU fault.

Faults are made on the host (a schedule whose wait target no step reaches, an
opcode outside the table, the stop word set before launch).  Every device wait
is bounded, so each case must come back as an error status within its limit,
leave the context usable, and after mk_reset the next step must again match the
oracle (Hyperkernel teardown, "Hardware fault detection and replanning": a
watchdog that voids the step instead of returning a number).
"""
import time

import numpy as np
import pytest

from decode_persistent_block_b200 import mk
from synth import configs
from tests import parity

pytestmark = pytest.mark.gpu

LIMIT_NS = 10_000_000  # 10 ms


@pytest.fixture(scope="module")
def tiny(cuda):
    return parity.Setup(configs.TINY)


def _recovers(tiny, dec):
    """After reset: a clean run from the pre-filled cache matches the oracle."""
    import torch
    dec.reset()
    tiny.fresh_caches()
    orc = tiny.oracle()
    lg = torch.empty(configs.TINY.vocab, device="cuda")
    reps = []
    nxt = None
    for pos, tok in parity.schedule(configs.TINY, 6):
        t = tok if tok is not None else nxt
        g = dec.step(t, pos, logits=lg)
        o = orc.step(t, pos)
        reps.append(parity.compare_step(configs.TINY, dec, lg.cpu().numpy(), o, g))
        nxt = o["next"]
    parity.assert_parity(reps)


@pytest.mark.parametrize("attn_merge", [1, 2], ids=["merge_in_oproj", "merge_once"])
@pytest.mark.parametrize("block", [0, 3, 147])
def test_unreachable_wait_times_out_and_recovers(tiny, block, attn_merge):
    # With 4 splits, block 0's first waiting instruction is split 0 of kv head 0 in layer 0: with the
    # once-per-head merge the other 3 splits of that head have counted themselves when the step gives
    # up, and the reset must clear those arrivals too, or the next step would take the wrong split
    # for the last one.
    tiny.fresh_caches()
    with tiny.decoder(spin_limit_ns=LIMIT_NS, attn_merge=attn_merge, kv_splits=4) as dec:
        dec.step(1, 0)
        dec.inject_fault(mk.FAULT_UNREACHABLE_WAIT, block)
        t0 = time.perf_counter()
        rc = dec.step_rc(2, 1)
        dt = time.perf_counter() - t0
        assert rc == mk.CODES["MK_ERR_TIMEOUT"], mk.ERRORS.get(rc, rc)
        assert dt < 5.0
        st = dec.status()
        assert st["code"] == rc
        # the block that gave up is the faulted one, or one waiting on it
        assert 0 <= st["sm"] < 148 and st["counter"] >= -1
        if st["counter"] >= 0:
            assert st["expected"] > st["observed"]
        # the stop word makes the following step fail fast too, until reset
        assert dec.step_rc(3, 2) != mk.MK_OK
        _recovers(tiny, dec)


def test_bad_opcode_is_reported(tiny):
    tiny.fresh_caches()
    with tiny.decoder(spin_limit_ns=LIMIT_NS) as dec:
        dec.inject_fault(mk.FAULT_BAD_OPCODE, 5)
        rc = dec.step_rc(4, 0)
        assert rc == mk.CODES["MK_ERR_BAD_INSTR"], mk.ERRORS.get(rc, rc)
        st = dec.status()
        assert st["sm"] == 5 and st["instr"] == 0 and st["opcode"] == 99
        _recovers(tiny, dec)


def test_preset_stop_word(tiny):
    tiny.fresh_caches()
    with tiny.decoder(spin_limit_ns=LIMIT_NS) as dec:
        dec.inject_fault(mk.FAULT_PRESET_STOP)
        t0 = time.perf_counter()
        rc = dec.step_rc(4, 0)
        assert rc == mk.CODES["MK_ERR_STOPPED"] and time.perf_counter() - t0 < 2.0
        _recovers(tiny, dec)


def test_trace_stamps_are_ordered(tiny):
    tiny.fresh_caches()
    with tiny.decoder(trace=1) as dec:
        dec.step(3, 0)
        sched = dec.schedule()
        tr = dec.trace().reshape(sched.shape[0], sched.shape[1], -1).astype(np.int64)
        assert tr.shape[2] == 32  # 8 instruction stamps, then 8 stages x (ready, consumed, issued)
        n = (sched[:, :, 0] != 0).sum(1)
        for sm in range(tr.shape[0]):
            t = tr[sm, :n[sm]]
            # consumer stamps: reached <= dependency <= ready <= first stage <= main done <= end
            assert np.all(t[:, 0] > 0) and np.all(t[:, 5] >= t[:, 1]) and np.all(t[:, 1] >= t[:, 0])
            for a, b in ((1, 2), (2, 3), (3, 4), (4, 5)):
                hit = (t[:, a] > 0) & (t[:, b] > 0)
                assert np.all(t[hit, b] >= t[hit, a]), (sm, a, b)
            assert np.all(np.diff(t[:, 0]) >= 0)
            # loader: the first stage of an instruction is issued before its consumers see it full
            hit = (t[:, 6] > 0) & (t[:, 3] > 0)
            assert np.all(t[hit, 3] >= t[hit, 6]) and np.all(t[t[:, 7] > 0, 7] >= t[t[:, 7] > 0, 6])
            # per stage: issued <= the consumers' wait returned <= their share consumed
            for s_ in range(8):
                ready, done, issued = t[:, 8 + s_], t[:, 16 + s_], t[:, 24 + s_]
                hit = (ready > 0) & (done > 0) & (issued > 0)
                assert np.all(done[hit] >= ready[hit]) and np.all(ready[hit] >= issued[hit]), (sm, s_)
