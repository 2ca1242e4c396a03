"""Per-SM streaming speed, measured with the device trace, for `mk_options.sm_speed`.

On a given B200 some SMs stream weights persistently slower than others: the
per-SM time of the fused FFN correlates from layer to layer.  Rows split
evenly then leave the slowest SM to set the end of every FFN and of the LM
head.  This module runs a few decode steps with the trace on, and gives each
block the weight bytes it streamed per ns in the dense fused FFN and the LM
head, from dependency met to done.  The result is normalised to mean 1, and a
schedule built with it splits those rows in proportion.
"""
from __future__ import annotations

import numpy as np

from .mk import Decoder

OP_LMHEAD_ARGMAX = 6
OP_FFN = 9
T_DEP, T_END = 1, 5


def sm_speed_from_trace(schedule: np.ndarray, trace: np.ndarray, hidden: int):
    """(bytes, ns) per block from one step's schedule [n_sm, max_instr, 16] and
    trace [n_sm, max_instr, words]: each dense fused-FFN row streams 3 weight rows
    (up, gate, transposed down) of `hidden` bf16, and each LM-head row one."""
    n_sm = schedule.shape[0]
    nbytes = np.zeros(n_sm)
    ns = np.zeros(n_sm)
    op = schedule[:, :, 0]
    rows = (schedule[:, :, 4] - schedule[:, :, 3]).astype(np.float64)
    dur = trace[:, :, T_END].astype(np.int64) - trace[:, :, T_DEP].astype(np.int64)
    ok = (trace[:, :, T_DEP] > 0) & (trace[:, :, T_END] > 0) & (dur > 0)
    for code, per_row in ((OP_FFN, 3 * 2 * hidden), (OP_LMHEAD_ARGMAX, 2 * hidden)):
        m = (op == code) & ok
        nbytes += np.where(m, rows * per_row, 0.0).sum(axis=1)
        ns += np.where(m, dur, 0).sum(axis=1)
    return nbytes, ns


def measure_sm_speed(cfg, weights, kcache, vcache, token: int, pos: int, steps: int = 8, clip: float = 2.0,
                     **options) -> np.ndarray:
    """Relative streaming speed of every block (mean 1, clipped to [1/clip, clip]).

    Runs `steps` + 1 decode steps from (`token`, `pos`) on a traced handle.  The
    first step is not counted.  This writes the KV caches at pos..pos+steps,
    like any decode from `pos`, so run it before decoding from `pos` for real."""
    opts = dict(options)
    opts.pop("sm_speed", None)
    opts["trace"] = 1
    with Decoder(cfg, weights, kcache, vcache, **opts) as d:
        sched = d.schedule()
        nbytes = np.zeros(sched.shape[0])
        ns = np.zeros(sched.shape[0])
        tok = d.step(token, pos)
        for i in range(1, steps + 1):
            tok = d.step(tok, pos + i)
            tr = d.trace().reshape(sched.shape[0], sched.shape[1], -1)
            b, t = sm_speed_from_trace(sched, tr, cfg.hidden)
            nbytes += b
            ns += t
    if not (ns > 0).all():
        raise RuntimeError("calibration: some block streamed no FFN or LM-head rows")
    speed = nbytes / ns
    speed = speed / speed.mean()
    return np.clip(speed, 1.0 / clip, clip)
