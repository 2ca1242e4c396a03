"""Stored expected values under tests/golden/.

- byte_floor.txt: the byte-floor arithmetic the pages work through (Hyperkernel
  teardown, "Where the numbers sit against the hardware").  It pins the floor
  that bench.py reports (`floor_us_at_8tbs`) to the printed figures.
- tiny_oracle_steps.txt: the fp64 oracle's greedy decode of the tiny workload,
  written by tests/golden/make_tiny_oracle.py (which calls only the oracle and
  the input generators).  It guards the oracle against unintended changes.
"""
import os
import sys

import numpy as np
import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
sys.path.insert(0, ROOT)
GOLDEN = os.path.join(HERE, "golden")


def _rows(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]


@pytest.mark.parametrize("row", _rows("byte_floor.txt"), ids=lambda r: r[0])
def test_byte_floor_matches_the_pages_worked_examples(row):
    import bench
    _, nbytes, steps, gbs, floor_ms, dec, reported_ms, ratio, rdec = row
    floor = bench.byte_floor_us(float(nbytes) * int(steps), float(gbs)) / 1000.0
    assert round(floor, int(dec)) == pytest.approx(float(floor_ms), abs=1e-9)
    if ratio != "-":
        assert round(float(reported_ms) / floor, int(rdec)) == pytest.approx(float(ratio), abs=1e-9)
    else:  # the page: the reported time is within 2x of the floor
        assert 1.0 < float(reported_ms) / floor < 2.0


def test_byte_floor_of_the_workloads():
    # the floors of the decode workloads at 8 TB/s: 2.507 GB -> 313.4 us (1B), 6.668 GB -> 833.5 us (3B)
    import bench
    from synth import configs

    def avg_bytes(cfg):
        p0 = cfg.prefill + cfg.prompt_len
        return np.mean([cfg.weight_bytes_per_token() + cfg.kv_bytes_per_token(p0 + i) for i in range(cfg.steps)])

    assert bench.byte_floor_us(avg_bytes(configs.LLAMA_1B), 8000) == pytest.approx(313.4, abs=0.05)
    assert bench.byte_floor_us(avg_bytes(configs.LLAMA_3B), 8000) == pytest.approx(833.5, abs=0.05)


def test_oracle_reproduces_its_stored_tiny_decode():
    sys.path.insert(0, GOLDEN)
    import make_tiny_oracle

    want = _rows("tiny_oracle_steps.txt")
    got = make_tiny_oracle.decode_tiny()
    assert len(got) == len(want) == 24
    for g, w in zip(got, want):
        assert (g[0], g[1], g[2]) == (int(w[0]), int(w[1]), int(w[2]))
        np.testing.assert_allclose(g[3:], [float(x) for x in w[3:]], rtol=1e-9, atol=1e-12)
