"""The N > 1 path of bench.py on CPU: world size 2 over gloo (127.0.0.1).

Replicas share no data-path collective; what crosses ranks is the barrier,
the max-over-ranks of the timed region, and rank 0 alone printing (and, for
the reference arm, alone running the oracle).
"""
import json
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE="2", RANK=str(rank),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    rank_, world, local = bench.dist_setup()
    try:
        res = {"rank": rank_, "world": world, "backend": dist.get_backend()}
        res["max"] = bench.reduce_max(float(rank + 1), world)
        # rank 0 timed 10 ms, rank 1 12 ms, 4 tokens each: 12 ms over 8 tokens
        res["us_per_token"] = bench.job_us_per_token(10.0 if rank == 0 else 12.0, 4, world)
        bench.barrier(world)
        sys.argv = ["bench.py", "--impl", "reference", "--config", "tiny", "--steps", "2", "--warmup", "1"]
        line = bench.run_reference(bench.parse(), rank_, world)
        res["line"] = line
        bench.barrier(world)
    finally:
        dist.destroy_process_group()
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump(res, f)


def test_two_rank_gloo_bench_path(tmp_path):
    import torch.multiprocessing as mp
    import oracle
    oracle.build()  # compiled once here, not concurrently by the ranks
    mp.start_processes(_rank_main, args=(_free_port(), str(tmp_path)), nprocs=2, join=True, start_method="spawn")
    r0 = json.load(open(tmp_path / "rank0.json"))
    r1 = json.load(open(tmp_path / "rank1.json"))
    for r in (r0, r1):
        assert r["world"] == 2 and r["backend"] == "gloo"
        assert r["max"] == 2.0
        assert r["us_per_token"] == pytest.approx(12.0 * 1000.0 / 8)
    assert r1["line"] is None  # only rank 0 runs and prints the reference arm
    line = r0["line"]
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["higher_is_better"] is False
    assert line["value"] > 0 and line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]
