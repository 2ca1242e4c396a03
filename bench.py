#!/usr/bin/env python
"""Batch-1 decode benchmark of the persistent megakernel on B200.

One "step" is one decode step (one token) of the configured workload: the
Llama-3.2-1B-shaped random-init model with its KV cache pre-filled to 1024
positions, decoding positions 1024..1151 (cycled when more steps are timed).
Prints ONE JSON line (rank 0):
  value            device-timed µs/token (CUDA events around K back-to-back
                   launches on the launching stream, token fed on the device),
                   whole job: max-over-ranks time / (K * ranks)
  e2e              the same metric through the C ABI with a host round trip
                   per step (token in by value, next token + status read back
                   from device to pinned host memory, synchronised)
  e2e_serve        the same through launch-once serving (mk_serve_step): one
                   resident grid, each step a mailbox round trip
  roofline         algorithmic bytes per token / mean launch duration vs the
                   measured HBM copy bandwidth
  cpu_baseline     the fp64 oracle on this host's cores, bounded sample
  baselines        the plain multi-kernel path of the same opcodes, stream
                   launches and a CUDA graph
  per_config       the Llama-3B-shaped and Mixtral-shaped workloads timed the
                   same way in the same run (value, roofline, e2e, clocks,
                   baselines), beside the Llama-1B headline
`--impl reference` times the fp64 oracle instead (rank 0 only).
Multi-GPU (torchrun): independent replicas, one per GPU, no collective on the
data path ("scaling": "weak").
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "batch-1 decode µs/token and achieved HBM GB/s vs ~8 TB/s roofline (1×B200)"
UNIT = "µs/token"
ROOFLINE_NOMINAL_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0


def byte_floor_us(n_bytes: float, gbs: float) -> float:
    """Least time, in µs, to stream `n_bytes` from HBM at `gbs` GB/s.  At batch 1
    every weight byte crosses HBM at least once per step, so bytes over
    bandwidth bounds any kernel from below (Hyperkernel teardown, "Where the
    numbers sit against the hardware")."""
    return n_bytes / (gbs * 1e9) * 1e6


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1280)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default="llama1b")
    ap.add_argument("--mode", default="megakernel", choices=["megakernel", "multi_kernel", "multi_kernel_graph"])
    ap.add_argument("--layers", type=int, default=0, help="override n_layers (profiling small cases only)")
    ap.add_argument("--l2-prefetch", type=int, default=-1)
    ap.add_argument("--ring-stages", type=int, default=0)
    ap.add_argument("--stage-bytes", type=int, default=0)
    ap.add_argument("--kv-splits", type=int, default=0)
    ap.add_argument("--batch-only", type=int, default=0,
                    help="profiling: time only batched decode of this many sequences (no headline line)")
    ap.add_argument("--batch-sizes", default="2,4,8",
                    help="batched-decode sizes measured after the headline (comma list; empty: none)")
    ap.add_argument("--spec-experts", type=int, default=-1,
                    help="MoE configs: speculative expert prediction (0 off, 1 on, 2 mispredict; -1: the "
                         "library default)")
    ap.add_argument("--attn-merge", type=int, default=0,
                    help="merge of the attention splits: 1 in every O-projection block, 2 once per kv head "
                         "(0: the library default)")
    ap.add_argument("--ffn-early-stages", type=int, default=0,
                    help="dense FFN stages the loader issues before the FFN's dependency is met (-1: no limit; "
                         "0: the library default)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-baselines", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--per-config", type=int, default=1,
                    help="1: with the default llama1b workload, also time llama3b and mixtral8l (per_config)")
    ap.add_argument("--calibrate", type=int, default=0,
                    help="1: split the FFN and LM-head rows by per-SM speed measured on this GPU at start-up")
    return ap.parse_args()


# ---- process group (replicas) ---------------------------------------------------------------

def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def reduce_max(x: float, world: int) -> float:
    if world <= 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if torch.cuda.is_available() and dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_us_per_token(local_ms: float, steps: int, world: int) -> float:
    """Whole-job time per token: the slowest rank's device time over the
    tokens all ranks decoded (each rank decodes `steps` tokens of its own
    replica)."""
    return reduce_max(local_ms, world) * 1000.0 / (steps * world)


# ---- clocks during the timed region ---------------------------------------------------------------

class Clocks:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "50"], stdout=self.f,
                                         stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None

    def stop(self) -> dict | None:
        if not self.proc:
            return None
        time.sleep(0.1)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower().startswith("active")})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(float(r[2]) for r in rows if r[2].replace(".", "").isdigit()),
                "samples": len(rows), "power_w_max": max(float(r[3]) for r in rows
                                                          if r[3].replace(".", "").isdigit()),
                "reasons": reasons}


# ---- measured peaks and committed ncu traffic ---------------------------------------------------------

def hbm_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        v = float(json.load(open(p))["hbm_gbs"])
        return v, "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


_COMMENT = re.compile(r"//[^\n]*|/\*.*?\*/", re.S)


def kernel_source_hash() -> str:
    """Hash of the library sources with comments and whitespace removed, so a
    profile summary stays attached to the code it measured across comment-only
    edits."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "decode_persistent_block_b200", "csrc")
    for f in sorted(os.listdir(csrc)):
        code = _COMMENT.sub(" ", open(os.path.join(csrc, f), encoding="utf-8").read())
        h.update(f.encode())
        h.update(" ".join(code.split()).encode())
    return h.hexdigest()[:16]


def committed_traffic(config: str, mode: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current kernel sources (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        d = json.load(open(p))
        e = d[f"{mode}:{config}"]
        if e.get("kernel_hash") == kernel_source_hash():
            return e["dram_bytes_per_launch"]
    except Exception:
        pass
    return None


# ---- workload ---------------------------------------------------------------------------------------

def workload(args):
    from synth import configs
    cfg = configs.get(args.config)
    if args.layers:
        cfg = cfg.with_(name=f"{cfg.name}_L{args.layers}", n_layers=args.layers)
    p0 = cfg.prefill + cfg.prompt_len
    positions = [p0 + (i % cfg.steps) for i in range(max(args.steps, args.warmup) + 1)]
    return cfg, p0, positions


def oracle_steps(cfg, seconds: float, max_steps: int | None = None, min_steps: int = 2):
    """Time the fp64 oracle on consecutive decode positions: until `max_steps`
    steps or about `seconds` of work, whichever comes first (at least
    `min_steps`)."""
    import oracle
    import synth
    W = synth.make_model(cfg)
    kc, vc = synth.make_kv_cache(cfg)
    orc = oracle.Model(cfg, W, kc, vc)
    p0 = cfg.prefill + cfg.prompt_len
    tok = int(synth.prompt_tokens(cfg)[0])
    times = []
    t_start = time.perf_counter()
    i = 0
    while True:
        t0 = time.perf_counter()
        tok = orc.step(tok, p0 + (i % cfg.steps), want_hidden=False)["next"]
        times.append(time.perf_counter() - t0)
        i += 1
        if max_steps is not None and i >= max_steps:
            break
        if time.perf_counter() - t_start >= seconds and i >= min_steps:
            break
    return times, oracle.num_threads()


def single_thread_oracle_ms(args, steps: int = 2):
    """ms/token of the fp64 oracle on one host thread (OMP_NUM_THREADS=1, a
    child process), over `steps` decode steps of the workload."""
    code = ("import sys, json; sys.path.insert(0, %r); import bench, statistics; "
            "a = bench.parse(); cfg, p0, pos = bench.workload(a); "
            "t, c = bench.oracle_steps(cfg, 0, max_steps=%d); "
            "print(json.dumps([statistics.fmean(t) * 1e3, c]))") % (ROOT, steps)
    env = dict(os.environ, OMP_NUM_THREADS="1")
    argv = [sys.executable, "-c", code, "--config", args.config] + (["--layers", str(args.layers)] if args.layers else [])
    try:
        out = subprocess.run(argv, env=env, capture_output=True, text=True, timeout=300)
        ms, cores = json.loads(out.stdout.strip().splitlines()[-1])
        return round(ms, 1) if cores == 1 else None
    except Exception:
        return None


def bytes_per_token(cfg, positions):
    return cfg.weight_bytes_per_token() + statistics.fmean(cfg.kv_bytes_per_token(p) for p in positions)


# ---- our arm --------------------------------------------------------------------------------------------

def measure(args, cfg, p0, positions, K, Wm, rank, world, local, with_extras=True):
    """Device-timed steps of one workload through the megakernel (or the
    multi-kernel path), plus the C-ABI end-to-end loops and the multi-kernel
    baselines; returns the measured fields of one bench entry."""
    import numpy as np
    import torch

    import synth
    from decode_persistent_block_b200 import Decoder, to_device
    from decode_persistent_block_b200.calibrate import measure_sm_speed
    torch.cuda.set_device(local)
    W = synth.make_model(cfg)
    kc, vc = synth.make_kv_cache(cfg)
    dW = to_device(W)
    del W
    dk = torch.from_numpy(kc.view(np.int16)).cuda()
    dv = torch.from_numpy(vc.view(np.int16)).cuda()
    del kc, vc
    first = int(synth.prompt_tokens(cfg)[0])
    mode = {"megakernel": 0, "multi_kernel": 1, "multi_kernel_graph": 2}[args.mode]
    opts = dict(mode=mode, l2_prefetch=args.l2_prefetch, ring_stages=args.ring_stages,
                stage_bytes=args.stage_bytes, kv_splits=args.kv_splits, serve_idle_ns=2_000_000_000)
    if cfg.n_experts and args.spec_experts >= 0:
        opts["spec_experts"] = args.spec_experts
    if args.attn_merge:
        opts["attn_merge"] = args.attn_merge
    if args.ffn_early_stages:
        opts["ffn_early_stages"] = args.ffn_early_stages
    calib = None
    if args.calibrate and args.mode == "megakernel":
        # start-up calibration, outside the timed region: a few traced steps from p0
        speed = measure_sm_speed(cfg, dW, dk, dv, first, positions[0], steps=8, **opts)
        opts["sm_speed"] = speed
        calib = {"steps": 8, "min": round(float(speed.min()), 3), "max": round(float(speed.max()), 3)}
    dec = Decoder(cfg, dW, dk, dv, **opts)

    def timed(d, k, warm):
        d.step(first, positions[0])
        for i in range(1, warm):
            d.step(-1, positions[i], sync=False)
        torch.cuda.synchronize()
        barrier(world)
        torch.cuda.synchronize()
        stream = torch.cuda.current_stream()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(k)]
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(k):
            evs[i][0].record(stream)
            d.step(-1, positions[i % len(positions)], sync=False)
            evs[i][1].record(stream)
        e1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        st = d.status()
        if st["code"] != 0:
            raise RuntimeError(f"device status after timed steps: {st}")
        return e0.elapsed_time(e1), [a.elapsed_time(b) for a, b in evs]

    clocks = Clocks(int(os.environ.get("CUDA_VISIBLE_DEVICES", str(local)).split(",")[0])
                    if os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",")[0].isdigit() else local)
    clocks.start()
    total_ms, per_launch = timed(dec, K, Wm)
    clk = clocks.stop()
    us_per_token = job_us_per_token(total_ms, K, world)
    launch_ms = statistics.fmean(per_launch)
    bpt = bytes_per_token(cfg, [positions[i % len(positions)] for i in range(K)])
    peak, peak_kind = hbm_peak()
    achieved = bpt / (launch_ms * 1e-3) / 1e9

    # e2e through the C ABI: token in by value, next token + status back to pinned host memory, per step
    e2e = None
    if not args.no_e2e:
        tok = dec.step(first, positions[0])
        torch.cuda.synchronize()
        barrier(world)
        t0 = time.perf_counter()
        for i in range(K):
            tok = dec.step(tok, positions[i % len(positions)])
        t1 = time.perf_counter()
        e2e_s = reduce_max(t1 - t0, world)
        e2e = {"value": round(e2e_s * 1e6 / (K * world), 3), "unit": UNIT, "h2d_bytes_per_step": 4,
               "d2h_bytes_per_step": 64}

    # launch-once serving through the C ABI: the grid stays resident, each step is one
    # mailbox round trip (token and pos in, next token and status out, pinned host memory)
    # (a profiler that runs each launch to completion before the host continues
    # cannot serve: the grid then leaves when idle and this measurement is skipped)
    e2e_serve = None
    if with_extras and not args.no_e2e and args.mode == "megakernel":
        from decode_persistent_block_b200 import MkError
        torch.cuda.synchronize()
        dec.serve_start()
        served = None
        try:
            tok = dec.serve_step(first, positions[0])
            barrier(world)
            t0 = time.perf_counter()
            for i in range(K):
                tok = dec.serve_step(tok, positions[i % len(positions)])
            t1 = time.perf_counter()
            served = t1 - t0
        except MkError as e:
            if e.name != "MK_ERR_STOPPED":
                raise
        finally:
            dec.serve_stop()
        st = dec.status()
        if st["code"] != 0:
            raise RuntimeError(f"device status after served steps: {st}")
        if served is not None:
            e2e_serve = {"value": round(reduce_max(served, world) * 1e6 / (K * world), 3), "unit": UNIT,
                         "h2d_bytes_per_step": 16, "d2h_bytes_per_step": 12,
                         "path": "mk_serve_step (resident grid, pinned mailbox)"}

    # speculative expert prediction (MoE): how many of the fused FFN's expert slots the prediction
    # named, over a few untimed steps (the getters synchronise)
    prediction = None
    if cfg.n_experts and args.mode == "megakernel" and dec.options.spec_experts:
        from decode_persistent_block_b200 import MkError
        try:
            hit = slots = 0
            tok = dec.step(first, positions[0])
            n = min(16, len(positions))
            for i in range(1, n):
                tok = dec.step(tok, positions[i])
                for l in range(cfg.n_layers):
                    pe, re_ = sorted(dec.predicted_experts(l).tolist()), sorted(dec.router(l)[0].tolist())
                    hit += sum(a == b for a, b in zip(pe, re_))
                    slots += len(pe)
            prediction = {"option": int(dec.options.spec_experts), "slots_hit": hit, "slots": slots,
                          "hit_rate": round(hit / max(slots, 1), 4), "steps": n - 1}
        except MkError:  # the kernel chosen for these options does not predict
            prediction = {"option": int(dec.options.spec_experts), "active": False}

    baselines = {}
    if not args.no_baselines and args.mode == "megakernel":
        for name, m in (("multi_kernel", 1), ("multi_kernel_graph", 2)):
            with Decoder(cfg, dW, dk, dv, mode=m) as b:
                kb = min(K, 128)
                tms, _ = timed(b, kb, 3)
                baselines[name] = round(reduce_max(tms, world) * 1000.0 / (kb * world), 3)
    dec.close()
    del dW, dk, dv
    torch.cuda.empty_cache()
    return {
        "value": round(us_per_token, 3), "tokens_per_s": round(1e6 / us_per_token, 1),
        "hbm_gbs": round(achieved, 1), "frac_of_8tbs": round(achieved / ROOFLINE_NOMINAL_GBS, 4),
        "floor_us_at_8tbs": round(byte_floor_us(bpt, ROOFLINE_NOMINAL_GBS), 1), "bytes_per_token": int(bpt),
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "peak_kind": f"{peak_kind} copy bandwidth",
                     "traffic": committed_traffic(cfg.name, args.mode), "launch_us": round(launch_ms * 1000, 2)},
        "e2e": e2e, "e2e_serve": e2e_serve, "baselines": baselines, "clocks": clk, "calib": calib,
        "steps": K, "warmup": Wm, "expert_prediction": prediction,
    }


def measure_batch(args, cfg, p0, B, K, Wm, world, local, dW=None):
    """Device-timed batched decode steps (B sequences per launch, each with its own cache and
    token, all at the same positions as the batch-1 workload); returns one `batch` entry.
    dW: the model's device weights, if already made."""
    import numpy as np
    import torch

    import synth
    from decode_persistent_block_b200 import Decoder, to_device
    torch.cuda.set_device(local)
    if dW is None:
        dW = to_device(synth.make_model(cfg))
    caches = [synth.make_kv_cache(cfg, stream=f".{b}") for b in range(B)]
    dk = torch.from_numpy(np.stack([c[0] for c in caches]).view(np.int16)).cuda()
    dv = torch.from_numpy(np.stack([c[1] for c in caches]).view(np.int16)).cuda()
    del caches
    first = [int(synth.prompt_tokens(cfg, stream=f".{b}")[0]) for b in range(B)]
    pos = [p0 + (i % cfg.steps) for i in range(max(K, Wm) + 1)]
    with Decoder(cfg, dW, dk, dv, batch=B) as dec:
        dec.step_batch(first, [pos[0]] * B)
        for i in range(1, Wm):
            dec.step_batch([-1] * B, [pos[i]] * B, sync=False)
        torch.cuda.synchronize()
        barrier(world)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for i in range(K):
            dec.step_batch([-1] * B, [pos[i % len(pos)]] * B, sync=False)
        e1.record()
        torch.cuda.synchronize()
        barrier(world)
        st = dec.status()
        if st["code"] != 0:
            raise RuntimeError(f"device status after batched steps: {st}")
    step_us = reduce_max(e0.elapsed_time(e1), world) * 1000.0 / K
    bpt = cfg.weight_bytes_per_token() + B * statistics.fmean(cfg.kv_bytes_per_token(q) for q in pos[:K])
    del dk, dv
    torch.cuda.empty_cache()
    return {"batch": B, "us_per_step": round(step_us, 1), "us_per_token": round(step_us / B, 2),
            "tokens_per_s": round(B * world * 1e6 / step_us, 1), "gb_per_step": round(bpt / 1e9, 4),
            "hbm_gbs": round(bpt / (step_us * 1e-6) / 1e9, 1), "steps": K, "warmup": Wm,
            "workload": f"{cfg.name}: {B} sequences per step, each with its own KV cache pre-filled to "
                        f"{cfg.prefill} and its own tokens, positions {p0}..{p0 + cfg.steps - 1}"}


def workload_name(cfg, p0):
    return (f"{cfg.name}: batch-1 greedy decode, KV pre-filled to {cfg.prefill}, positions "
            f"{p0}..{p0 + cfg.steps - 1}")


# The other target shape and the MoE shape, measured in the same run as the headline workload (fewer
# timed steps each: their steps are 2-3x longer), so every target config has a number in one bench line.
PER_CONFIG = (("llama3b", 384), ("mixtral8l", 256))


def run_ours(args, rank, world, local):
    from synth import configs
    cfg, p0, positions = workload(args)
    K, Wm = args.steps, args.warmup
    if args.batch_only > 1:  # a profiling run of the batched kernel alone
        b = measure_batch(args, cfg, p0, args.batch_only, K, Wm, world, local)
        return {"impl": "ours", "batched_only": b} if rank == 0 else None
    r = measure(args, cfg, p0, positions, K, Wm, rank, world, local)

    per_config = {}
    if args.per_config and not args.layers and args.config == "llama1b":
        for name, k in PER_CONFIG:
            c2 = configs.get(name)
            q0 = c2.prefill + c2.prompt_len
            pos2 = [q0 + (i % c2.steps) for i in range(max(k, Wm) + 1)]
            m = measure(args, c2, q0, pos2, min(k, K), Wm, rank, world, local, with_extras=False)
            per_config[name] = {"workload": workload_name(c2, q0), "value": m["value"], "unit": UNIT,
                                "tokens_per_s": m["tokens_per_s"], "roofline": m["roofline"],
                                "frac_of_8tbs": m["frac_of_8tbs"], "bytes_per_token": m["bytes_per_token"],
                                "e2e": m["e2e"], "baselines": m["baselines"], "clocks": m["clocks"],
                                "steps": m["steps"], "warmup": m["warmup"]}
            if m["expert_prediction"] is not None:
                per_config[name]["expert_prediction"] = m["expert_prediction"]

    batched = []
    if args.batch_sizes and not args.layers and args.mode == "megakernel" and not cfg.n_experts:
        import synth
        import torch
        from decode_persistent_block_b200 import MkError, to_device
        torch.cuda.set_device(local)
        dW = to_device(synth.make_model(cfg))  # one copy of the weights for every batch size
        for B in (int(x) for x in args.batch_sizes.split(",") if x):
            try:
                batched.append(measure_batch(args, cfg, p0, B, min(K, 256), Wm, world, local, dW))
            except MkError as e:  # no kernel for this batch size on this shape
                batched.append({"batch": B, "unsupported": e.name})
        del dW
        torch.cuda.empty_cache()

    cpu = None
    if rank == 0 and not args.no_cpu_baseline:
        times, cores = oracle_steps(cfg, args.cpu_seconds)
        cpu = {"value": round(statistics.fmean(times) * 1e6, 1), "unit": UNIT, "cores": cores, "kind": "oracle",
               "sample": f"{len(times)} fp64 oracle decode steps of {cfg.name} at positions {p0}..",
               "ms_per_token": round(statistics.fmean(times) * 1e3, 2)}
        single = single_thread_oracle_ms(args)
        if single is not None:
            cpu["single_thread_ms_per_token"] = single

    if rank != 0:
        return None
    line = {
        "metric": METRIC, "value": r["value"], "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": Wm, "ms_per_step": round(r["value"] * world / 1000.0, 6), "higher_is_better": False,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16 weights/KV, fp32 accumulate",
        "data": "synthetic random-init weights and KV prefill (seeded generator)",
        "config": {"workload": workload_name(cfg, p0), "layers": cfg.n_layers, "hidden": cfg.hidden,
                   "vocab": cfg.vocab, "mode": args.mode, "parallelism": f"replicas x{world}",
                   "l2": f"no flush: {r['bytes_per_token'] / 1e9:.2f} GB streamed per token > 126 MB L2",
                   "sm_speed": r["calib"] or "equal"},
        "tokens_per_s": r["tokens_per_s"],
        "hbm_gbs": r["hbm_gbs"],
        "frac_of_8tbs": r["frac_of_8tbs"],
        "floor_us_at_8tbs": r["floor_us_at_8tbs"],
        "bytes_per_token": r["bytes_per_token"],
        "roofline": r["roofline"],
        "e2e": r["e2e"],
        "e2e_serve": r["e2e_serve"],
        "gpu_launches": K if args.mode == "megakernel" else None,
        "baselines": r["baselines"],
        "per_config": per_config or None,
        "batched": batched or None,
        "expert_prediction": r["expert_prediction"],
        "cpu_baseline": cpu,
        "clocks": r["clocks"],
    }
    if args.mode != "megakernel":
        per_step = 6 * cfg.n_layers + 3 + (cfg.n_layers * cfg.top_k if cfg.n_experts else 0)
        line["gpu_launches"] = K * (per_step + 1)
    return line


# ---- reference arm: the fp64 oracle on the host cores ---------------------------------------------------

REFERENCE_SECONDS = 90.0  # bound on the reference arm's timed oracle work


def run_reference(args, rank, world):
    """The fp64 oracle on the host cores, rank 0 only: W warm-up steps (at most
    one), then up to K timed decode steps, stopping early once about
    REFERENCE_SECONDS of oracle work is done (each step is one whole decode step
    of the workload; the sample says how many were timed)."""
    if rank != 0:
        return None
    cfg, p0, positions = workload(args)
    warm = min(args.warmup, 1)
    times, cores = oracle_steps(cfg, REFERENCE_SECONDS, max_steps=warm + args.steps, min_steps=warm + 2)
    t = times[warm:]
    v = statistics.fmean(t) * 1e6
    sample = (f"{len(t)} of the {args.steps} requested fp64 oracle decode steps of {cfg.name} at positions "
              f"{p0}.. (bounded to about {REFERENCE_SECONDS:.0f} s), after {warm} warm-up")
    return {"impl": "reference", "metric": METRIC, "value": round(v, 1), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(v / 1000.0, 3),
            "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic random-init weights and KV prefill (seeded generator)",
            "config": {"workload": f"{cfg.name}: batch-1 greedy decode, KV pre-filled to {cfg.prefill}, positions "
                                   f"{p0}..{p0 + cfg.steps - 1}", "layers": cfg.n_layers, "hidden": cfg.hidden,
                       "vocab": cfg.vocab, "mode": "fp64 CPU oracle"},
            "cpu_baseline": {"value": round(v, 1), "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": round(v, 1), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    args = parse()
    rank, world, local = dist_setup()
    try:
        if args.impl == "reference":
            line = run_reference(args, rank, world)
        else:
            line = run_ours(args, rank, world, local)
        if line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
