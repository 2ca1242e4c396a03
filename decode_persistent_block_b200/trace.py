"""Per-instruction device trace (`mk_options.trace = 1`): per-op latency
breakdown and per-SM spread.

`Decoder.trace()` returns, for the last step, eight globaltimer stamps (ns, 0 =
not reached) per instruction of the schedule [n_sm][max_instr]:
  0 reached, 1 dependency met, 2 input vector ready, 3 first stage full,
  4 main stages consumed, 5 done and signalled (consumer warps);
  6 first stage issued, 7 last stage issued (loader warp).

Records of 32 words add, for each instruction's first 8 ring stages, consumer
thread 0's full-barrier wait returned (8 + s), its share of the stage consumed
(16 + s) and the loader's issue (24 + s); `stage_breakdown` reduces those.

`op_breakdown` reduces them to the phases of each op, averaged over layers:
  phase   previous op's last end -> this op's last end (the op's share of the step)
  hop     previous op's last end -> dependency met (mean over blocks)
  ready   dependency met -> input vector ready
  first   -> first stage full
  main    first stage -> main stages consumed
  epi     -> done and signalled
  spread  last end - first end across the op's blocks
  ld_lead loader's first issue -> dependency met (how far the loader ran ahead)
  ld_last dependency met -> loader's last issue

Command line (on a GPU):
  python -m decode_persistent_block_b200.trace llama1b [--steps 4] [--npz out.npz] [key=value options]
"""
from __future__ import annotations

import numpy as np

OP_NAMES = {1: "QKV", 2: "ATTN", 3: "OPROJ", 4: "UG", 5: "DOWN", 6: "LM", 7: "MOE_UG", 8: "MOE_DOWN", 9: "FFN",
            10: "MOE_FFN"}
ORDER = ["QKV", "ATTN", "OPROJ", "UG", "DOWN", "FFN", "MOE_UG", "MOE_DOWN", "MOE_FFN", "LM"]
COLUMNS = ["phase", "hop", "ready", "first", "main", "epi", "spread", "ld_lead", "ld_last"]
T_START, T_DEP, T_READY, T_FIRST, T_MAIN, T_END, T_LD_FIRST, T_LD_LAST = range(8)
N_STAGES = 8
T_SREADY, T_SDONE, T_SISSUE = 8, 8 + N_STAGES, 8 + 2 * N_STAGES


def _groups(schedule: np.ndarray, trace: np.ndarray):
    """{(layer, op name): array [blocks, 8] of stamps in µs from the step's first stamp (nan = not reached)}."""
    tr = trace.reshape(schedule.shape[0], schedule.shape[1], -1).astype(np.int64)
    reached = tr[:, :, T_START][tr[:, :, T_START] > 0]
    if reached.size == 0:
        return {}
    t0 = reached.min()
    out = {}
    for sm in range(schedule.shape[0]):
        for i in range(schedule.shape[1]):
            op = int(schedule[sm, i, 0])
            if op == 0:
                continue
            out.setdefault((int(schedule[sm, i, 1]), OP_NAMES.get(op, str(op))), []).append(tr[sm, i])
    return {k: np.where(np.array(v) > 0, (np.array(v) - t0) / 1000.0, np.nan) for k, v in out.items()}


def op_breakdown(schedule: np.ndarray, trace: np.ndarray) -> dict:
    """{op name: {column: mean µs over the layers}} in step order (see the module doc)."""
    g = _groups(schedule, trace)
    keys = sorted(g, key=lambda k: (k[0], np.nanmin(g[k][:, T_START])))
    agg: dict = {}
    prev_end = None
    for key in keys:
        a = g[key]
        end_max = np.nanmax(a[:, T_END])
        row = {
            "phase": end_max - prev_end if prev_end is not None else np.nan,
            "hop": np.nanmean(a[:, T_DEP] - prev_end) if prev_end is not None else np.nan,
            "ready": np.nanmean(a[:, T_READY] - a[:, T_DEP]),
            "first": np.nanmean(a[:, T_FIRST] - np.fmax(a[:, T_READY], a[:, T_DEP])),
            "main": np.nanmean(a[:, T_MAIN] - a[:, T_FIRST]),
            "epi": np.nanmean(a[:, T_END] - a[:, T_MAIN]),
            "spread": end_max - np.nanmin(a[:, T_END]),
            "ld_lead": np.nanmean(a[:, T_DEP] - a[:, T_LD_FIRST]),
            "ld_last": np.nanmean(a[:, T_LD_LAST] - a[:, T_DEP]),
        }
        prev_end = end_max
        agg.setdefault(key[1], []).append(row)
    return {op: {c: _mean([r[c] for r in agg[op]]) for c in COLUMNS} for op in ORDER if op in agg}


def stage_breakdown(schedule: np.ndarray, trace: np.ndarray, n_stages: int = 4) -> dict:
    """{op name: [n_stages][3] mean µs over blocks and layers} from the per-stage stamps:
    wait (previous stage consumed, or the input vector ready, -> this stage's wait returned),
    consume (wait returned -> consumed) and lead (loader issue -> wait returned)."""
    g = _groups(schedule, trace)
    acc: dict = {}
    for (layer, op), a in g.items():
        if a.shape[1] < T_SISSUE + N_STAGES:
            return {}
        rows = []
        for s in range(n_stages):
            prev = a[:, T_SDONE + s - 1] if s > 0 else np.fmax(a[:, T_READY], a[:, T_DEP])
            rows.append([a[:, T_SREADY + s] - prev, a[:, T_SDONE + s] - a[:, T_SREADY + s],
                         a[:, T_SREADY + s] - a[:, T_SISSUE + s]])
        acc.setdefault(op, []).append(np.array(rows))  # [stages][3][blocks]
    out = {}
    for op in ORDER:
        if op in acc:
            cat = np.concatenate(acc[op], axis=2)
            with np.errstate(all="ignore"):
                out[op] = [[_mean(cat[s, k]) for k in range(3)] for s in range(n_stages)]
    return out


def format_stages(sb: dict) -> str:
    if not sb:
        return ""
    n = len(next(iter(sb.values())))
    lines = [f"{'op':8s} " + " ".join(f"{'s%d wait/cons/lead' % s:>20s}" for s in range(n))]
    for op, st in sb.items():
        lines.append(f"{op:8s} " + " ".join(f"{w:6.2f}/{c:5.2f}/{l:6.2f} " for w, c, l in st))
    return "\n".join(lines)


def _mean(xs) -> float:
    a = np.asarray(xs, dtype=np.float64)
    a = a[~np.isnan(a)]
    return float(a.mean()) if a.size else float("nan")


def per_sm_duration(schedule: np.ndarray, trace: np.ndarray, op_name: str, n_layers: int) -> np.ndarray:
    """[n_sm, n_layers] dependency-met -> done µs of `op_name` (nan where the block has none)."""
    tr = trace.reshape(schedule.shape[0], schedule.shape[1], -1).astype(np.int64)
    out = np.full((schedule.shape[0], max(n_layers, 1)), np.nan)
    for sm in range(schedule.shape[0]):
        for i in range(schedule.shape[1]):
            if OP_NAMES.get(int(schedule[sm, i, 0])) == op_name:
                l = int(schedule[sm, i, 1])
                if 0 <= l < out.shape[1] and tr[sm, i, T_DEP] > 0 and tr[sm, i, T_END] > 0:
                    out[sm, l] = (tr[sm, i, T_END] - tr[sm, i, T_DEP]) / 1000.0
    return out


def layer_timeline(schedule: np.ndarray, trace: np.ndarray, layer: int) -> str:
    """Per op of one layer, µs from the layer's first QKV dependency: first start, first and last
    dependency met, first and last end (the op's blocks)."""
    g = _groups(schedule, trace)
    keys = [k for k in g if k[0] == layer]
    if not keys:
        return ""
    q = g.get((layer, "QKV"))
    t0 = np.nanmin(q[:, T_DEP]) if q is not None else min(np.nanmin(g[k][:, T_START]) for k in keys)
    lines = [f"layer {layer}: {'op':8s} {'start0':>8s} {'dep0':>8s} {'dep1':>8s} {'end0':>8s} {'end1':>8s} {'blocks':>6s}"]
    for k in sorted(keys, key=lambda k: np.nanmin(g[k][:, T_START])):
        a = g[k]
        lines.append(f"         {k[1]:8s} " + " ".join(f"{v - t0:8.2f}" for v in (
            np.nanmin(a[:, T_START]), np.nanmin(a[:, T_DEP]), np.nanmax(a[:, T_DEP]), np.nanmin(a[:, T_END]),
            np.nanmax(a[:, T_END]))) + f" {a.shape[0]:6d}")
    return "\n".join(lines)


def format_breakdown(bd: dict) -> str:
    lines = [f"{'op':8s} " + " ".join(f"{c:>8s}" for c in COLUMNS)]
    for op, row in bd.items():
        lines.append(f"{op:8s} " + " ".join(f"{row[c]:8.2f}" for c in COLUMNS))
    return "\n".join(lines)


def main(argv=None) -> None:
    import argparse
    import os
    import sys

    import torch

    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import synth
    from synth import configs

    from .mk import Decoder, to_device

    ap = argparse.ArgumentParser(description="per-op latency breakdown from the device trace")
    ap.add_argument("config")
    ap.add_argument("--steps", type=int, default=4)
    ap.add_argument("--npz", default="")
    ap.add_argument("--batch", type=int, default=1, help="sequences per step (batched decode)")
    ap.add_argument("options", nargs="*", help="mk_options fields as key=value (integers)")
    args = ap.parse_intermixed_args(argv)
    cfg = configs.get(args.config)
    opts = {k: int(v) for k, v in (kv.split("=") for kv in args.options)}
    W = synth.make_model(cfg)
    B = args.batch
    caches = [synth.make_kv_cache(cfg, stream=f".{b}" if b else "") for b in range(B)]
    stack = (lambda a: a[0]) if B == 1 else np.stack
    dk = torch.from_numpy(stack([c[0] for c in caches]).view(np.int16)).cuda()
    dv = torch.from_numpy(stack([c[1] for c in caches]).view(np.int16)).cuda()
    p0 = cfg.prefill + cfg.prompt_len
    if B > 1:
        opts["batch"] = B
    with Decoder(cfg, to_device(W), dk, dv, trace=1, **opts) as dec:
        if B == 1:
            tok = dec.step(int(synth.prompt_tokens(cfg)[0]), p0)
            for i in range(1, args.steps):
                tok = dec.step(tok, p0 + i)
        else:
            toks = dec.step_batch([int(synth.prompt_tokens(cfg, stream=f".{b}")[0]) for b in range(B)], [p0] * B)
            for i in range(1, args.steps):
                toks = dec.step_batch(toks, [p0 + i] * B)
        sched, tr = dec.schedule(), dec.trace()
        print(f"{cfg.name}: last step {dec.last_step_ns() / 1000:.1f} us (traced)")
    print(format_breakdown(op_breakdown(sched, tr)))
    print(format_stages(stage_breakdown(sched, tr)))
    for layer in sorted({0, cfg.n_layers // 2, cfg.n_layers - 1}):
        if cfg.n_layers:
            print(layer_timeline(sched, tr, layer))
    present = {OP_NAMES.get(int(o)) for o in np.unique(sched[:, :, 0])}
    big = next((n for n in ("FFN", "MOE_FFN", "UG", "MOE_UG") if n in present), "LM")
    d = per_sm_duration(sched, tr, big, cfg.n_layers)
    mean = np.nanmean(d, axis=1)
    print(f"{big} dependency->done per SM: mean {np.nanmean(mean):.2f} min {np.nanmin(mean):.2f} "
          f"max {np.nanmax(mean):.2f} us; even/odd-layer correlation "
          f"{np.corrcoef(np.nanmean(d[:, 0::2], 1), np.nanmean(d[:, 1::2], 1))[0, 1]:.2f}")
    if args.npz:
        np.savez(args.npz, schedule=sched, trace=tr.reshape(sched.shape[0], sched.shape[1], -1))


if __name__ == "__main__":
    main()
