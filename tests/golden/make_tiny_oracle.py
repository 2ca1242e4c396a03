"""Writes tiny_oracle_steps.txt: the fp64 oracle's greedy decode of the tiny
Llama-style workload (2 layers, hidden 256, 4 query / 2 KV heads, head_dim 64,
FFN 768, vocab 4096, seed 0; a 16-token random prompt, then 8 greedy steps).

Only the oracle and the seeded input generators are used.  The file pins the
oracle against unintended changes: `tests/test_golden.py` re-runs the same
decode and compares.  Run from the repository root:
    python tests/golden/make_tiny_oracle.py
"""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
import synth  # noqa: E402
from synth import configs  # noqa: E402

OUT = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_oracle_steps.txt")


def decode_tiny():
    """Rows (pos, token_in, next, top1_top2_margin, logit[0], logit[next], |x_L|_2)."""
    cfg = configs.TINY
    w = synth.make_model(cfg)
    kc, vc = synth.make_kv_cache(cfg)
    m = oracle.Model(cfg, w, kc, vc)
    prompt = synth.prompt_tokens(cfg)
    rows, prev = [], None
    for pos in range(cfg.prompt_len + cfg.steps):
        tok = int(prompt[pos]) if pos < cfg.prompt_len else prev
        r = m.step(tok, pos)
        lg = r["logits"]
        top2 = np.sort(lg)[-2:]
        rows.append((pos, tok, int(r["next"]), float(top2[1] - top2[0]), float(lg[0]), float(lg[r["next"]]),
                     float(np.linalg.norm(r["hidden"][-1]))))
        prev = int(r["next"])
    return rows


def main():
    rows = decode_tiny()
    with open(OUT, "w") as f:
        f.write("# fp64 oracle, tiny workload (seed 0): written by tests/golden/make_tiny_oracle.py\n")
        f.write("# pos token_in next margin logit0 logit_next norm_x_final\n")
        for r in rows:
            f.write(f"{r[0]} {r[1]} {r[2]} {r[3]:.12e} {r[4]:.12e} {r[5]:.12e} {r[6]:.12e}\n")


if __name__ == "__main__":
    main()
