"""Launch-once serving (mk_serve_*): the resident grid gives the same steps as
one launch per step, leaves on request or when idle, and the per-launch path
continues afterwards.

The serving grid occupies its handle's stream, so each test gives the decoder
a stream of its own and reads logits on the default stream.
"""
import time

import numpy as np
import pytest

from synth import configs
from tests import parity

pytestmark = pytest.mark.gpu

IDLE = 5_000_000_000  # a grid left behind by a failing test leaves after 5 s


@pytest.fixture(scope="module")
def tiny(cuda):
    return parity.Setup(configs.TINY)


def _steps(tiny, n=None):
    return parity.schedule(configs.TINY, n)


def _per_launch(tiny, **opts):
    import torch
    tiny.fresh_caches()
    lg = torch.empty(configs.TINY.vocab, device="cuda")
    toks, logits = [], []
    with tiny.decoder(**opts) as dec:
        nxt = None
        for pos, tok in _steps(tiny):
            nxt = dec.step(tok if tok is not None else nxt, pos, logits=lg)
            toks.append(nxt)
            logits.append(lg.cpu().numpy().copy())
    return toks, logits


def _served(tiny, **opts):
    import torch
    from decode_persistent_block_b200 import Decoder
    tiny.fresh_caches()
    torch.cuda.synchronize()
    lg = torch.empty(configs.TINY.vocab, device="cuda")
    s = torch.cuda.Stream()
    toks, logits = [], []
    dec = Decoder(configs.TINY, tiny.dW, tiny.dk, tiny.dv, stream=s, serve_idle_ns=IDLE, **opts)
    try:
        dec.serve_start(lg)
        nxt = None
        for pos, tok in _steps(tiny):
            nxt = dec.serve_step(tok if tok is not None else nxt, pos)
            toks.append(nxt)
            logits.append(lg.cpu().numpy().copy())  # default stream: runs beside the resident grid
        dec.serve_stop()
        assert dec.status()["code"] == 0
    finally:
        dec.close()
    return toks, logits


@pytest.mark.parametrize("attn_merge", [1, 2], ids=["merge_in_oproj", "merge_once"])
def test_served_steps_equal_per_launch_steps_bitwise(tiny, attn_merge):
    # split FFN: every sum has a fixed order (the once-per-head merge too, whichever split does it),
    # so the two paths agree bit for bit
    t1, l1 = _per_launch(tiny, split_ffn=1, attn_merge=attn_merge)
    t2, l2 = _served(tiny, split_ffn=1, attn_merge=attn_merge)
    assert t1 == t2
    for a, b in zip(l1, l2):
        assert np.array_equal(a, b)


def test_served_steps_default_options(tiny):
    t1, l1 = _per_launch(tiny)
    t2, l2 = _served(tiny)
    assert t1 == t2
    for a, b in zip(l1, l2):
        np.testing.assert_allclose(a, b, rtol=1e-4, atol=1e-4)


@pytest.mark.parametrize("spec", [0, 1, 2], ids=["no_spec", "spec", "spec_miss"])
def test_serve_moe(cuda, spec):
    # the resident grid carries the speculative expert prediction across its served steps
    cfg = configs.TINY.with_(name="tiny_moe4_2", n_experts=4, top_k=2)
    setup = parity.Setup(cfg)
    import torch
    from decode_persistent_block_b200 import Decoder
    ref = []
    setup.fresh_caches()
    with setup.decoder(spec_experts=spec) as dec:
        nxt = None
        for pos, tok in parity.schedule(cfg):
            nxt = dec.step(tok if tok is not None else nxt, pos)
            ref.append(nxt)
    setup.fresh_caches()
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    dec = Decoder(cfg, setup.dW, setup.dk, setup.dv, stream=s, serve_idle_ns=IDLE, spec_experts=spec)
    try:
        dec.serve_start()
        got, nxt = [], None
        for pos, tok in parity.schedule(cfg):
            nxt = dec.serve_step(tok if tok is not None else nxt, pos)
            got.append(nxt)
        dec.serve_stop()
    finally:
        dec.close()
    assert got == ref


def test_device_feed_stop_restart_and_per_launch_after(tiny):
    import torch
    from decode_persistent_block_b200 import Decoder, MkError
    tiny.fresh_caches()
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    dec = Decoder(configs.TINY, tiny.dW, tiny.dk, tiny.dv, stream=s, split_ffn=1, serve_idle_ns=IDLE)
    try:
        dec.serve_start()
        a = dec.serve_step(5, 0)
        b = dec.serve_step(-1, 1)  # previous argmax, fed on the device
        with pytest.raises(MkError) as e:
            dec.step(3, 2)  # the per-launch path is closed while serving
        assert e.value.name == "MK_ERR_INVALID_ARG"
        dec.serve_stop()
        c = dec.step(-1, 2)  # per-launch continues the same sequence
        dec.serve_start()
        d = dec.serve_step(-1, 3)
        dec.serve_stop()
        assert (dec.counters() == 4 * dec.counter_increments().astype(np.uint64)).all()
    finally:
        dec.close()
    # the same four steps, one launch each
    tiny.fresh_caches()
    with tiny.decoder(split_ffn=1) as ref:
        assert [ref.step(5, 0), ref.step(-1, 1), ref.step(-1, 2), ref.step(-1, 3)] == [a, b, c, d]


def test_idle_grid_leaves_by_itself(tiny):
    import torch
    from decode_persistent_block_b200 import Decoder, MkError
    tiny.fresh_caches()
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    dec = Decoder(configs.TINY, tiny.dW, tiny.dk, tiny.dv, stream=s, serve_idle_ns=200_000_000)
    try:
        dec.serve_start()
        dec.serve_step(7, 0)
        time.sleep(1.0)  # longer than the idle limit: the grid has left
        with pytest.raises(MkError) as e:
            dec.serve_step(-1, 1)
        assert e.value.name == "MK_ERR_STOPPED"
        assert dec.status()["code"] == 0  # an idle exit is not an error
        dec.step(-1, 1)  # the per-launch path works again
    finally:
        dec.close()


def _served_vs_oracle(setup, steps=None, **opts):
    """Teacher-forced launch-once serving against the fp64 oracle: every served
    step's logits and token, then (after the grid has left) the last step's
    per-layer hidden states."""
    import torch
    from decode_persistent_block_b200 import Decoder
    cfg = setup.cfg
    orc = setup.oracle()
    setup.fresh_caches()
    torch.cuda.synchronize()
    lg = torch.empty(cfg.vocab, device="cuda")
    s = torch.cuda.Stream()
    reports = []
    dec = Decoder(cfg, setup.dW, setup.dk, setup.dv, stream=s, serve_idle_ns=IDLE, snapshots=1, **opts)
    try:
        dec.serve_start(lg)
        nxt = None
        for pos, tok in parity.schedule(cfg, steps):
            t = tok if tok is not None else nxt
            got = dec.serve_step(t, pos)
            o = orc.step(t, pos)
            lo = o["logits"]
            srt = np.sort(lo)
            reports.append({"logit_err": float(np.max(np.abs(lg.cpu().numpy().astype(np.float64) - lo))),
                            "margin": float(srt[-1] - srt[-2]), "next_orc": o["next"], "next_gpu": got, "pos": pos})
            nxt = o["next"]
        dec.serve_stop()
        assert dec.status()["code"] == 0
        hg = dec.hidden_all().astype(np.float64)
        ho = o["hidden"]
        reports[-1]["hidden_rel"] = (np.linalg.norm(hg - ho, axis=1) /
                                     np.maximum(np.linalg.norm(ho, axis=1), 1e-30)).tolist()
    finally:
        dec.close()
    return reports


@pytest.mark.parametrize("opts", [dict(split_ffn=0), dict(split_ffn=1), dict(attn_merge=2),
                                  dict(ffn_early_stages=1, n_sm=7)],
                         ids=["fused_ffn", "split_ffn", "merge_once", "ffn_gate"])
def test_served_steps_match_oracle_tiny(tiny, opts):
    reps = _served_vs_oracle(tiny, **opts)
    assert len(reps) == configs.TINY.prompt_len + configs.TINY.steps
    parity.assert_parity(reps)


def test_served_steps_match_oracle_llama1b(cuda):
    # the full-size shape in the benchmark's launch configuration (default options), 3 positions
    reps = _served_vs_oracle(parity.Setup(configs.LLAMA_1B), steps=3)
    parity.assert_parity(reps)
