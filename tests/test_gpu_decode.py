"""GPU parity of the decode step (through the C ABI) against the fp64 oracle.

Small configs run every step of their workload on both execution modes; the
full-size configs (Llama-1B/3B shapes, the KV-length sweep, Mixtral-shaped
MoE) run a teacher-forced subset of their decode positions in the same launch
configuration the benchmark times (set MK_FULL_PARITY=1 for every step).
"""
import os

import numpy as np
import pytest

from synth import configs
from tests import parity

pytestmark = pytest.mark.gpu

FULL = os.environ.get("MK_FULL_PARITY") == "1"
MODES = {"megakernel": 0, "multi_kernel": 1, "multi_kernel_graph": 2}


@pytest.fixture(scope="module")
def tiny(cuda):
    return parity.Setup(configs.TINY)


@pytest.mark.parametrize("mode", list(MODES))
def test_tiny_all_steps(tiny, mode):
    reps = parity.run(tiny, mode=MODES[mode])
    assert len(reps) == configs.TINY.prompt_len + configs.TINY.steps
    h, l = parity.assert_parity(reps)
    assert h < 1e-4 and l < 1e-3  # fp32 vs fp64 on identical bf16 bytes: far inside the bar


@pytest.mark.parametrize("opts", [
    dict(n_sm=7), dict(n_sm=1), dict(kv_splits=1), dict(kv_splits=40), dict(ring_stages=2),
    dict(stage_bytes=4096), dict(stage_bytes=4096, ring_stages=3, l2_prefetch=16384), dict(rows_per_instr=3),
    dict(l2_prefetch=65536), dict(split_ffn=1), dict(split_ffn=1, n_sm=7),
    dict(attn_merge=2), dict(attn_merge=2, n_sm=7), dict(attn_merge=2, n_sm=1), dict(attn_merge=2, kv_splits=1),
    dict(attn_merge=2, kv_splits=40), dict(attn_merge=2, split_ffn=1), dict(attn_merge=2, general_kernel=1),
    dict(ffn_early_stages=1, n_sm=7), dict(ffn_early_stages=1, stage_bytes=4096),
    dict(ffn_early_stages=3, stage_bytes=4096, ring_stages=4), dict(ffn_early_stages=1, n_sm=7, general_kernel=1),
], ids=lambda o: ",".join(f"{k}={v}" for k, v in o.items()))
def test_tiny_schedule_options(tiny, opts):
    parity.assert_parity(parity.run(tiny, **opts))


@pytest.mark.parametrize("E,k", [(4, 2), (2, 1), (8, 2)])
@pytest.mark.parametrize("mode", ["megakernel", "megakernel_split_ffn", "multi_kernel"])
def test_tiny_moe(cuda, E, k, mode):
    cfg = configs.TINY.with_(name=f"tiny_moe{E}_{k}", n_experts=E, top_k=k)
    split = mode == "megakernel_split_ffn"
    parity.assert_parity(parity.run(parity.Setup(cfg), mode=MODES["megakernel" if split else mode],
                                    split_ffn=int(split)), cfg)


def test_no_layers_is_lm_head_of_embedding(cuda):
    cfg = configs.TINY.with_(n_layers=0, steps=2)
    parity.assert_parity(parity.run(parity.Setup(cfg)))


@pytest.mark.parametrize("attn_merge", [1, 2], ids=["merge_in_oproj", "merge_once"])
def test_head_dim_128_group_3(cuda, attn_merge):
    cfg = configs.TINY.with_(name="tiny_d128", n_heads=6, n_kv_heads=2, head_dim=128, hidden=384, ffn=1024)
    parity.assert_parity(parity.run(parity.Setup(cfg), attn_merge=attn_merge))


def test_group_1_and_wide_rows(cuda):
    # n_heads == n_kv_heads, and an ffn wider than 8192 columns (column-part phases)
    cfg = configs.TINY.with_(name="tiny_wide", n_heads=2, n_kv_heads=2, ffn=9216, steps=3)
    setup = parity.Setup(cfg)
    for mode, split in ((0, 0), (0, 1), (1, 0)):
        parity.assert_parity(parity.run(setup, mode=mode, split_ffn=split))


@pytest.mark.parametrize("attn_merge", [1, 2], ids=["merge_in_oproj", "merge_once"])
def test_counters_are_exact_multiples_after_steps(tiny, attn_merge):
    tiny.fresh_caches()
    with tiny.decoder(attn_merge=attn_merge) as dec:
        inc = dec.counter_increments()
        for s, (pos, tok) in enumerate(parity.schedule(configs.TINY)):
            dec.step(tok if tok is not None else 1, pos)
            assert np.array_equal(dec.counters(), (s + 1) * inc.astype(np.uint64)), s
        dec.reset()
        assert not dec.counters().any()


def _repeat(tiny, n, **opts):
    import torch
    outs = []
    for _ in range(n):
        tiny.fresh_caches()
        lg = torch.empty(configs.TINY.vocab, device="cuda")
        with tiny.decoder(**opts) as dec:
            for pos, tok in parity.schedule(configs.TINY, 20):
                dec.step(tok if tok is not None else 7, pos, logits=lg)
            outs.append((lg.cpu().numpy().copy(), tiny.dk.cpu().numpy().copy()))
    return outs


@pytest.mark.parametrize("attn_merge", [1, 2], ids=["merge_in_oproj", "merge_once"])
def test_determinism_bitwise(tiny, attn_merge):
    # split FFN: every sum has a fixed order (the once-per-head merge reads the splits in order,
    # whichever split runs it), so repeated runs agree bit for bit
    outs = _repeat(tiny, 2, split_ffn=1, attn_merge=attn_merge)
    assert np.array_equal(outs[0][0], outs[1][0]) and np.array_equal(outs[0][1], outs[1][1])


def test_fused_ffn_runs_agree_within_fp32_reordering(tiny):
    # fused FFN: the down-projection partials of all blocks meet in fp32 atomics,
    # so only the summation order differs between runs
    outs = _repeat(tiny, 3)
    for o in outs[1:]:
        np.testing.assert_allclose(o[0], outs[0][0], rtol=1e-4, atol=1e-4)
        a = (o[1].view(np.uint16).astype(np.uint32) << 16).view(np.float32)
        b = (outs[0][1].view(np.uint16).astype(np.uint32) << 16).view(np.float32)
        assert np.all(np.abs(a - b) <= np.abs(b) * 2.0 ** -7 + 1e-6)


@pytest.mark.parametrize("split_ffn", [1, 0], ids=["split_ffn", "fused_ffn"])
def test_on_device_token_feed_matches_host_feed(tiny, split_ffn):
    import torch
    res = []
    for feed in ("host", "device"):
        tiny.fresh_caches()
        lg = torch.empty(configs.TINY.vocab, device="cuda")
        with tiny.decoder(split_ffn=split_ffn) as dec:
            nxt = dec.step(5, 0)
            for pos in range(1, 6):
                if feed == "host":
                    nxt = dec.step(nxt, pos, logits=lg)
                else:
                    dec.step(-1, pos, logits=lg, sync=False)
            res.append(lg.cpu().numpy().copy())
    if split_ffn:
        assert np.array_equal(res[0], res[1])
    else:  # same tokens fed; only the fp32 order of the FFN's atomic sums differs
        np.testing.assert_allclose(res[0], res[1], rtol=1e-4, atol=1e-4)


def test_kv_append_matches_oracle_cache(tiny):
    orc = tiny.oracle()
    reps = parity.run(tiny, orc=orc)
    parity.assert_parity(reps)
    g = tiny.dk.cpu().numpy().view(np.uint16)
    o = orc.k
    n = configs.TINY.prompt_len + configs.TINY.steps
    a = (g[:, :, :n].astype(np.uint32) << 16).view(np.float32)
    b = (o[:, :, :n].astype(np.uint32) << 16).view(np.float32)
    # identical bf16 bits except where the fp32 value and the fp64 one round to neighbouring bf16
    # values (one ulp), or where k is the small remainder of a cancelling dot product, whose
    # fp32 error is small against the layer's largest |k| but not against k itself
    atol = 1e-4 * np.abs(b).max(axis=(1, 2, 3), keepdims=True)
    bound = np.abs(b) * 2.0 ** -7 + atol
    ratio = np.abs(a - b) / bound
    worst = np.argsort(ratio, axis=None)[-3:]
    detail = [(np.unravel_index(i, a.shape), float(a.flat[i]), float(b.flat[i])) for i in worst]
    assert np.all(ratio <= 1.0), detail
    assert np.mean(a == b) > 0.99


def test_argument_errors(tiny):
    from decode_persistent_block_b200 import MkError
    with tiny.decoder() as dec:
        for tok, pos in ((configs.TINY.vocab, 0), (0, configs.TINY.max_seq), (0, -1)):
            with pytest.raises(MkError) as e:
                dec.step(tok, pos)
            assert e.value.name == "MK_ERR_INVALID_ARG"
        with pytest.raises(MkError):
            dec.router(0)  # dense model


# ---- full-size configs -----------------------------------------------------------------

def _full(cfg, steps, mode=0, **opts):
    s = parity.Setup(cfg)
    reps = parity.run(s, steps=None if FULL else steps, mode=mode, **opts)
    h, l = parity.assert_parity(reps, cfg)
    return reps


def test_llama1b(cuda):
    _full(configs.LLAMA_1B, 4)


def test_llama1b_calibrated_sm_speed(cuda):
    # FFN and LM-head rows split by the per-SM speed measured on this GPU: same bar
    from decode_persistent_block_b200.calibrate import measure_sm_speed
    cfg = configs.LLAMA_1B
    s = parity.Setup(cfg)
    p0 = cfg.prefill + cfg.prompt_len
    speed = measure_sm_speed(cfg, s.dW, s.dk, s.dv, int(parity.synth.prompt_tokens(cfg)[0]), p0, steps=3)
    assert np.all(np.isfinite(speed)) and abs(speed.mean() - 1.0) < 0.05 and speed.min() >= 0.5
    reps = parity.run(s, steps=None if FULL else 3, sm_speed=speed)
    parity.assert_parity(reps, cfg)


def test_tiny_skewed_sm_speed(tiny):
    import torch
    n = torch.cuda.get_device_properties(0).multi_processor_count
    parity.assert_parity(parity.run(tiny, sm_speed=np.linspace(0.5, 1.5, n)))


def test_llama1b_split_ffn(cuda):
    _full(configs.LLAMA_1B, 2, split_ffn=1)


def test_llama1b_multi_kernel(cuda):
    _full(configs.LLAMA_1B, 2, mode=1)


def test_llama3b(cuda):
    _full(configs.LLAMA_3B, 3)  # the attention splits merged once per kv head (204 KB of partials)


def test_llama3b_merge_in_oproj(cuda):
    _full(configs.LLAMA_3B, 2, attn_merge=1)


def test_llama1b_merge_once(cuda):
    # the head_dim-64 tensor-core attention with the once-per-head merge
    _full(configs.LLAMA_1B, 2, attn_merge=2)


@pytest.mark.parametrize("prefill", configs.LONG_PREFILLS)
def test_llama1b_long_context(cuda, prefill):
    _full(configs.llama1b_sweep(prefill), 2)


@pytest.mark.parametrize("prefill", configs.SWEEP_PREFILLS)
def test_llama1b_kv_sweep(cuda, prefill):
    _full(configs.llama1b_sweep(prefill), 2)


def test_mixtral8l(cuda):
    _full(configs.MIXTRAL_8L, 3)


# ---- speculative expert prediction ------------------------------------------------

def _pred_stats(reports):
    """(layers predicted as the oracle predicts where the margin allows, slots hit, slots)."""
    hits = slots = 0
    for r in reports:
        for got, want, margin, h in r["pred"]:
            hits += h
            slots += len(got)
    return hits, slots


@pytest.mark.parametrize("spec", [1, 2], ids=["predict", "mispredict"])
@pytest.mark.parametrize("E,k", [(4, 2), (2, 1), (8, 2)])
def test_tiny_moe_speculative_experts(cuda, E, k, spec):
    # spec 1 streams the predicted experts' first FFN stages before the routing; spec 2 predicts the
    # lowest-scoring experts, so most slots miss and their speculative stages are dropped
    cfg = configs.TINY.with_(name=f"tiny_moe{E}_{k}", n_experts=E, top_k=k)
    reps = parity.run(parity.Setup(cfg), spec_experts=spec)
    parity.assert_parity(reps, cfg)
    assert all("pred" in r for r in reps)


def _no_attention_mixing(W):
    for L in W["layers"]:
        L["wo"] = np.zeros_like(L["wo"])
        L["ffn_norm"] = L["attn_norm"].copy()


@pytest.mark.parametrize("spec", [1, 2], ids=["all_hit", "all_miss"])
def test_tiny_moe_speculative_experts_all_hit_or_all_miss(cuda, spec):
    # With W_o = 0 and one set of norm weights the router sees the attention input itself: the
    # prediction is the routing (every slot hits), and its inverse (bottom-2 of 4) misses every slot.
    cfg = configs.TINY.with_(name="tiny_moe4_2", n_experts=4, top_k=2)
    W = parity.synth.make_model(cfg)
    _no_attention_mixing(W)
    reps = parity.run(parity.Setup(cfg, W), spec_experts=spec)
    parity.assert_parity(reps, cfg)
    hits, slots = _pred_stats(reps)
    assert slots == len(reps) * cfg.n_layers * cfg.top_k
    assert hits == (slots if spec == 1 else 0), (hits, slots)


def test_tiny_moe_speculative_experts_off_is_rejected_by_the_getter(cuda):
    from decode_persistent_block_b200 import MkError
    cfg = configs.TINY.with_(name="tiny_moe4_2", n_experts=4, top_k=2)
    s = parity.Setup(cfg)
    with s.decoder() as dec:
        dec.step(1, 0)
        with pytest.raises(MkError):
            dec.predicted_experts(0)
    with s.decoder(spec_experts=1, l2_prefetch=65536) as dec:  # the general kernel does not predict
        dec.step(1, 0)
        with pytest.raises(MkError):
            dec.predicted_experts(0)


def test_mixtral8l_speculative_experts(cuda):
    reps = _full(configs.MIXTRAL_8L, 3, spec_experts=1)
    hits, slots = _pred_stats(reps)
    print(f"mixtral8l speculative experts: {hits}/{slots} slots hit")


# ---- batched decode ------------------------------------------------------------------

# head_dim 128, two chunks per thread (the Llama-3B kernel's widths) at small depth and vocabulary
H3K_SMALL = configs.TINY.with_(name="tiny_h3072", hidden=3072, n_heads=24, n_kv_heads=8, head_dim=128, ffn=1024)


@pytest.mark.parametrize("B", [2, 3, 4, 5, 8])
def test_tiny_batch(cuda, B):
    # ragged positions: sequence b starts 3 b positions later, with its own cache, prompt and tokens
    parity.assert_parity(parity.run_batch(configs.TINY, [3 * b for b in range(B)], steps=20), configs.TINY)


@pytest.mark.parametrize("B", [2, 4])
def test_head_dim_128_batch(cuda, B):
    parity.assert_parity(parity.run_batch(H3K_SMALL, [5 * b + 1 for b in range(B)], steps=6), H3K_SMALL)


def test_tiny_batch_ring_and_split_options(cuda):
    for opts in (dict(ring_stages=2), dict(kv_splits=3), dict(stage_bytes=32768), dict(n_sm=7)):
        parity.assert_parity(parity.run_batch(configs.TINY, [0, 4, 9, 2], steps=8, **opts), configs.TINY)


def test_batch_handle_rejects_single_steps_and_bad_arguments(cuda):
    import torch
    from decode_persistent_block_b200 import Decoder, MkError, to_device
    cfg = configs.TINY
    W = to_device(parity.synth.make_model(cfg))
    kc, vc = parity.synth.make_kv_cache(cfg)
    dk = torch.from_numpy(np.stack([kc, kc]).view(np.int16)).cuda()
    dv = torch.from_numpy(np.stack([vc, vc]).view(np.int16)).cuda()
    with Decoder(cfg, W, dk, dv, batch=2) as dec:
        with pytest.raises(MkError) as e:
            dec.step(1, 0)
        assert e.value.name == "MK_ERR_INVALID_ARG"
        for toks, pos in (([1, cfg.vocab], [0, 0]), ([1, 2], [0, cfg.max_seq]), ([1, 2], [-1, 0])):
            with pytest.raises(MkError) as e:
                dec.step_batch(toks, pos)
            assert e.value.name == "MK_ERR_INVALID_ARG"
        with pytest.raises(MkError) as e:
            dec.serve_start()
        assert e.value.name == "MK_ERR_INVALID_ARG"
        out = dec.step_batch([1, 2], [0, 0])  # still usable
        assert out.shape == (2,) and dec.status()["code"] == 0
    moe = cfg.with_(name="tiny_moe", n_experts=4, top_k=2)
    Wm = to_device(parity.synth.make_model(moe))
    with pytest.raises(MkError) as e:
        Decoder(moe, Wm, dk, dv, batch=2)
    assert e.value.name == "MK_ERR_UNSUPPORTED"


def test_llama1b_batch2(cuda):
    # two sequences: the FFN stage gate is on by default here, as at batch 1
    cfg = configs.LLAMA_1B
    parity.assert_parity(parity.run_batch(cfg, [cfg.prefill, cfg.prefill - 101], steps=2), cfg)


def test_llama1b_batch8(cuda):
    cfg = configs.LLAMA_1B
    parity.assert_parity(parity.run_batch(cfg, [cfg.prefill - 37 * b for b in range(8)], steps=3), cfg)


def test_llama3b_batch4(cuda):
    cfg = configs.LLAMA_3B
    parity.assert_parity(parity.run_batch(cfg, [cfg.prefill - 101 * b for b in range(4)], steps=2), cfg)
