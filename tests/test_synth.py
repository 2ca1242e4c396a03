"""The seeded input generator: determinism, split-independence, distribution."""
import numpy as np
import torch

import synth
from synth import configs


def test_same_stream_same_bits_other_stream_differs():
    a = synth.normal_bf16((1000,), 0, "layers.0.wq", 0.02)
    b = synth.normal_bf16((1000,), 0, "layers.0.wq", 0.02)
    c = synth.normal_bf16((1000,), 0, "layers.0.wk", 0.02)
    d = synth.normal_bf16((1000,), 1, "layers.0.wq", 0.02)
    assert np.array_equal(a, b)
    assert not np.array_equal(a, c) and not np.array_equal(a, d)


def test_element_depends_only_on_index():
    a = synth.normal_bf16((10001,), 3, "x", 1.0)
    b = synth.normal_bf16((5000,), 3, "x", 1.0)
    assert np.array_equal(a[:5000], b)


def test_normal_moments():
    a = synth.bf16_to_f32(synth.normal_bf16((1 << 21,), 0, "moments", 0.02)).astype(np.float64)
    assert abs(a.mean()) < 1e-4
    assert abs(a.std() / 0.02 - 1.0) < 5e-3
    within = np.mean(np.abs(a) < 0.02)
    assert abs(within - 0.6827) < 3e-3


def test_f32_to_bf16_matches_torch():
    x = np.random.default_rng(0).standard_normal(100000).astype(np.float32) * 7
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(synth.f32_to_bf16(x), ref)
    assert synth.lib().synth_f32_to_bf16(1.0) == 0x3F80


def test_kv_prefill_independent_of_max_seq_and_zero_tail():
    cfg = configs.TINY.with_(prefill=10, prompt_len=0, steps=5)
    k1, v1 = synth.make_kv_cache(cfg, max_seq=15)
    k2, v2 = synth.make_kv_cache(cfg, max_seq=40)
    assert np.array_equal(k1[:, :, :10], k2[:, :, :10]) and np.array_equal(v1[:, :, :10], v2[:, :, :10])
    assert not np.any(k2[:, :, 10:]) and not np.any(v1[:, :, 10:])
    assert not np.array_equal(k1[:, :, :10], v1[:, :, :10])


def test_tokens_in_range_and_model_shapes():
    t = synth.tokens(10000, 0, "prompt", 4096)
    assert t.min() >= 0 and t.max() < 4096 and len(np.unique(t)) > 3000
    cfg = configs.TINY
    m = synth.make_model(cfg)
    assert m["embed"].shape == (cfg.vocab, cfg.hidden)
    assert m["layers"][1]["wq"].shape == (cfg.n_heads * cfg.head_dim, cfg.hidden)
    assert m["layers"][0]["w_down"].shape == (cfg.hidden, cfg.ffn)
    assert np.all(m["final_norm"] == 0x3F80)
    assert m["lm_head"] is not m["embed"]
    assert synth.make_model(cfg.with_(tied=True))["lm_head"] is not None


def test_byte_accounting_matches_shapes():
    # Weight bytes per token for the 1B shape: 16 layers of (qkv 3072x2048, o 2048^2,
    # gate/up/down 3 x 8192x2048, two norms) + one embedding row + 128256x2048 head + final norm.
    assert configs.LLAMA_1B.weight_bytes_per_token() == 2_471_632_896
    assert configs.LLAMA_3B.weight_bytes_per_token() == 6_425_505_792
    assert configs.MIXTRAL_8L.weight_bytes_per_token() == 6_571_048_960
    assert configs.LLAMA_1B.kv_bytes_per_token(1024) == 1025 * 32768
