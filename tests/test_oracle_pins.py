"""Pins for the fp64 oracle against facts fixed outside it.

Each test checks an oracle function against a closed form, an invariant, a
special case that reduces to a library routine, or brute force on a tiny
input, chosen so that a plausible slip (a dropped term, a wrong sign or index,
a transposed operand, a missing scale) fails at least one of them.  None of
these re-types the oracle's own formula for the same input.
"""
import itertools
import math

import numpy as np
import pytest
import scipy.special
import torch

import oracle
import synth
from synth import configs


def bf(vals) -> np.ndarray:
    """float values exactly representable in bf16 -> bf16 bit patterns."""
    a = np.asarray(vals, dtype=np.float32)
    b = synth.f32_to_bf16(a)
    assert np.array_equal(synth.bf16_to_f32(b), a), "test value not exact in bf16"
    return b


# ---- bf16 conversions --------------------------------------------------------

def test_bf16_widening_known_patterns():
    assert oracle.bf16_to_double(0x3F80) == 1.0
    assert oracle.bf16_to_double(0xC000) == -2.0
    assert oracle.bf16_to_double(0x3F81) == 1.0 + 2.0 ** -7
    assert oracle.bf16_to_double(0x0000) == 0.0
    assert math.isinf(oracle.bf16_to_double(0x7F80))


def test_bf16_rounding_ties_to_even():
    assert oracle.bf16_from_double(1.0 + 2.0 ** -8) == 0x3F80            # tie -> even (down)
    assert oracle.bf16_from_double(1.0 + 3 * 2.0 ** -8) == 0x3F82        # tie -> even (up)
    assert oracle.bf16_from_double(1.0 + 2.0 ** -8 + 2.0 ** -30) == 0x3F81  # just above the tie
    assert oracle.bf16_from_double(-(1.0 + 2.0 ** -8 + 2.0 ** -30)) == 0xBF81
    assert oracle.bf16_from_double(0.0) == 0


def test_bf16_rounding_matches_torch_on_float_inputs():
    rng = np.random.default_rng(1)
    vals = rng.standard_normal(4000).astype(np.float32) * np.float32(3.0)
    ref = torch.from_numpy(vals).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([oracle.bf16_from_double(float(v)) for v in vals], dtype=np.uint16)
    assert np.array_equal(ref, got)


# ---- RMSNorm -----------------------------------------------------------------

@pytest.mark.parametrize("c", [0.7, -2.5, 1e-3])
def test_rmsnorm_constant_vector(c):
    n, eps = 64, 1e-5
    w = synth.f32_to_bf16(np.linspace(-2, 2, n).astype(np.float32))
    out = oracle.rmsnorm(np.full(n, c), w, eps)
    expect = c / math.sqrt(c * c + eps) * synth.bf16_to_f32(w).astype(np.float64)
    np.testing.assert_allclose(out, expect, rtol=1e-14, atol=0)


def test_rmsnorm_scale_invariance_and_unit_rms():
    rng = np.random.default_rng(2)
    x = rng.standard_normal(300)
    ones = bf(np.ones(300))
    a = oracle.rmsnorm(x, ones, 0.0)
    b = oracle.rmsnorm(37.0 * x, ones, 0.0)
    np.testing.assert_allclose(a, b, rtol=1e-13)
    assert abs(np.sqrt(np.mean(a ** 2)) - 1.0) < 1e-13


# ---- GEMV --------------------------------------------------------------------

@pytest.mark.parametrize("rows,cols", [(5, 7), (7, 5), (33, 130)])
def test_gemv_exact_on_integers(rows, cols):
    rng = np.random.default_rng(rows * 100 + cols)
    Wi = rng.integers(-8, 9, size=(rows, cols))
    xi = rng.integers(-20, 21, size=cols)
    y = oracle.gemv(bf(Wi), xi.astype(np.float64))
    assert np.array_equal(y, (Wi.astype(np.int64) @ xi.astype(np.int64)).astype(np.float64))


# ---- RoPE (rotate-half) --------------------------------------------------------

def test_rope_position_zero_is_identity():
    v = np.random.default_rng(3).standard_normal(3 * 64)
    np.testing.assert_array_equal(oracle.rope(v, 3, 64, 0, 10000.0), v)


@pytest.mark.parametrize("d,theta,pos", [(64, 10000.0, 5), (128, 500000.0, 1023), (64, 1e6, 16383)])
def test_rope_basis_vectors_rotate_half_pairing(d, theta, pos):
    half = d // 2
    for i in (0, 1, half // 2, half - 1):
        f = theta ** (-2.0 * i / d)
        a = pos * f
        e = np.zeros(d)
        e[i] = 1.0
        r = oracle.rope(e, 1, d, pos, theta)
        expect = np.zeros(d)
        expect[i], expect[i + half] = math.cos(a), math.sin(a)
        np.testing.assert_allclose(r, expect, atol=1e-12)
        e2 = np.zeros(d)
        e2[i + half] = 1.0
        r2 = oracle.rope(e2, 1, d, pos, theta)
        expect2 = np.zeros(d)
        expect2[i], expect2[i + half] = -math.sin(a), math.cos(a)
        np.testing.assert_allclose(r2, expect2, atol=1e-12)


def test_rope_norm_composition_relative_position():
    rng = np.random.default_rng(4)
    d, theta = 64, 10000.0
    q, k = rng.standard_normal(d), rng.standard_normal(d)
    half = d // 2
    r = oracle.rope(q, 1, d, 77, theta)
    # pairwise norms preserved
    np.testing.assert_allclose(q[:half] ** 2 + q[half:] ** 2, r[:half] ** 2 + r[half:] ** 2, rtol=1e-12)
    # R(a) R(b) = R(a + b)
    np.testing.assert_allclose(oracle.rope(oracle.rope(q, 1, d, 30, theta), 1, d, 47, theta), r, atol=1e-11)
    # <R(m) q, R(n) k> depends on m - n only
    base = np.dot(oracle.rope(q, 1, d, 9, theta), oracle.rope(k, 1, d, 4, theta))
    for t in (1, 13, 100):
        np.testing.assert_allclose(np.dot(oracle.rope(q, 1, d, 9 + t, theta), oracle.rope(k, 1, d, 4 + t, theta)),
                                   base, rtol=1e-10)


# ---- softmax / attention -------------------------------------------------------

def test_softmax_matches_scipy_and_sums_to_one():
    s = np.random.default_rng(5).standard_normal(97) * 30
    p = oracle.softmax(s)
    assert abs(p.sum() - 1.0) < 1e-14
    np.testing.assert_allclose(p, scipy.special.softmax(s), rtol=1e-12)


def test_attention_length_one_returns_v():
    rng = np.random.default_rng(6)
    d = 64
    K = synth.f32_to_bf16(rng.standard_normal((1, d)).astype(np.float32))
    V = synth.f32_to_bf16(rng.standard_normal((1, d)).astype(np.float32))
    out = oracle.attend(rng.standard_normal(d) * 10, K, V)
    np.testing.assert_array_equal(out, synth.bf16_to_f32(V[0]).astype(np.float64))


def test_attention_equal_scores_is_mean_of_v():
    rng = np.random.default_rng(7)
    n, d = 50, 64
    K = synth.f32_to_bf16(rng.standard_normal((n, d)).astype(np.float32))
    V = synth.f32_to_bf16(rng.standard_normal((n, d)).astype(np.float32))
    out = oracle.attend(np.zeros(d), K, V)
    np.testing.assert_allclose(out, synth.bf16_to_f32(V).astype(np.float64).mean(0), atol=1e-14)


def test_attention_two_positions_logistic_and_scale():
    # K rows 0 and a*e0; q = b*e0: scores (0, ab/sqrt(d)) -> weight of row 1 is logistic(ab/sqrt(d)).
    d, a, b = 64, 2.0, 3.0
    K = np.zeros((2, d), dtype=np.float32)
    K[1, 0] = a
    V = np.zeros((2, d), dtype=np.float32)
    V[0, 5] = 1.0
    V[1, 9] = 1.0
    q = np.zeros(d)
    q[0] = b
    out = oracle.attend(q, bf(K), bf(V))
    p1 = 1.0 / (1.0 + math.exp(-a * b / math.sqrt(d)))
    assert abs(out[9] - p1) < 1e-15 and abs(out[5] - (1 - p1)) < 1e-15


def test_attention_one_hot_large_score_selects_row():
    d, n = 64, 8
    K = np.zeros((n, d), dtype=np.float32)
    for j in range(n):
        K[j, j] = 1.0
    V = np.arange(n * d, dtype=np.float32).reshape(n, d) % 97
    q = np.zeros(d)
    q[5] = 4000.0
    out = oracle.attend(q, bf(K), bf(V))
    np.testing.assert_allclose(out, V[5].astype(np.float64), atol=1e-9)


# ---- SiLU -------------------------------------------------------------------------

def test_silu_closed_forms():
    ln3 = math.log(3.0)
    assert oracle.silu(0.0) == 0.0
    assert abs(oracle.silu(ln3) - 0.75 * ln3) < 1e-15        # sigmoid(ln 3) = 3/4
    assert abs(oracle.silu(-ln3) + 0.25 * ln3) < 1e-15       # sigmoid(-ln 3) = 1/4
    assert abs(oracle.silu(40.0) - 40.0) < 1e-12
    assert abs(oracle.silu(-40.0)) < 1e-15


# ---- MoE routing --------------------------------------------------------------

def brute_top2(r):
    best = None
    for i, j in itertools.combinations(range(len(r)), 2):   # lexicographic order
        s = r[i] + r[j]
        # pair of the two largest: maximise the smaller member first, then the larger
        key = (min(r[i], r[j]), max(r[i], r[j]))
        if best is None or key > best[0]:
            best = (key, (i, j) if r[i] >= r[j] else (j, i))
    return best[1]


def test_top2_exhaustive_and_weights():
    rng = np.random.default_rng(8)
    for trial in range(300):
        r = rng.standard_normal(8) * 6.4
        idx, w = oracle.topk(r, 2)
        i, j = brute_top2(r)
        assert (idx[0], idx[1]) == (i, j)
        w1 = 1.0 / (1.0 + math.exp(r[j] - r[i]))
        assert abs(w[0] - w1) < 1e-15 and abs(w[1] - (1 - w1)) < 1e-15
        # equals the full softmax renormalised over the two selected experts
        p = scipy.special.softmax(r)
        np.testing.assert_allclose(w, p[[i, j]] / p[[i, j]].sum(), rtol=1e-12)


def test_top2_ties_go_to_lower_index():
    idx, w = oracle.topk(np.array([1.0, 3.0, 3.0, 0.0, 3.0]), 2)
    assert list(idx) == [1, 2] and abs(w[0] - 0.5) < 1e-15
    idx, _ = oracle.topk(np.array([2.0, 2.0, 2.0]), 1)
    assert list(idx) == [0]


def test_argmax_ties_lowest_index():
    assert oracle.argmax([0.0, 5.0, 1.0, 5.0]) == 1
    assert oracle.argmax([-1.0]) == 0


# ---- whole decode step: special cases with closed forms --------------------------

TINY = configs.TINY


def _np_norm(x, w_bf16, eps):
    return x / np.sqrt(np.mean(x * x) + eps) * synth.bf16_to_f32(w_bf16).astype(np.float64)


def _f(a):
    return synth.bf16_to_f32(a).astype(np.float64)


def _zero_like(a):
    return np.zeros_like(a)


def test_model_zero_mixers_is_embedding_head():
    cfg = TINY
    W = synth.make_model(cfg)
    for L in W["layers"]:
        L["wo"] = _zero_like(L["wo"])
        L["w_down"] = _zero_like(L["w_down"])
    kc, vc = synth.make_kv_cache(cfg)
    m = oracle.Model(cfg, W, kc, vc)
    tok = 1234
    out = m.step(tok, 0)
    e = _f(W["embed"][tok])
    for l in range(cfg.n_layers + 1):
        np.testing.assert_array_equal(out["hidden"][l], e)
    logits = _f(W["lm_head"]) @ _np_norm(e, W["final_norm"], cfg.rms_eps)
    np.testing.assert_allclose(out["logits"], logits, rtol=1e-10, atol=1e-12)
    assert out["next"] == int(np.argmax(logits))
    # the append at pos 0 (RoPE at pos 0 is the identity) stores bf16(Wk xn), bf16(Wv xn)
    for l in range(cfg.n_layers):
        xn = _np_norm(e, W["layers"][l]["attn_norm"], cfg.rms_eps)
        kk = (_f(W["layers"][l]["wk"]) @ xn).reshape(cfg.n_kv_heads, cfg.head_dim)
        vv = (_f(W["layers"][l]["wv"]) @ xn).reshape(cfg.n_kv_heads, cfg.head_dim)
        np.testing.assert_array_equal(kc[l, :, 0], synth.f32_to_bf16(kk.astype(np.float32)))
        np.testing.assert_array_equal(vc[l, :, 0], synth.f32_to_bf16(vv.astype(np.float32)))


def test_model_without_layers_is_lm_head_of_embedding():
    cfg = TINY.with_(n_layers=0)
    W = synth.make_model(cfg)
    kc, vc = synth.make_kv_cache(TINY.with_(n_layers=1))
    m = oracle.Model(cfg, W, kc, vc)
    out = m.step(77, 3)
    e = _f(W["embed"][77])
    np.testing.assert_allclose(out["logits"], _f(W["lm_head"]) @ _np_norm(e, W["final_norm"], cfg.rms_eps),
                               rtol=1e-10, atol=1e-12)


def _ffn_np(xn, wg, wu, wd):
    g, u = _f(wg) @ xn, _f(wu) @ xn
    return _f(wd) @ (g / (1.0 + np.exp(-g)) * u)


def test_model_first_position_attention_is_v_with_gqa_mapping():
    # At pos 0 the cache holds one entry, so each query head's attention output
    # is that entry's V row of its kv group g = floor(h / (nq / nkv)).
    cfg = TINY.with_(n_layers=1, n_heads=6, n_kv_heads=3)
    W = synth.make_model(cfg)
    kc, vc = synth.make_kv_cache(cfg)
    out = oracle.Model(cfg, W, kc, vc).step(2024, 0)
    L = W["layers"][0]
    e = _f(W["embed"][2024])
    xn = _np_norm(e, L["attn_norm"], cfg.rms_eps)
    v = (_f(L["wv"]) @ xn).astype(np.float32)
    vb = synth.bf16_to_f32(synth.f32_to_bf16(v)).astype(np.float64).reshape(cfg.n_kv_heads, cfg.head_dim)
    att = np.concatenate([vb[h // (cfg.n_heads // cfg.n_kv_heads)] for h in range(cfg.n_heads)])
    x1 = e + _f(L["wo"]) @ att
    np.testing.assert_allclose(out["hidden"][1] - (x1 + _ffn_np(_np_norm(x1, L["ffn_norm"], cfg.rms_eps),
                                                                 L["w_gate"], L["w_up"], L["w_down"])),
                               0, atol=1e-12)


def _moe_cfg(E, k):
    return TINY.with_(name="tiny_moe", n_layers=1, n_experts=E, top_k=k)


def test_moe_identical_experts_equal_dense_ffn():
    cfg_d = TINY.with_(n_layers=1)
    Wd = synth.make_model(cfg_d)
    cfg_m = _moe_cfg(4, 2)
    Wm = synth.make_model(cfg_m)
    L = Wm["layers"][0]
    for name in ("attn_norm", "wq", "wk", "wv", "wo", "ffn_norm"):
        L[name] = Wd["layers"][0][name]
    for name in ("w_gate", "w_up", "w_down"):
        L[name] = [Wd["layers"][0][name]] * 4
    Wm["embed"], Wm["lm_head"] = Wd["embed"], Wd["lm_head"]
    kc, vc = synth.make_kv_cache(cfg_d)
    a = oracle.Model(cfg_d, Wd, kc.copy(), vc.copy()).step(9, 0)
    b = oracle.Model(cfg_m, Wm, kc.copy(), vc.copy()).step(9, 0)
    np.testing.assert_allclose(b["hidden"], a["hidden"], rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(b["router_w"].sum(), 1.0, rtol=1e-15)


def test_moe_single_expert_top1_is_dense():
    cfg_d = TINY.with_(n_layers=1)
    Wd = synth.make_model(cfg_d)
    cfg_m = _moe_cfg(1, 1)
    Wm = dict(Wd)
    L = dict(Wd["layers"][0])
    L["router"] = synth.normal_bf16((1, cfg_m.hidden), 0, "r", 0.1)
    for name in ("w_gate", "w_up", "w_down"):
        L[name] = [Wd["layers"][0][name]]
    Wm["layers"] = [L]
    kc, vc = synth.make_kv_cache(cfg_d)
    a = oracle.Model(cfg_d, Wd, kc.copy(), vc.copy()).step(11, 0)
    b = oracle.Model(cfg_m, Wm, kc.copy(), vc.copy()).step(11, 0)
    np.testing.assert_array_equal(b["hidden"], a["hidden"])
    assert b["router_w"][0, 0] == 1.0


def test_moe_router_choice_is_exhaustive_top2_of_router_scores():
    cfg = _moe_cfg(8, 2)
    W = synth.make_model(cfg)
    kc, vc = synth.make_kv_cache(cfg)
    for tok in (5, 600, 3000):
        out = oracle.Model(cfg, W, kc.copy(), vc.copy()).step(tok, 0)
        L = W["layers"][0]
        e = _f(W["embed"][tok])
        xn = _np_norm(e, L["attn_norm"], cfg.rms_eps)
        v = (_f(L["wv"]) @ xn).astype(np.float32)
        vb = synth.bf16_to_f32(synth.f32_to_bf16(v)).astype(np.float64).reshape(cfg.n_kv_heads, cfg.head_dim)
        att = np.concatenate([vb[h // (cfg.n_heads // cfg.n_kv_heads)] for h in range(cfg.n_heads)])
        x1 = e + _f(L["wo"]) @ att
        xn2 = _np_norm(x1, L["ffn_norm"], cfg.rms_eps)
        r = _f(L["router"]) @ xn2
        i, j = brute_top2(r)
        assert tuple(out["router_idx"][0]) == (i, j)
        w1 = 1.0 / (1.0 + math.exp(r[j] - r[i]))
        expect = x1 + w1 * _ffn_np(xn2, L["w_gate"][i], L["w_up"][i], L["w_down"][i]) + \
            (1 - w1) * _ffn_np(xn2, L["w_gate"][j], L["w_up"][j], L["w_down"][j])
        np.testing.assert_allclose(out["hidden"][1], expect, atol=1e-12)


def _no_attention_mixing(W):
    """Attention adds nothing to the residual (W_o = 0) and the FFN norm weights are the attention
    norm weights: the FFN's router then sees exactly the attention input of its layer."""
    for L in W["layers"]:
        L["wo"] = _zero_like(L["wo"])
        L["ffn_norm"] = L["attn_norm"].copy()


def test_prediction_is_the_routing_when_attention_adds_nothing():
    # Speculative expert prediction reads the residual entering the layer; the router reads it after
    # attention.  With nothing added by attention (and one set of norm weights) the two agree in every
    # layer, which fixes the prediction's input to the layer's own entering residual.
    cfg = TINY.with_(name="tiny_moe", n_layers=3, n_experts=8, top_k=2)
    W = synth.make_model(cfg)
    _no_attention_mixing(W)
    kc, vc = synth.make_kv_cache(cfg)
    m = oracle.Model(cfg, W, kc, vc)
    for pos, tok in enumerate((5, 600, 3000, 77)):
        out = m.step(tok, pos)
        np.testing.assert_array_equal(out["pred_idx"], out["router_idx"])
    # top-1 of 4 experts too
    cfg1 = cfg.with_(n_experts=4, top_k=1)
    W1 = synth.make_model(cfg1)
    _no_attention_mixing(W1)
    kc, vc = synth.make_kv_cache(cfg1)
    out = oracle.Model(cfg1, W1, kc, vc).step(42, 0)
    np.testing.assert_array_equal(out["pred_idx"], out["router_idx"])


def test_prediction_ignores_the_ffn_norm_weights():
    # The prediction of layer 0 is made from the embedding row with the attention norm weights: changing
    # the FFN norm weights changes the routing but never the prediction.
    cfg = TINY.with_(name="tiny_moe", n_layers=1, n_experts=8, top_k=2)
    W = synth.make_model(cfg)
    _no_attention_mixing(W)
    kc, vc = synth.make_kv_cache(cfg)
    preds, routes = [], []
    for seed in range(6):
        W["layers"][0]["ffn_norm"] = synth.normal_bf16((cfg.hidden,), 0, f"fn{seed}", 1.0)
        out = oracle.Model(cfg, W, kc.copy(), vc.copy()).step(321, 0)
        preds.append(tuple(out["pred_idx"][0]))
        routes.append(tuple(out["router_idx"][0]))
    assert len(set(preds)) == 1
    assert len(set(routes)) > 1  # the FFN norm weights did change the routing
    W["layers"][0]["ffn_norm"] = W["layers"][0]["attn_norm"].copy()
    out = oracle.Model(cfg, W, kc.copy(), vc.copy()).step(321, 0)
    assert tuple(out["router_idx"][0]) == preds[0]


def test_rejects_bad_token_and_position():
    cfg = TINY
    W = synth.make_model(cfg)
    kc, vc = synth.make_kv_cache(cfg)
    m = oracle.Model(cfg, W, kc, vc)
    with pytest.raises(ValueError):
        m.step(cfg.vocab, 0)
    with pytest.raises(ValueError):
        m.step(0, kc.shape[2])


def test_oracle_agrees_with_independent_fp32_restatement():
    # Tiny model: the 16-token prompt decoded from pos 0 then 8 greedy steps,
    # run through the fp64 oracle and through an fp32 torch restatement.
    from oracle.fp32_torch import Fp32Model
    cfg = TINY
    W = synth.make_model(cfg)
    kc, vc = synth.make_kv_cache(cfg)
    a = oracle.Model(cfg, W, kc.copy(), vc.copy())
    b = Fp32Model(cfg, W, kc.copy(), vc.copy())
    toks = list(synth.prompt_tokens(cfg))
    pos = 0
    worst_h, worst_l = 0.0, 0.0
    for step in range(cfg.prompt_len + cfg.steps):
        t = toks[step] if step < len(toks) else nxt
        oa, ob = a.step(t, pos), b.step(t, pos)
        rel = np.linalg.norm(ob["hidden"] - oa["hidden"], axis=1) / np.linalg.norm(oa["hidden"], axis=1)
        worst_h = max(worst_h, float(rel.max()))
        worst_l = max(worst_l, float(np.abs(ob["logits"] - oa["logits"]).max()))
        nxt = oa["next"]
        pos += 1
    assert worst_h < 1e-4, worst_h
    assert worst_l < 1e-3, worst_l
