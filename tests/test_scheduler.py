"""Host scheduler: bit-exact integer checks, no GPU needed.

The schedule must cover every output row of every op exactly once, order each
block's queue by op so that no wait can deadlock, and give every dependency
counter a per-step increment equal to the number of instructions that signal
it (after S steps on the device every counter must read exactly S times that).
"""
import itertools

import numpy as np
import pytest

import decode_persistent_block_b200 as dpb
from decode_persistent_block_b200 import mk
from synth import configs

OP = dict(RMS_QKV=1, ATTN=2, OPROJ=3, UG=4, DOWN=5, LM=6, MOE_UG=7, MOE_DOWN=8, FFN=9, MOE_FFN=10)
W_OP, W_LAYER, W_SUB, W_BEGIN, W_END, W_WAIT, W_WINC, W_SIG, W_AUX, W_AINC, W_SEQ = range(11)

CFGS = [configs.TINY, configs.LLAMA_1B, configs.LLAMA_3B, configs.MIXTRAL_8L, configs.llama1b_sweep(16384),
        configs.TINY.with_(name="tiny_moe", n_experts=4, top_k=2),
        configs.TINY.with_(name="tiny_moe1", n_experts=2, top_k=1),
        configs.TINY.with_(name="tiny_l0", n_layers=0)]


@pytest.fixture(scope="module", autouse=True)
def _built():
    dpb.build()


def instrs(words, n_instr):
    for sm in range(words.shape[0]):
        for i in range(n_instr[sm]):
            yield sm, i, words[sm, i]


def n_ctr_per_layer(cfg):
    return 5  # QKV, ATTN, OPROJ, FFN1, FFN2


@pytest.mark.parametrize("split_ffn", [0, 1], ids=["fused_ffn", "split_ffn"])
@pytest.mark.parametrize("cfg", CFGS, ids=lambda c: c.name)
@pytest.mark.parametrize("n_sm", [148, 37, 1])
def test_plan_covers_rows_and_counts_signals(cfg, n_sm, split_ffn):
    words, n_instr, inc = dpb.plan(cfg, n_sm, split_ffn=split_ffn)
    L, nkv, d = cfg.n_layers, cfg.n_kv_heads, cfg.head_dim
    per = n_ctr_per_layer(cfg)
    assert inc.size == L * per + 1
    rows = {OP["RMS_QKV"]: {0: cfg.n_heads * d, 1: nkv * d, 2: nkv * d}, OP["OPROJ"]: {0: cfg.hidden},
            OP["UG"]: {0: cfg.ffn}, OP["DOWN"]: {0: cfg.hidden}, OP["LM"]: {0: cfg.vocab},
            OP["MOE_UG"]: {s: cfg.ffn for s in range(max(cfg.top_k, 1))}, OP["MOE_DOWN"]: {0: cfg.hidden},
            OP["FFN"]: {0: cfg.ffn}, OP["MOE_FFN"]: {s: cfg.ffn for s in range(max(cfg.top_k, 1))}}
    cover = {}
    signals = np.zeros_like(inc)
    splits = None
    attn_seen = set()
    for sm, i, w in instrs(words, n_instr):
        op, l = int(w[W_OP]), int(w[W_LAYER])
        if op == OP["ATTN"]:
            splits = int(w[W_END])
            key = (l, int(w[W_SUB]), int(w[W_BEGIN]))
            assert key not in attn_seen
            attn_seen.add(key)
            assert w[W_AUX] == -1 and w[W_SIG] == l * per + 1 and w[W_WAIT] == l * per + 0
            signals[w[W_SIG]] += 1
            continue
        key = (l, op, int(w[W_SUB]))
        hit = cover.setdefault(key, np.zeros(rows[op][int(w[W_SUB])], dtype=np.int32))
        hit[w[W_BEGIN]:w[W_END]] += 1
        assert 0 < w[W_END] - w[W_BEGIN] <= 1024
        signals[w[W_AUX] if op == OP["LM"] else w[W_SIG]] += 1
    for key, hit in cover.items():
        assert np.all(hit == 1), key
    moe = cfg.n_experts > 0
    if split_ffn:
        ffn_ops = (OP["MOE_UG"], OP["MOE_DOWN"]) if moe else (OP["UG"], OP["DOWN"])
    else:
        ffn_ops = (OP["MOE_FFN"],) if moe else (OP["FFN"],)
        for l in range(L):  # the fused FFN signals the post-FFN counter; the mid-FFN one is unused
            assert inc[l * per + 3] == 0
    for l in range(L):
        for op in (OP["RMS_QKV"], OP["OPROJ"]) + ffn_ops:
            assert (l, op, 0) in cover
    assert (L, OP["LM"], 0) in cover
    assert np.array_equal(signals, inc)
    if L:
        assert len(attn_seen) == L * nkv * splits
        # closed form: every split of every kv head signals; the O-projection waits for all
        for l in range(L):
            assert inc[l * per + 1] == nkv * splits


def _ranges(total, n_sm):
    return [(total * s // n_sm, total * (s + 1) // n_sm) for s in range(n_sm)]


@pytest.mark.parametrize("split_ffn", [0, 1], ids=["fused_ffn", "split_ffn"])
@pytest.mark.parametrize("n_sm", [148, 132, 64])
def test_increment_closed_forms_llama1b(n_sm, split_ffn):
    cfg = configs.LLAMA_1B
    words, n_instr, inc = dpb.plan(cfg, n_sm, split_ffn=split_ffn)
    per = n_ctr_per_layer(cfg)
    lm = sum(-(-(b - a) // 1024) for a, b in _ranges(cfg.vocab, n_sm))
    for l in range(cfg.n_layers):
        assert inc[l * per + 0] == n_sm      # QKV: every block holds rows of exactly one of q, k, v
        assert inc[l * per + 2] == n_sm      # O-proj: hidden >= n_sm rows, <= 1024 per block
        assert inc[l * per + 3] == (n_sm if split_ffn else 0)  # up/gate (split FFN only)
        assert inc[l * per + 4] == n_sm      # down, or the fused FFN slice
    assert inc[-1] == lm
    # every block's queue is sorted by (layer, op slot)
    order = {OP["RMS_QKV"]: 0, OP["ATTN"]: 1, OP["OPROJ"]: 2, OP["UG"]: 3, OP["FFN"]: 3, OP["DOWN"]: 4,
             OP["LM"]: 0}
    for sm in range(n_sm):
        keys = [int(w[W_LAYER]) * 5 + order[int(w[W_OP])] for w in words[sm, :n_instr[sm]]]
        assert keys == sorted(keys)


@pytest.mark.parametrize("cfg", [configs.LLAMA_1B, configs.LLAMA_3B, configs.MIXTRAL_8L], ids=lambda c: c.name)
def test_segments_get_blocks_in_proportion_to_rows(cfg):
    # QKV (and the MoE expert slots): blocks are shared out by rows, so the
    # largest per-block row count stays within one row of the even split.
    n_sm = 148
    words, n_instr, _ = dpb.plan(cfg, n_sm)
    op = OP["RMS_QKV"]
    rows = [int(w[W_END] - w[W_BEGIN]) for _, _, w in instrs(words, n_instr) if w[W_OP] == op and w[W_LAYER] == 0]
    assert len(rows) == n_sm
    assert max(rows) <= -(-cfg.qkv_rows // n_sm) + 1


def test_plan_is_deterministic():
    a = dpb.plan(configs.LLAMA_3B, 148)
    b = dpb.plan(configs.LLAMA_3B, 148)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


@pytest.mark.parametrize("split_ffn", [0, 1], ids=["fused_ffn", "split_ffn"])
@pytest.mark.parametrize("cfg", CFGS, ids=lambda c: c.name)
def test_simulated_interleavings_complete_and_counters_match(cfg, split_ffn):
    words, n_instr, inc = dpb.plan(cfg, 148 if cfg.hidden > 256 else 23, split_ffn=split_ffn)
    for seed in range(3):
        rc, done = dpb.simulate(words, n_instr, inc, steps=3, seed=seed)
        assert rc == mk.MK_OK
        assert done == 3 * int(n_instr.sum())


def test_simulator_detects_deadlock_and_count_mismatch():
    cfg = configs.TINY
    words, n_instr, inc = dpb.plan(cfg, 4, split_ffn=1)
    # move block 0's first layer-1 QKV in front of its layer-0 down-projection
    q = words[0, :n_instr[0]].copy()
    i_down = next(i for i, w in enumerate(q) if w[W_OP] == OP["DOWN"] and w[W_LAYER] == 0)
    i_qkv = next(i for i, w in enumerate(q) if w[W_OP] == OP["RMS_QKV"] and w[W_LAYER] == 1)
    bad = words.copy()
    bad[0, [i_down, i_qkv]] = q[[i_qkv, i_down]]
    rc, done = dpb.simulate(bad, n_instr, inc, steps=1, seed=0)
    assert rc == mk.CODES["MK_ERR_SCHEDULE"] and done < n_instr.sum()
    wrong = inc.copy()
    wrong[0] += 1
    rc, _ = dpb.simulate(words, n_instr, wrong, steps=1, seed=0)
    assert rc != mk.MK_OK


def test_plan_rejects_unsupported_shapes():
    with pytest.raises(mk.MkError) as e:
        dpb.plan(configs.TINY.with_(head_dim=96), 148)
    assert e.value.name == "MK_ERR_UNSUPPORTED"
    with pytest.raises(mk.MkError) as e:
        dpb.plan(configs.TINY.with_(n_heads=10, n_kv_heads=2), 148)  # 5 query heads per kv head
    assert e.value.name == "MK_ERR_UNSUPPORTED"
    with pytest.raises(mk.MkError) as e:
        dpb.plan(configs.TINY, 0)
    assert e.value.name == "MK_ERR_INVALID_ARG"
    with pytest.raises(mk.MkError):
        dpb.plan(configs.TINY, 148, stage_bytes=1000)


@pytest.mark.parametrize("splits", [1, 3, 40])
def test_kv_splits_option(splits):
    words, n_instr, inc = dpb.plan(configs.TINY, 16, kv_splits=splits)
    attn = [w for _, _, w in instrs(words, n_instr) if w[W_OP] == OP["ATTN"]]
    assert len(attn) == configs.TINY.n_layers * configs.TINY.n_kv_heads * splits
    assert all(w[W_END] == splits for w in attn)


def test_rows_per_instr_cap_splits_instructions():
    words, n_instr, inc = dpb.plan(configs.TINY, 2, rows_per_instr=64)
    for _, _, w in instrs(words, n_instr):
        if w[W_OP] != OP["ATTN"]:
            assert w[W_END] - w[W_BEGIN] <= 64


def test_fused_ffn_is_the_default_for_every_supported_hidden_size():
    # hidden <= 8192 and a stage holds a whole hidden row: the fused form always applies
    ops = lambda cfg, **kw: {int(w[W_OP]) for _, _, w in instrs(*dpb.plan(cfg, 148, **kw)[:2])}
    for cfg in (configs.LLAMA_3B, configs.TINY.with_(hidden=8192)):
        assert OP["FFN"] in ops(cfg) and OP["UG"] not in ops(cfg)
        assert OP["FFN"] not in ops(cfg, split_ffn=1) and {OP["UG"], OP["DOWN"]} <= ops(cfg, split_ffn=1)


@pytest.mark.parametrize("cfg,expect", [(configs.LLAMA_1B, 6), (configs.LLAMA_3B, 17), (configs.TINY, 1),
                                        (configs.llama1b_sweep(128), 3), (configs.llama1b_sweep(2048), 8),
                                        (configs.llama1b_sweep(16384), 16), (configs.llama1b_sweep(65536), 18),
                                        (configs.MIXTRAL_8L, 9)], ids=lambda x: getattr(x, "name", x))
def test_default_kv_splits(cfg, expect):
    # head_dim 64: the split count minimising 10 ns * rows per split + 0.3 us per split
    # + 1 us per merge round trip of 8 splits (exhaustive here); head_dim 128: about one
    # split per 128 positions.  Both at most one split per SM per kv head.
    words, n_instr, inc = dpb.plan(cfg, 148)
    attn = [w for _, _, w in instrs(words, n_instr) if w[W_OP] == OP["ATTN"]]
    s = int(attn[0][W_END]) if attn else 0
    cap = min(148 // cfg.n_kv_heads, 2048 // cfg.n_heads)
    if cfg.head_dim == 64:
        cost = {k: 10 * cfg.max_seq / k + 300 * k + 1000 * -(-k // 8) for k in range(1, cap + 1)}
        want = min(cost, key=lambda k: (cost[k], k))
    else:
        want = min(-(-cfg.max_seq // 128), cap)
    assert s == want
    if expect is not None:
        assert s == expect


def test_kv_splits_limit_is_checked():
    cfg = configs.LLAMA_1B  # 32 query heads: at most 64 splits merged per head
    dpb.plan(cfg, 148, kv_splits=64)
    with pytest.raises(mk.MkError) as e:
        dpb.plan(cfg, 148, kv_splits=65)
    assert e.value.name == "MK_ERR_INVALID_ARG"


@pytest.mark.parametrize("permille", [950, 1000, 800])
def test_attention_blocks_take_fewer_ffn_rows(permille):
    cfg = configs.LLAMA_1B
    words, n_instr, _ = dpb.plan(cfg, 148, attn_sm_ffn_permille=permille)
    for l in (0, 1):
        attn_sms = {sm for sm in range(148) for w in words[sm, :n_instr[sm]]
                    if w[W_OP] == OP["ATTN"] and w[W_LAYER] == l}
        rows = {sm: int(w[W_END] - w[W_BEGIN]) for sm in range(148) for w in words[sm, :n_instr[sm]]
                if w[W_OP] == OP["FFN"] and w[W_LAYER] == l}
        assert sum(rows.values()) == cfg.ffn and len(rows) == 148
        a = np.mean([rows[s] for s in attn_sms])
        b = np.mean([rows[s] for s in rows if s not in attn_sms])
        assert a / b == pytest.approx(permille / 1000, abs=0.03)


def _rows_per_sm(words, n_instr, op, layer):
    r = np.zeros(words.shape[0], dtype=np.int64)
    for sm, _, w in instrs(words, n_instr):
        if w[W_OP] == OP[op] and w[W_LAYER] == layer:
            r[sm] += int(w[W_END]) - int(w[W_BEGIN])
    return r


@pytest.mark.parametrize("n_sm", [148, 13])
def test_sm_speed_splits_ffn_and_lm_rows_in_proportion(n_sm):
    cfg = configs.LLAMA_1B
    speed = np.linspace(0.5, 1.5, n_sm)
    words, n_instr, inc = dpb.plan(cfg, n_sm, sm_speed=speed)
    for op, layer, total in (("FFN", 3, cfg.ffn), ("LM", cfg.n_layers, cfg.vocab)):
        rows = _rows_per_sm(words, n_instr, op, layer)
        assert rows.sum() == total
        # each block's share is its speed's share of the total, to a row (the cut points round)
        want = total * speed / speed.sum()
        assert np.abs(rows - want).max() <= 1.0 + 1e-9
    # every other op keeps the even split of the default schedule
    w0, n0, inc0 = dpb.plan(cfg, n_sm)
    for op in ("RMS_QKV", "OPROJ"):
        np.testing.assert_array_equal(_rows_per_sm(words, n_instr, op, 3), _rows_per_sm(w0, n0, op, 3))
    # QKV, attention and O-projection counters keep their increments; the FFN's and the LM head's
    # count their instructions: one per started 512 FFN rows (two accumulator sets of 1024 slots)
    # or 1024 LM rows of a block's share
    L = cfg.n_layers
    for slot in (0, 1, 2):
        np.testing.assert_array_equal(inc[slot:5 * L:5], inc0[slot:5 * L:5])
    ffn = _rows_per_sm(words, n_instr, "FFN", 3)
    assert inc[5 * 3 + 4] == sum(-(-int(r) // 512) for r in ffn)
    lm = _rows_per_sm(words, n_instr, "LM", L)
    assert inc[-1] == sum(-(-int(r) // 1024) for r in lm)
    rc, done = mk.simulate(words, n_instr, inc, steps=2, seed=3)
    assert rc == 0 and done == 2 * int(n_instr.sum())


def test_sm_speed_uniform_matches_default_and_bad_speeds_are_rejected():
    # equal speeds give the default split (the LM head's cut points may round the other way: +-1 row)
    cfg = configs.LLAMA_1B
    w0, n0, _ = dpb.plan(cfg, 148)
    w1, n1, _ = dpb.plan(cfg, 148, sm_speed=np.full(148, 2.5))
    np.testing.assert_array_equal(n0, n1)
    for layer in range(cfg.n_layers):
        for op in ("RMS_QKV", "ATTN", "OPROJ", "FFN"):
            np.testing.assert_array_equal(_rows_per_sm(w0, n0, op, layer), _rows_per_sm(w1, n1, op, layer))
    d = _rows_per_sm(w0, n0, "LM", cfg.n_layers) - _rows_per_sm(w1, n1, "LM", cfg.n_layers)
    assert np.abs(d).max() <= 1 and d.sum() == 0
    for bad in (np.ones(147), np.r_[np.ones(147), 0.0], np.r_[np.ones(147), -1.0], np.r_[np.ones(147), np.nan],
                np.r_[np.ones(147), np.inf]):
        with pytest.raises(mk.MkError):
            dpb.plan(cfg, 148, sm_speed=bad)


W_SPEC = 11


@pytest.mark.parametrize("n_sm", [148, 37, 600, 1])
@pytest.mark.parametrize("cfg", [configs.MIXTRAL_8L, configs.TINY.with_(name="tiny_moe", n_experts=4, top_k=2),
                                 configs.TINY.with_(name="tiny_moe1", n_experts=2, top_k=1)], ids=lambda c: c.name)
def test_speculative_prediction_marks(cfg, n_sm):
    # Every block that runs a QKV instruction and a fused MoE FFN slice of a layer predicts the layer's
    # experts after its last QKV instruction of the layer; those FFN slices stream the prediction; the
    # lowest such block publishes.  Nothing else carries the mark.
    words, n_instr, _ = dpb.plan(cfg, n_sm, spec_experts=1)
    L = cfg.n_layers
    expect = np.zeros_like(words[:, :, W_SPEC])
    publisher = [None] * L
    for sm in range(n_sm):
        q = words[sm, :n_instr[sm]]
        for l in range(L):
            qkv = [i for i in range(len(q)) if q[i, W_OP] == OP["RMS_QKV"] and q[i, W_LAYER] == l]
            ffn = [i for i in range(len(q)) if q[i, W_OP] == OP["MOE_FFN"] and q[i, W_LAYER] == l]
            if qkv and ffn:
                assert max(qkv) < min(ffn)
                expect[sm, max(qkv)] = 1
                expect[sm, ffn] = 1
                if publisher[l] is None:
                    publisher[l] = sm
                    expect[sm, max(qkv)] = 2
    np.testing.assert_array_equal(words[:, :, W_SPEC], expect)
    if (cfg.n_heads + 2 * cfg.n_kv_heads) * cfg.head_dim >= n_sm:
        # every block holds QKV rows of every layer: every FFN slice streams a prediction
        ffn = words[:, :, W_OP] == OP["MOE_FFN"]
        assert np.all(words[:, :, W_SPEC][ffn] == 1)
    else:  # more blocks than QKV rows: the blocks without QKV rows stream no prediction
        assert np.any(expect[words[:, :, W_OP] == OP["MOE_FFN"]] == 0)
    # the mark changes nothing else
    base, n0, inc0 = dpb.plan(cfg, n_sm)
    assert np.all(base[:, :, W_SPEC] == 0)
    w2 = words.copy()
    w2[:, :, W_SPEC] = 0
    np.testing.assert_array_equal(w2, base)


@pytest.mark.parametrize("cfg,opts", [(configs.LLAMA_1B, {}), (configs.MIXTRAL_8L, dict(split_ffn=1))],
                         ids=["dense", "moe_split_ffn"])
def test_speculative_prediction_needs_the_fused_moe_ffn(cfg, opts):
    words, _, _ = dpb.plan(cfg, 148, spec_experts=1, **opts)
    assert np.all(words[:, :, W_SPEC] == 0)


def test_speculative_prediction_option_range():
    for bad in (-1, 3):
        with pytest.raises(mk.MkError):
            dpb.plan(configs.MIXTRAL_8L, 148, spec_experts=bad)


@pytest.mark.parametrize("B", [2, 5, 8])
@pytest.mark.parametrize("n_sm", [148, 37])
def test_batch_schedule(B, n_sm):
    # every (sequence, kv head, split) attention instruction once per layer; every GEMV instruction keeps
    # B accumulator sets per row within the shared-memory slots; counters count the batch's signals
    cfg = configs.LLAMA_1B
    words, n_instr, inc = dpb.plan(cfg, n_sm, batch=B)
    S = None
    seen = set()
    for sm, i, w in instrs(words, n_instr):
        op = int(w[W_OP])
        if op == OP["ATTN"]:
            S = int(w[W_END])
            key = (int(w[W_LAYER]), int(w[W_SEQ]), int(w[W_SUB]), int(w[W_BEGIN]))
            assert key not in seen and 0 <= key[1] < B
            seen.add(key)
        else:
            sets = 2 if op == OP["FFN"] else 1
            if op != OP["LM"]:  # the LM head goes through its rows in chunks
                assert (w[W_END] - w[W_BEGIN]) * sets * B <= 1024
    assert len(seen) == cfg.n_layers * B * cfg.n_kv_heads * S
    assert inc[1] == B * cfg.n_kv_heads * S  # layer 0's attention counter
    assert B * cfg.n_kv_heads * S <= max(n_sm, B * cfg.n_kv_heads)
    rc, done = dpb.simulate(words, n_instr, inc, steps=2, seed=B)
    assert rc == 0 and done == 2 * int(n_instr.sum())


def test_batch_options_are_checked():
    with pytest.raises(mk.MkError) as e:
        dpb.plan(configs.LLAMA_1B, 148, batch=9)
    assert e.value.name == "MK_ERR_INVALID_ARG"
    for cfg, opts in ((configs.LLAMA_3B, dict(batch=8)), (configs.MIXTRAL_8L, dict(batch=2)),
                      (configs.LLAMA_1B, dict(batch=2, split_ffn=1)), (configs.LLAMA_1B, dict(batch=2, mode=1)),
                      (configs.LLAMA_1B, dict(batch=2, l2_prefetch=65536))):
        with pytest.raises(mk.MkError) as e:
            dpb.plan(cfg, 148, **opts)
        assert e.value.name == "MK_ERR_UNSUPPORTED", (cfg.name, opts)
    dpb.plan(configs.LLAMA_3B, 148, batch=4)


W_MERGE = 12


@pytest.mark.parametrize("cfg,opts", [
    (configs.LLAMA_1B, {}),                  # 148 blocks: 32 heads x 6 splits x 64 x 4 B = 48 KB of partials
    (configs.LLAMA_3B, {}),                  # 24 x 17 x 128 x 4 B = 204 KB
    (configs.MIXTRAL_8L, {}),                # 32 x 9 x 128 x 4 B = 144 KB
    (configs.llama1b_sweep(16384), {}),      # 32 x 16 x 64 x 4 B = 128 KB
    (configs.LLAMA_1B, dict(kv_splits=12)),  # exactly 96 KB: not above the bound
    (configs.LLAMA_1B, dict(kv_splits=13)),
    (configs.LLAMA_1B, dict(attn_merge=2)),
    (configs.LLAMA_3B, dict(attn_merge=1)),
    (configs.LLAMA_3B, dict(batch=2)),       # batched decode merges in the O-projection
    (configs.TINY, dict(attn_merge=2)),
], ids=lambda x: getattr(x, "name", str(x)))
@pytest.mark.parametrize("n_sm", [148, 37])
def test_attention_merge_marks(cfg, opts, n_sm):
    # Every attention split and O-projection instruction of every layer carries the same merge mark:
    # forced by attn_merge, else set when the partials every O-projection block would read
    # (n_q_heads x splits x head_dim fp32) exceed 96 KB at batch 1.  Nothing else carries it, and it
    # changes no other word and no counter increment.
    words, n_instr, inc = dpb.plan(cfg, n_sm, **opts)
    ops = words[:, :, W_OP]
    marked = (ops == OP["ATTN"]) | (ops == OP["OPROJ"])
    S = int(words[:, :, W_END][ops == OP["ATTN"]][0])
    forced = opts.get("attn_merge", 0)
    auto = opts.get("batch", 1) == 1 and cfg.n_heads * S * cfg.head_dim * 4 > 96 * 1024
    expect = 1 if forced == 2 or (forced == 0 and auto) else 0
    if cfg is configs.LLAMA_3B and n_sm == 148 and not opts:
        assert S == 17 and expect == 1
    if cfg is configs.LLAMA_1B and n_sm == 148 and not opts:
        assert S == 6 and expect == 0
    assert marked.any()
    assert np.all(words[:, :, W_MERGE][marked] == expect)
    assert np.all(words[:, :, W_MERGE][~marked] == 0)
    base, _, inc0 = dpb.plan(cfg, n_sm, **{**opts, "attn_merge": 1})
    w2 = words.copy()
    w2[:, :, W_MERGE] = 0
    np.testing.assert_array_equal(w2, base)
    np.testing.assert_array_equal(inc, inc0)
    rc, done = dpb.simulate(words, n_instr, inc, steps=2, seed=n_sm)
    assert rc == 0 and done == 2 * int(n_instr.sum())


def test_attention_merge_option_is_checked():
    for bad in (-1, 3):
        with pytest.raises(mk.MkError) as e:
            dpb.plan(configs.LLAMA_1B, 148, attn_merge=bad)
        assert e.value.name == "MK_ERR_INVALID_ARG"
    with pytest.raises(mk.MkError) as e:
        dpb.plan(configs.LLAMA_1B, 148, attn_merge=2, batch=2)
    assert e.value.name == "MK_ERR_UNSUPPORTED"


W_GATE = 13


@pytest.mark.parametrize("cfg,opts,expect", [
    (configs.LLAMA_1B, {}, 1),                         # 680 KB of FFN per block: 10.6 stages of 64 KB
    (configs.LLAMA_1B, dict(batch=2), 1),              # 7 stages of 96 KB
    (configs.LLAMA_1B, dict(batch=8), 0),
    (configs.LLAMA_3B, {}, 0),                         # hidden 3072
    (configs.TINY, {}, 0),                             # 8 KB of FFN per block
    (configs.TINY, dict(ffn_early_stages=2), 2),
    (configs.LLAMA_1B, dict(ffn_early_stages=-1), 0),
    (configs.LLAMA_1B, dict(split_ffn=1), 0),          # no fused FFN instruction
    (configs.MIXTRAL_8L, {}, 0),                       # MoE: the routing gates the expert stream already
    (configs.MIXTRAL_8L, dict(ffn_early_stages=1), 0),
], ids=lambda x: getattr(x, "name", str(x)))
def test_ffn_gate_marks(cfg, opts, expect):
    # Every dense fused FFN instruction carries the gate (the stage from which the loader waits for the
    # FFN's dependency); nothing else does, and it changes no other word and no counter increment.
    words, n_instr, inc = dpb.plan(cfg, 148, **opts)
    ops = words[:, :, W_OP]
    ffn = ops == OP["FFN"]
    assert np.all(words[:, :, W_GATE][ffn] == expect)
    assert np.all(words[:, :, W_GATE][~ffn] == 0)
    base, _, inc0 = dpb.plan(cfg, 148, **{**opts, "ffn_early_stages": -1})
    w2 = words.copy()
    w2[:, :, W_GATE] = 0
    np.testing.assert_array_equal(w2, base)
    np.testing.assert_array_equal(inc, inc0)


def test_ffn_gate_option_is_checked():
    for bad in (-2, 65):
        with pytest.raises(mk.MkError) as e:
            dpb.plan(configs.LLAMA_1B, 148, ffn_early_stages=bad)
        assert e.value.name == "MK_ERR_INVALID_ARG"
