"""CPU model of the split-attention merge (no GPU).

Split-KV decoding combines S partial results of one query head: split s holds
the unnormalised output o_s = sum_j 2^(x_j - m_s) v_j, its running maximum m_s
(log2 domain) and its sum l_s = sum_j 2^(x_j - m_s).  The attention output is
sum_s 2^(m_s - M) o_s / sum_s 2^(m_s - M) l_s with M = max_s m_s.  The kernels
take the splits in groups per round trip (8 or 4 in every O-projection block,
16 in the last split of a kv head) with an online rescale between groups, and
skip groups whose splits are all empty (m = -inf, o = 0, l = 0).  This test
restates that grouped loop in numpy and checks it against exact softmax
attention over the concatenated positions, for every group size the kernels
use, with empty splits first, in the middle and last.  A wrong rescale factor,
a dropped group or an empty group that poisons the sums with NaN would fail.
"""
import numpy as np
import pytest


def split_partials(scores, values, bounds):
    """Per split (o, m, l) in the kernels' convention: log2-domain scores, unnormalised o."""
    parts = []
    for b0, b1 in bounds:
        if b1 <= b0:
            parts.append((np.zeros(values.shape[1]), -np.inf, 0.0))
            continue
        x = scores[b0:b1]
        m = x.max()
        p = np.exp2(x - m)
        parts.append((p @ values[b0:b1], m, p.sum()))
    return parts


def grouped_merge(parts, group):
    """The kernels' loop: `group` splits per round trip, online rescale, empty groups skipped."""
    M, den = -np.inf, 0.0
    acc = np.zeros_like(parts[0][0])
    for s0 in range(0, len(parts), group):
        blk = parts[s0:s0 + group]
        bm = max([M] + [m for _, m, _ in blk])
        if bm == -np.inf:
            continue
        r = np.exp2(M - bm)
        den *= r
        acc = acc * r
        for o, m, l in blk:
            f = np.exp2(m - bm)
            den += f * l
            acc = acc + f * o
        M = bm
    return acc / den


def exact(scores, values):
    p = np.exp2(scores - scores.max())
    return (p / p.sum()) @ values


@pytest.mark.parametrize("group", [4, 8, 16])
@pytest.mark.parametrize("n_splits", [1, 3, 6, 9, 17, 18, 40])
@pytest.mark.parametrize("empty", ["none", "first", "middle", "last"])
def test_grouped_merge_equals_exact_attention(group, n_splits, empty):
    rng = np.random.default_rng(1000 * group + 10 * n_splits + len(empty))
    d, per = 64, 23
    n = per * n_splits
    scores = rng.normal(0, 3, n)            # log2-domain scores (q.k / sqrt(d) / ln 2)
    values = rng.normal(0, 1, (n, d))
    bounds = [(s * per, (s + 1) * per) for s in range(n_splits)]
    if empty != "none" and n_splits > 1:
        k = {"first": 0, "middle": n_splits // 2, "last": n_splits - 1}[empty]
        bounds[k] = (bounds[k][0], bounds[k][0])  # an empty split: its positions are not attended
    keep = np.concatenate([np.arange(b0, b1) for b0, b1 in bounds])
    ref = exact(scores[keep], values[keep])
    got = grouped_merge(split_partials(scores, values, bounds), group)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_all_empty_groups_before_the_first_position_are_skipped():
    # positions only in the last split (a short context over many splits): the leading groups are
    # all empty and must leave the running state untouched
    rng = np.random.default_rng(7)
    d, n_splits = 16, 20
    scores = rng.normal(0, 2, 5)
    values = rng.normal(0, 1, (5, d))
    parts = [(np.zeros(d), -np.inf, 0.0)] * (n_splits - 1) + split_partials(scores, values, [(0, 5)])
    for group in (4, 8, 16):
        got = grouped_merge(parts, group)
        assert np.all(np.isfinite(got))
        np.testing.assert_allclose(got, exact(scores, values), rtol=1e-12, atol=1e-12)


def test_group_size_does_not_change_the_result_beyond_rounding():
    # the per-block merge (8 or 4 per round trip) and the once-per-head merge (16) agree
    rng = np.random.default_rng(3)
    d, n_splits, per = 128, 17, 128
    scores = rng.normal(0, 4, n_splits * per)
    values = rng.normal(0, 1, (n_splits * per, d))
    parts = split_partials(scores, values, [(s * per, (s + 1) * per) for s in range(n_splits)])
    a, b, c = (grouped_merge(parts, g) for g in (4, 8, 16))
    np.testing.assert_allclose(a, c, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(b, c, rtol=1e-12, atol=1e-13)
