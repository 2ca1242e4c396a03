"""The attention entry point for callers that cannot allocate device memory.

mk_attention_decode_noalloc keeps its split partials in a fixed device array
inside the library instead of a caller workspace, for code where cudaMalloc is
not allowed (device memory owned by another allocator, or a decode loop that
must not allocate).  It must give the same result as mk_attention_decode on
two calls in a row (the shared scratch keeps the previous call's contents) and
reject shapes whose partials do not fit.  This file is collected last, and it
passes alone in a fresh process as well as after the other tests.
"""
import ctypes

import numpy as np
import pytest

import oracle
import synth

pytestmark = pytest.mark.gpu


def _inputs(rng, nq, nkv, d, n_pos, max_seq):
    import torch
    q = torch.from_numpy(rng.standard_normal((nq, d)).astype(np.float32)).cuda()
    kc = synth.f32_to_bf16(rng.standard_normal((nkv, max_seq, d)).astype(np.float32))
    vc = synth.f32_to_bf16(rng.standard_normal((nkv, max_seq, d)).astype(np.float32))
    return q, torch.from_numpy(kc.view(np.int16)).cuda(), torch.from_numpy(vc.view(np.int16)).cuda()


@pytest.mark.parametrize("nq,nkv,d,n_pos,splits", [(32, 8, 64, 1100, 18), (24, 8, 128, 2100, 18), (4, 2, 64, 5, 9)])
def test_noalloc_matches_workspace_entry_point_twice(cuda, nq, nkv, d, n_pos, splits):
    import torch
    from decode_persistent_block_b200 import mk
    rng = np.random.default_rng(n_pos)
    for call in range(2):  # two calls in a row, different inputs, same shared scratch
        q, kc, vc = _inputs(rng, nq, nkv, d, n_pos, n_pos + 7)
        ref = torch.empty_like(q)
        got = torch.full_like(q, float("nan"))
        mk.attention_decode(q, kc, vc, n_pos, splits, ref)
        mk.attention_decode_noalloc(q, kc, vc, n_pos, splits, got)
        torch.cuda.synchronize()
        r, g = ref.cpu().numpy(), got.cpu().numpy()
        assert np.all(np.isfinite(g)), call
        assert np.max(np.abs(g - r)) <= 1e-5 * max(1.0, np.max(np.abs(r))), (call, np.max(np.abs(g - r)))


def test_noalloc_rejects_sizes_beyond_its_scratch(cuda):
    import torch
    from decode_persistent_block_b200 import mk
    lib = mk.load()
    nq, d = 32, 128
    splits = mk.NOALLOC_SCRATCH_BYTES // (4 * nq * (d + 2)) + 1  # one split too many
    assert lib.mk_attention_workspace_bytes(nq, d, splits) > mk.NOALLOC_SCRATCH_BYTES
    q, kc, vc = _inputs(np.random.default_rng(1), nq, 8, d, 64, 64)
    out = torch.empty_like(q)
    with pytest.raises(mk.MkError) as e:
        mk.attention_decode_noalloc(q, kc, vc, 64, splits, out)
    assert e.value.name == "MK_ERR_CAPACITY"
    # the largest split count that fits still runs and agrees
    ok = splits - 1
    ref = torch.empty_like(q)
    mk.attention_decode(q, kc, vc, 64, ok, ref)
    mk.attention_decode_noalloc(q, kc, vc, 64, ok, out)
    torch.cuda.synchronize()
    assert np.max(np.abs(out.cpu().numpy() - ref.cpu().numpy())) <= 1e-5 * max(1.0, ref.abs().max().item())


def _oracle_attention(q, kc, vc, n_pos):
    """fp64 attention of every query head (the oracle's definition) on the bf16 caches."""
    qh, k16, v16 = q.cpu().numpy(), kc.cpu().numpy().view(np.uint16), vc.cpu().numpy().view(np.uint16)
    nq, nkv = qh.shape[0], k16.shape[0]
    return np.stack([oracle.attend(qh[h].astype(np.float64), k16[h // (nq // nkv), :n_pos],
                                   v16[h // (nq // nkv), :n_pos]) for h in range(nq)])


def test_noalloc_matches_oracle_after_a_larger_call(cuda):
    """A call with many splits and heads fills more of the shared scratch than
    the call after it; the second call, with fewer splits and heads, must not
    read any partial the first one left behind: both match the fp64 oracle."""
    import torch
    from decode_persistent_block_b200 import mk
    rng = np.random.default_rng(7)
    for nq, nkv, d, n_pos, splits in ((32, 8, 128, 3000, 40), (4, 2, 64, 37, 3)):
        q, kc, vc = _inputs(rng, nq, nkv, d, n_pos, n_pos + 5)
        got = torch.full_like(q, float("nan"))
        mk.attention_decode_noalloc(q, kc, vc, n_pos, splits, got)
        torch.cuda.synchronize()
        ref = _oracle_attention(q, kc, vc, n_pos)
        g = got.cpu().numpy().astype(np.float64)
        assert np.max(np.abs(g - ref)) <= 1e-5 * max(1.0, np.max(np.abs(ref))), (nq, splits, np.max(np.abs(g - ref)))
