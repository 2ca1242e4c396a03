"""Per-opcode GPU parity: the standalone attention op (through the C ABI)
against the oracle's attention of each query head (fp64), including empty
splits, a single position, ragged split sizes and every group size."""
import numpy as np
import pytest

import oracle
import synth

pytestmark = pytest.mark.gpu


def _case(rng, nq, nkv, d, n_pos, max_seq):
    q = rng.standard_normal((nq, d)).astype(np.float32)
    kc = synth.f32_to_bf16(rng.standard_normal((nkv, max_seq, d)).astype(np.float32))
    vc = synth.f32_to_bf16(rng.standard_normal((nkv, max_seq, d)).astype(np.float32))
    ref = np.stack([oracle.attend(q[h].astype(np.float64), kc[h // (nq // nkv), :n_pos],
                                  vc[h // (nq // nkv), :n_pos]) for h in range(nq)])
    return q, kc, vc, ref


@pytest.mark.parametrize("nq,nkv,d", [(4, 2, 64), (8, 8, 64), (24, 8, 128), (32, 8, 64), (12, 4, 128), (4, 1, 128)])
@pytest.mark.parametrize("n_pos,splits", [(1, 1), (1, 7), (7, 3), (64, 5), (1000, 18), (4097, 18), (300, 400)])
def test_attention_decode_matches_oracle(cuda, nq, nkv, d, n_pos, splits):
    import torch
    from decode_persistent_block_b200 import mk
    rng = np.random.default_rng(nq * 1000 + n_pos + splits)
    max_seq = n_pos + 3
    q, kc, vc, ref = _case(rng, nq, nkv, d, n_pos, max_seq)
    tq = torch.from_numpy(q).cuda()
    tk = torch.from_numpy(kc.view(np.int16)).cuda()
    tv = torch.from_numpy(vc.view(np.int16)).cuda()
    out = torch.empty_like(tq)
    mk.attention_decode(tq, tk, tv, n_pos, splits, out)
    got = out.cpu().numpy().astype(np.float64)
    assert np.max(np.abs(got - ref)) <= 1e-5 * max(1.0, np.max(np.abs(ref))), np.max(np.abs(got - ref))


def test_attention_decode_argument_errors(cuda):
    import torch
    from decode_persistent_block_b200 import mk
    q = torch.zeros(4, 64, device="cuda")
    kv = torch.zeros(2, 8, 64, dtype=torch.int16, device="cuda")
    out = torch.empty_like(q)
    ws = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(mk.MkError) as e:
        mk.attention_decode(q, kv, kv, 4, 2, out, workspace=ws)  # workspace too small
    assert e.value.name == "MK_ERR_CAPACITY"
    with pytest.raises(mk.MkError) as e:
        mk.attention_decode(q, kv, kv, 9, 2, out)  # n_pos > max_seq
    assert e.value.name == "MK_ERR_INVALID_ARG"
    with pytest.raises(mk.MkError) as e:
        mk.attention_decode(torch.zeros(4, 96, device="cuda"), kv, kv, 4, 2, torch.zeros(4, 96, device="cuda"))
    assert e.value.name == "MK_ERR_UNSUPPORTED"
