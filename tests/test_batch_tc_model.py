"""CPU model of the batched decode's tensor-core GEMV index math (no GPU).

With options.batch > 1 every GEMV is a skinny GEMM, y[row][q] = W[row] . x_q,
run with mma m16n8k16 (bf16, fp32 accumulate): the ring stage's weight rows,
stored at a padded pitch, are the A operand (ldmatrix), the 8 sequence slots
the N dimension, each warp one eighth of the columns; the fused FFN's
transposed down-projection rows go through ldmatrix.trans with h as the B
operand.  The activations enter as bf16 high and low parts.  This test
restates the PTX fragment layouts in numpy, runs the kernel's loops and
checks them against plain products: a wrong lane, row, column or tile index
shows up as an O(1) error, a dropped low part as an error near 2^-9.
"""
import numpy as np
import pytest

from tests.test_attention_tc_model import a_frag, bf16, c_to_lanes, frags_to_A, frags_to_B, ldmatrix, mma

WARPS = 8


def split(x):
    hi = bf16(x)
    return hi, bf16(np.float32(x) - hi)


def stage(W, pitch):
    """Rows of W (bf16 values) stored pitch elements apart, as the padded bulk copies leave them."""
    buf = np.full(W.shape[0] * pitch + 64, np.nan, np.float32)  # padding and the tail stay NaN
    for r in range(W.shape[0]):
        buf[r * pitch: r * pitch + W.shape[1]] = W[r]
    return buf


def b_frags(X, K, warp, ks):
    """Lane (g, t) of `warp`: sequence g's columns kb + 2t, 2t+1 | kb + 2t + 8, 2t + 9 (high, low parts)."""
    kb = warp * (K // WARPS) + 16 * ks
    hi, lo = [], []
    for lane in range(32):
        g, t = lane // 4, lane % 4
        vals = [X[g, kb + 2 * t], X[g, kb + 2 * t + 1], X[g, kb + 2 * t + 8], X[g, kb + 2 * t + 9]]
        h, l = zip(*(split(v) for v in vals))
        hi.append([(h[0], h[1]), (h[2], h[3])])
        lo.append([(l[0], l[1]), (l[2], l[3])])
    return hi, lo


def rows_tc(buf, pitch, nr, K, X, nb):
    """stage_rows_tc for every warp, then the epilogue's sum over warps: [nr][8] row sums per slot."""
    out = np.zeros((nr, 8))
    for warp in range(WARPS):
        for m0 in range(0, nr, 16):
            C = np.zeros((16, 8))
            for ks in range(K // (16 * WARPS)):
                col = warp * (K // WARPS) + 16 * ks
                addrs = []
                for lane in range(32):
                    ar = min(m0 + lane % 16, nr - 1)
                    addrs.append(ar * pitch + col + (lane // 16) * 8)
                A = frags_to_A([[p for p in regs] for regs in ldmatrix(buf, addrs, False)])
                hi, lo = b_frags(X, K, warp, ks)
                C = mma(A, frags_to_B(hi), C)
                C = mma(A, frags_to_B(lo), C)
            for lane, (c0, c1, c2, c3) in enumerate(c_to_lanes(C)):
                g, t = lane // 4, lane % 4
                for r, (va, vb) in ((m0 + g, (c0, c1)), (m0 + g + 8, (c2, c3))):
                    if r < nr:
                        if 2 * t < nb:
                            out[r, 2 * t] += va
                        if 2 * t + 1 < nb:
                            out[r, 2 * t + 1] += vb
    return out


@pytest.mark.parametrize("K,nr,nb", [(2048, 15, 8), (2048, 7, 5), (3072, 10, 4), (256, 40, 3), (256, 16, 8)])
def test_rows_tc_equals_plain_product(K, nr, nb):
    rng = np.random.default_rng(K + nr + nb)
    W = bf16(rng.normal(0, 0.02, (nr, K)).astype(np.float32))
    X = np.zeros((8, K), np.float32)
    X[:nb] = rng.normal(0, 1, (nb, K)).astype(np.float32)
    pitch = K + 8  # row_bytes + 16 bytes, in bf16 elements
    got = rows_tc(stage(W, pitch), pitch, nr, K, X, nb)
    want = W.astype(np.float64) @ X.astype(np.float64).T
    assert np.all(got[:, nb:] == 0)
    err = np.max(np.abs(got[:, :nb] - want[:, :nb])) / np.max(np.abs(want[:, :nb]))
    assert err < 1e-4, err  # hi + lo carry ~16 mantissa bits of x; a dropped low part gives ~4e-3


def test_padded_pitch_puts_the_rows_of_an_ldmatrix_tile_in_different_banks():
    for K in (256, 2048, 3072):
        pitch_bytes = 2 * K + 16
        banks = {((r * pitch_bytes) % 128) // 16 for r in range(8)}  # 16-byte bank groups of a row's 8 columns
        assert len(banks) == 8


def down_tc(buf, pitch, nr, H, h, nb):
    """down_rows_tc for every warp: y[col][q] over the warp's columns."""
    y = np.zeros((H, 8))
    hs = np.zeros((max(nr, 16) + 16, 8), np.float32)
    hs[:nr, :nb] = h[:nr, :nb]
    for warp in range(WARPS):
        for k0 in range(0, nr, 16):
            bh, bl = [], []
            for lane in range(32):
                g, t = lane // 4, lane % 4
                vals = [hs[k0 + r, g] if (k0 + r < nr and g < nb) else 0.0 for r in (2 * t, 2 * t + 1, 2 * t + 8, 2 * t + 9)]
                hh, ll = zip(*(split(v) for v in vals))
                bh.append([(hh[0], hh[1]), (hh[2], hh[3])])
                bl.append([(ll[0], ll[1]), (ll[2], ll[3])])
            for mt in range(H // (16 * WARPS)):
                col = warp * (H // WARPS) + 16 * mt
                addrs = []
                for lane in range(32):
                    r = k0 + lane % 8 + 8 * (lane // 16)
                    addrs.append(min(r, nr - 1) * pitch + col + 8 * ((lane // 8) % 2))
                A = frags_to_A(ldmatrix(buf, addrs, True))
                C = np.zeros((16, 8))
                C = mma(A, frags_to_B(bh), C)
                C = mma(A, frags_to_B(bl), C)
                y[col: col + 16] += C
    return y


@pytest.mark.parametrize("H,nr,nb", [(2048, 15, 8), (3072, 10, 4), (256, 40, 2), (256, 3, 8)])
def test_down_tc_equals_plain_product(H, nr, nb):
    rng = np.random.default_rng(H + nr)
    Wt = bf16(rng.normal(0, 0.02, (nr, H)).astype(np.float32))  # transposed down-projection rows
    h = np.zeros((nr, 8), np.float32)
    h[:, :nb] = rng.normal(0, 1, (nr, nb)).astype(np.float32)
    pitch = H + 8
    got = down_tc(stage(Wt, pitch), pitch, nr, H, h, nb)
    want = Wt.astype(np.float64).T @ h.astype(np.float64)
    assert np.all(got[:, nb:] == 0)
    err = np.max(np.abs(got - want)) / np.max(np.abs(want))
    assert err < 1e-4, err


def test_a_fragments_of_the_transposed_load_are_the_transposed_tile():
    # ldmatrix.trans with the lane -> (row, column block) map above delivers Wt^T exactly
    rng = np.random.default_rng(7)
    Wt = bf16(rng.normal(0, 1, (16, 64)).astype(np.float32))
    pitch = 72
    buf = stage(Wt, pitch)
    addrs = [(lane % 8 + 8 * (lane // 16)) * pitch + 16 + 8 * ((lane // 8) % 2) for lane in range(32)]
    A = frags_to_A(ldmatrix(buf, addrs, True))
    np.testing.assert_array_equal(A, Wt[:, 16:32].T)
    assert a_frag(A, 5)[0] == (Wt[2, 16 + 1], Wt[3, 16 + 1])  # lane 5: g = 1, t = 1
