"""CPU model of the tensor-core decode attention's index math (no GPU).

The head_dim-64 attention computes each split with mma m16n8k16 (bf16 A
row-major, bf16 B column-major, fp32 accumulate) on K/V rows that TMA wrote
into shared memory with the 128-byte swizzle, loaded as fragments by
ldmatrix (.trans for V).  This test restates those layouts from the PTX ISA
in numpy, runs the kernel's tile loop (q and the probabilities split into bf16
high and low parts in rows 0-3 and 4-7, online softmax over 16-position
tiles), and checks the result against exact attention.  A wrong fragment
index, swizzle term or hi/lo row would show up as an O(1) error.
"""
import numpy as np
import pytest


def bf16(x):
    x = np.asarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32)

def mma(A, B, C):  # A [16,16], B [16,8] (k x n), C [16,8]
    return C + A.astype(np.float64) @ B.astype(np.float64)

# ---- fragment extraction per lane (PTX ISA m16n8k16 .bf16 layouts)
def a_frag(A, lane):
    g, t = lane // 4, lane % 4
    return [(A[g, 2*t], A[g, 2*t+1]), (A[g+8, 2*t], A[g+8, 2*t+1]),
            (A[g, 2*t+8], A[g, 2*t+9]), (A[g+8, 2*t+8], A[g+8, 2*t+9])]
def frags_to_A(fr):  # fr[lane] = 4 pairs -> A [16,16]
    A = np.zeros((16,16), np.float32)
    for lane in range(32):
        g, t = lane // 4, lane % 4
        (a0,a1),(a2,a3),(a4,a5),(a6,a7) = fr[lane]
        A[g,2*t],A[g,2*t+1]=a0,a1; A[g+8,2*t],A[g+8,2*t+1]=a2,a3
        A[g,2*t+8],A[g,2*t+9]=a4,a5; A[g+8,2*t+8],A[g+8,2*t+9]=a6,a7
    return A
def frags_to_B(fr):  # fr[lane] = [(b0,b1),(b2,b3)] ; B[k][n]
    B = np.zeros((16,8), np.float32)
    for lane in range(32):
        g, t = lane // 4, lane % 4
        (b0,b1),(b2,b3) = fr[lane]
        B[2*t, g], B[2*t+1, g], B[2*t+8, g], B[2*t+9, g] = b0, b1, b2, b3
    return B
def c_to_lanes(C):
    out = []
    for lane in range(32):
        g, t = lane // 4, lane % 4
        out.append((C[g,2*t], C[g,2*t+1], C[g+8,2*t], C[g+8,2*t+1]))
    return out

# ---- swizzled stage: half-boxes of 64 bf16 columns, rows of 128 B, chunk c of row r at c ^ (r & 7)
def stage_store(M, rps):  # M [rows<=rps][D] -> flat bf16 array as stored by TMA (SWIZZLE_128B)
    D = M.shape[1]; halves = D // 64
    buf = np.zeros(halves * rps * 64, np.float32)
    for h in range(halves):
        for r in range(M.shape[0]):
            for c in range(8):
                pc = c ^ (r & 7)
                buf[h*rps*64 + r*64 + pc*8: h*rps*64 + r*64 + pc*8 + 8] = M[r, h*64 + c*8: h*64 + c*8 + 8]
    return buf
def addr(rps, r, d):  # element index in the stage buffer
    h, dd = d // 64, d % 64
    c = dd // 8
    return h*rps*64 + r*64 + ((c ^ (r & 7)) * 8) + (dd % 8)
def ldmatrix(buf, row_addr, trans):
    # row_addr[lane] for lanes 0..31: 4 matrices, lanes 8i..8i+7 give matrix i's rows (8 consecutive bf16)
    mats = [np.array([buf[row_addr[8*i + j]: row_addr[8*i + j] + 8] for j in range(8)]) for i in range(4)]
    out = []
    for lane in range(32):
        g, t = lane // 4, lane % 4
        regs = []
        for M in mats:
            if not trans: regs.append((M[g, 2*t], M[g, 2*t+1]))
            else: regs.append((M[2*t, g], M[2*t+1, g]))
        out.append(regs)
    return out



def attention_tc_model(q, K, V, rps):
    """The kernel's tile loop over one stage of nrows <= rps cached rows."""
    G, D = q.shape
    nrows = K.shape[0]
    Kb, Vb = stage_store(K, rps), stage_store(V, rps)
    qhi = bf16(q)
    qlo = bf16(q - qhi)
    Qfull = np.zeros((16, D), np.float32)
    Qfull[:G] = qhi
    Qfull[4:4 + G] = qlo
    m = np.full(4, -np.inf)
    l = np.zeros(4)
    O = [np.zeros((16, 8)) for _ in range(D // 8)]
    for tile in range((nrows + 15) // 16):
        base = tile * 16
        S = [np.zeros((16, 8)) for _ in range(2)]
        for kk in range(D // 16):
            ra = [addr(rps, base + (8 if lane // 8 >= 2 else 0) + lane % 8, kk * 16 + (8 if (lane // 8) % 2 else 0))
                  for lane in range(32)]
            fr = ldmatrix(Kb, ra, trans=False)
            for nh in range(2):
                S[nh] = mma(Qfull[:, kk * 16:(kk + 1) * 16], frags_to_B([[fr[x][2 * nh], fr[x][2 * nh + 1]] for x in range(32)]), S[nh])
        Sc = np.concatenate(S, axis=1)
        sc = Sc[0:4] + Sc[4:8]
        valid = np.array([base + n < nrows for n in range(16)])
        sc[:, ~valid] = -np.inf
        mn = np.maximum(m, sc.max(axis=1))
        al = np.where(np.isinf(m), 0.0, np.exp2(m - mn))
        p = np.exp2(sc - mn[:, None])
        p[:, ~valid] = 0
        l = l * al + p.sum(axis=1)
        phi = bf16(p.astype(np.float32))
        P = np.zeros((16, 16), np.float32)
        P[0:4] = phi
        P[4:8] = bf16((p - phi).astype(np.float32))
        for nt in range(D // 8):
            O[nt][0:8] *= np.concatenate([al, al])[:, None]
        for n2 in range(D // 16):
            ra = [addr(rps, base + (8 if (lane // 8) % 2 else 0) + lane % 8, (2 * n2 + (1 if lane // 8 >= 2 else 0)) * 8)
                  for lane in range(32)]
            fr = ldmatrix(Vb, ra, trans=True)
            for half in range(2):
                O[2 * n2 + half] = mma(P, frags_to_B([[fr[x][2 * half], fr[x][2 * half + 1]] for x in range(32)]), O[2 * n2 + half])
        m = mn
    Of = np.concatenate(O, axis=1)
    return ((Of[0:4] + Of[4:8]) / l[:, None])[:G]


@pytest.mark.parametrize("D,G,nrows", [(64, 4, 45), (64, 2, 16), (128, 4, 37), (128, 3, 64), (64, 1, 1)])
def test_tensor_core_attention_model_matches_exact_attention(D, G, nrows):
    rng = np.random.default_rng(D * 100 + G * 10 + nrows)
    rps = min((16384 // D) & ~63, 256)
    K = bf16(rng.standard_normal((nrows, D)))
    V = bf16(rng.standard_normal((nrows, D)))
    q = rng.standard_normal((G, D)).astype(np.float32) * np.float32(1.4426950408889634 / np.sqrt(D))
    out = attention_tc_model(q, K, V, rps)
    s = q.astype(np.float64) @ K.T.astype(np.float64)
    pr = np.exp2(s - s.max(axis=1, keepdims=True))
    ref = (pr / pr.sum(axis=1, keepdims=True)) @ V.astype(np.float64)
    assert np.abs(out - ref).max() <= 2e-5 * np.abs(ref).max()


def test_swizzled_stage_addressing_is_a_bijection():
    rps, D = 64, 128
    seen = set(addr(rps, r, d) for r in range(rps) for d in range(D))
    assert len(seen) == rps * D and min(seen) == 0 and max(seen) == rps * D - 1
