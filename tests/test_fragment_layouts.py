"""The decode kernels' tensor-core fragment plumbing, emulated on the CPU.

The grouped-query block math (MmaMath and Fp8MmaMath in csrc/pa_decode.cuh)
loads K and V tiles from 128-byte-swizzled shared memory with ldmatrix, runs
m16n8k16 products with the query heads on the N = 8 side (S^T = K Q^T, then
O^T = V^T P^T with P moved across lanes by movmatrix.trans) and reads results
out of lane-distributed fragments.  Here the same index arithmetic runs on
numpy arrays, following the PTX ISA's fragment layouts, and must reproduce
the plain matrix products; every ldmatrix phase must also touch eight distinct
16-byte bank groups (no shared-memory bank conflicts).  For 1-byte E4M3 tiles
the K codes enter with head_dim permuted inside each k-step (the Q^T fragments
use the same permutation) and the V codes go through one byte permute, which
permutes the output rows; both are undone as in the kernel.
"""
import numpy as np

T, D, G = 16, 128, 4          # tokens per block, head_dim, query heads of one KV head
LANES = np.arange(32)


def tile_offset(t, c):
    """Byte offset of 16-byte chunk c of token t in a swizzled tile (the kernel's tile_offset)."""
    return ((c >> 3) * T + t) * 128 + (((c & 7) ^ (t & 7)) << 4)


def mma(C, A, B):
    """m16n8k16: A[32][4][2], B[32][2][2], C[32][4] lane fragments -> D fragments."""
    Am, Bm, Cm = np.zeros((16, 16)), np.zeros((16, 8)), np.zeros((16, 8))
    for l in range(32):
        g, t = l // 4, l % 4
        Am[g, 2 * t:2 * t + 2], Am[g + 8, 2 * t:2 * t + 2] = A[l][0], A[l][1]
        Am[g, 2 * t + 8:2 * t + 10], Am[g + 8, 2 * t + 8:2 * t + 10] = A[l][2], A[l][3]
        Bm[2 * t:2 * t + 2, g], Bm[2 * t + 8:2 * t + 10, g] = B[l][0], B[l][1]
        Cm[g, 2 * t:2 * t + 2], Cm[g + 8, 2 * t:2 * t + 2] = C[l][0:2], C[l][2:4]
    Dm = Am @ Bm + Cm
    return np.array([[Dm[l // 4, 2 * (l % 4)], Dm[l // 4, 2 * (l % 4) + 1],
                      Dm[l // 4 + 8, 2 * (l % 4)], Dm[l // 4 + 8, 2 * (l % 4) + 1]] for l in range(32)])


def movmatrix_trans(x):
    """movmatrix.sync.trans of an 8x8 matrix held two values per lane."""
    X = np.zeros((8, 8))
    for l in range(32):
        X[l // 4, 2 * (l % 4):2 * (l % 4) + 2] = x[l]
    Y = X.T
    return np.array([Y[l // 4, 2 * (l % 4):2 * (l % 4) + 2] for l in range(32)])


def accum_rows(S):
    """S^T [16 tokens][8 heads] from the accumulator fragments."""
    ST = np.zeros((16, 8))
    for l in range(32):
        g, t = l // 4, l % 4
        ST[g, 2 * t:2 * t + 2], ST[g + 8, 2 * t:2 * t + 2] = S[l, 0:2], S[l, 2:4]
    return ST


def conflict_free(addresses):
    """Each 8-lane phase of an ldmatrix.x4 reads 8 rows: 8 distinct 16-byte bank groups."""
    return all(len({(a % 128) // 16 for a in addresses[8 * m:8 * m + 8]}) == 8 for m in range(4))


def test_bf16_block_math():
    rng = np.random.default_rng(0)
    K, V, Q = rng.standard_normal((T, D)), rng.standard_normal((T, D)), rng.standard_normal((G, D))
    sm = {}
    for name, X in (("K", K), ("V", V)):
        s = np.full(T * D, np.nan)               # element view of the tile (2-byte elements)
        for t in range(T):
            for c in range(16):
                o = tile_offset(t, c) // 2
                s[o:o + 8] = X[t, 8 * c:8 * c + 8]
        assert not np.isnan(s).any()
        sm[name] = s

    def ldmatrix_x4(s, addrs, trans=False):
        regs = np.zeros((32, 4, 2))
        for m in range(4):
            M = np.array([s[addrs[8 * m + r] // 2:addrs[8 * m + r] // 2 + 8] for r in range(8)])
            M = M.T if trans else M
            for l in range(32):
                regs[l, m] = M[l // 4, 2 * (l % 4):2 * (l % 4) + 2]
        return regs

    mi, ri = LANES >> 3, LANES & 7
    qf = np.zeros((8, 32, 2, 2))                  # Q^T fragments per 16-wide k-step
    for c in range(8):
        for l in range(32):
            gid, tig = l >> 2, l & 3
            if gid < G:
                qf[c, l, 0] = Q[gid, 16 * c + 2 * tig:16 * c + 2 * tig + 2]
                qf[c, l, 1] = Q[gid, 16 * c + 8 + 2 * tig:16 * c + 8 + 2 * tig + 2]
    S = np.zeros((32, 4))
    for c in range(8):
        addrs = [tile_offset(ri[l] + 8 * (mi[l] & 1), 2 * c + (mi[l] >> 1)) for l in range(32)]
        assert conflict_free(addrs)
        S = mma(S, ldmatrix_x4(sm["K"], addrs), qf[c])
    Qp = np.zeros((8, D))
    Qp[:G] = Q
    ST = accum_rows(S)
    assert np.allclose(ST, K @ Qp.T)
    # P^T from the score fragments (S itself stands in for P: the check is linear)
    B = np.stack([movmatrix_trans(S[:, 0:2]), movmatrix_trans(S[:, 2:4])], axis=1)
    OT = np.zeros((D, 8))
    for m in range(8):
        addrs = [tile_offset(ri[l] + 8 * (mi[l] >> 1), 2 * m + (mi[l] & 1)) for l in range(32)]
        assert conflict_free(addrs)
        O = mma(np.zeros((32, 4)), ldmatrix_x4(sm["V"], addrs, trans=True), B)
        for l in range(32):
            g, t = l // 4, l % 4
            OT[16 * m + g, 2 * t:2 * t + 2], OT[16 * m + g + 8, 2 * t:2 * t + 2] = O[l, 0:2], O[l, 2:4]
    assert np.allclose(OT, V.T @ ST)


def test_fp8_block_math():
    rng = np.random.default_rng(1)
    Kc = rng.integers(0, 256, (T, D)).astype(np.uint8)     # code bytes; the plumbing treats each as a number
    Vc = rng.integers(0, 256, (T, D)).astype(np.uint8)
    Q = rng.standard_normal((G, D))

    def to_smem(X):                                        # 128-byte rows: 8 chunks of 16 codes
        s = np.zeros(T * 128, dtype=np.uint8)
        for t in range(T):
            for c in range(8):
                o = tile_offset(t, c)
                s[o:o + 16] = X[t, 16 * c:16 * c + 16]
        return s

    smK, smV = to_smem(Kc), to_smem(Vc)

    def ldmatrix_b16(s, addrs, trans):                     # 16-bit units = code pairs; 4 bytes per register
        regs = [[None] * 4 for _ in range(32)]
        for m in range(4):
            M = np.array([s[addrs[8 * m + r]:addrs[8 * m + r] + 16].reshape(8, 2) for r in range(8)])
            for l in range(32):
                g, t = l // 4, l % 4
                e0, e1 = (M[2 * t][g], M[2 * t + 1][g]) if trans else (M[g][2 * t], M[g][2 * t + 1])
                regs[l][m] = np.concatenate([e0, e1])
        return regs

    def cvt2(b):                                           # cvt.rn.f16x2.e4m3x2: low byte -> low half
        return np.array([float(b[0]), float(b[1])])

    off = [[tile_offset((l & 7) + 8 * ((l >> 3) & 1), 2 * x + ((l >> 3) >> 1)) for l in range(32)] for x in range(4)]
    assert all(conflict_free(o) for o in off)
    qf = np.zeros((8, 32, 2, 2))      # head_dim permuted inside each k-step: slots 2t,2t+1,2t+8,2t+9 <-> d 4t..4t+3
    for c in range(8):
        for l in range(32):
            g, t = l // 4, l % 4
            if g < G:
                qf[c, l, 0] = Q[g, 16 * c + 4 * t:16 * c + 4 * t + 2]
                qf[c, l, 1] = Q[g, 16 * c + 4 * t + 2:16 * c + 4 * t + 4]
    S = np.zeros((32, 4))
    for x in range(4):
        r = ldmatrix_b16(smK, off[x], False)
        for kk in range(2):
            A = [[cvt2(r[l][2 * kk][0:2]), cvt2(r[l][2 * kk + 1][0:2]), cvt2(r[l][2 * kk][2:4]),
                  cvt2(r[l][2 * kk + 1][2:4])] for l in range(32)]
            S = mma(S, A, qf[2 * x + kk])
    Qp = np.zeros((8, D))
    Qp[:G] = Q
    ST = accum_rows(S)
    assert np.allclose(ST, Kc.astype(float) @ Qp.T)
    B = [[b0, b1] for b0, b1 in zip(movmatrix_trans(S[:, 0:2]), movmatrix_trans(S[:, 2:4]))]
    OT = np.zeros((D, 8))
    for x in range(4):
        r = ldmatrix_b16(smV, off[x], True)
        for kk in range(2):
            # (token 2t: d0 d1 | token 2t+1: d0 d1) -> (d0: 2t 2t+1 | d1: 2t 2t+1)
            lo = [r[l][2 * kk][[0, 2, 1, 3]] for l in range(32)]
            hi = [r[l][2 * kk + 1][[0, 2, 1, 3]] for l in range(32)]
            A = [[cvt2(lo[l][0:2]), cvt2(lo[l][2:4]), cvt2(hi[l][0:2]), cvt2(hi[l][2:4])] for l in range(32)]
            O = mma(np.zeros((32, 4)), A, B)
            m = 2 * x + kk                                # output rows d = 16m + 2g (c0, c1) and 16m + 2g + 1 (c2, c3)
            for l in range(32):
                g, t = l // 4, l % 4
                OT[16 * m + 2 * g, 2 * t:2 * t + 2], OT[16 * m + 2 * g + 1, 2 * t:2 * t + 2] = O[l, 0:2], O[l, 2:4]
    assert np.allclose(OT, Vc.astype(float).T @ ST)


def test_fma_path_reads_are_conflict_free():
    """The CUDA-core path (fp32 / MHA): QK lane (token lane&15, half lane>>4)
    and PV lane (token pair 2i + lane>>4, chunk lane&15) address patterns."""
    assert all(len({(tile_offset(l & 15, (l >> 4) * 8 + c) % 128) // 16 for l in range(8 * ph, 8 * ph + 8)}) == 8
               for c in range(8) for ph in range(4))
    assert all(len({(tile_offset(2 * i + (l >> 4), l & 15) % 128) // 16 for l in range(8 * ph, 8 * ph + 8)}) == 8
               for i in range(8) for ph in range(4))


def test_emulation_catches_a_wrong_swizzle():
    """A tile offset without the XOR swizzle makes the K reads conflict."""
    def plain(t, c):
        return ((c >> 3) * T + t) * 128 + ((c & 7) << 4)
    mi, ri = LANES >> 3, LANES & 7
    addrs = [plain(ri[l] + 8 * (mi[l] & 1), 2 * 0 + (mi[l] >> 1)) for l in range(32)]
    assert not conflict_free(addrs)


def test_tile_offset_is_where_the_tma_box_lands():
    """The decode tiles arrive by TMA (box {128 B, 1, 1, 16 tokens, 1} per
    128-byte half, 128-byte swizzle: 16-byte chunk j of a 128-byte row moves to
    j ^ (row within the 1024-byte atom)); tile_offset must name the same bytes."""
    def swizzled(logical):
        return logical ^ (((logical >> 7) & 7) << 4)
    for t in range(T):
        for c in range(16):
            half, j = c >> 3, c & 7
            assert tile_offset(t, c) == swizzled(half * T * 128 + t * 128 + j * 16)
