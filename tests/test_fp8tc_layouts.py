"""The tcgen05 E4M3 decode kernel's operands and arithmetic, emulated on the CPU.

csrc/pa_decode_fp8tc.cuh lands a tile of 128 tokens as eight TMA boxes (16
rows of 128 one-byte codes, hardware 128-byte swizzle) for K and for V, writes
three E4M3 parts of q and of P per head with byte stores that apply the swizzle
themselves, and hands the tensor cores shared-memory descriptors: K-major K
and q parts for S^T = K Qp^T, MN-major V and K-major P parts for
O^T = V^T Pp^T, each product K = 32 codes deep.  Here the descriptors'
addressing reads back the operands from an emulated shared memory and the
products are formed in fp64 from those reads; they must equal the products
of the logical matrices.  Then the kernel's whole arithmetic for one CTA
(part splits, tile maxima, online softmax one tile behind, P parts) is run in
numpy and compared with fp64 attention on the dequantised cache: the error
must sit well inside the 16-bit decode tolerance.
"""
import numpy as np
import torch

TILE = 128                      # tokens per tile
STAGE = 2 * TILE * 128          # K tile then V tile


def e4m3_values():
    return torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()


VAL = e4m3_values()


def e4m3_rn(x):
    """Nearest-even E4M3 code of each |x| <= 448 (the cvt.rn.satfinite the kernel uses)."""
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def split3(x):
    """The kernel's three parts: x = v(c1) + v(c2) / 16 + v(c3) / 256 + r, remainders exact in fp32."""
    x = np.asarray(x, np.float32)
    codes = []
    for j in range(3):
        c = e4m3_rn(x)
        codes.append(c)
        x = ((x - VAL[c].astype(np.float32)) * np.float32(16)).astype(np.float32)
    return codes


def swz(a):
    return a ^ (((a >> 7) & 7) << 4)


def sw128_byte(n, col):
    """The kernel's sw128_byte (generic stores apply the swizzle themselves)."""
    return (n >> 3) * 1024 + (n & 7) * 128 + ((((col >> 4) ^ n) & 7) << 4) + (col & 15)


def read_kmajor8(sm, start, sbo, rows):
    """K-major 8-bit operand: rows x 32 codes, 128-byte rows, 8-row groups sbo apart."""
    r = np.arange(rows)[:, None]
    k = np.arange(32)[None, :]
    return sm[swz(start + (r % 8) * 128 + (r // 8) * sbo + k)]


def read_mnmajor8(sm, start, lbo, sbo, nmn):
    """MN-major 8-bit operand: 32 (K) x nmn codes; 128-element MN groups lbo apart,
    consecutive K in consecutive 128-byte rows, 8-row K groups sbo apart."""
    k = np.arange(32)[:, None]
    mn = np.arange(nmn)[None, :]
    return sm[swz(start + (mn % 128) + (mn // 128) * lbo + (k % 8) * 128 + (k // 8) * sbo)]


def tma_tile(sm, base, blocks):
    """Eight 16-token boxes of 128-byte rows at base + k * 2048 (hardware swizzle)."""
    for k, X in enumerate(blocks):
        for t in range(16):
            for c in range(128):
                sm[swz(base + k * 2048 + t * 128 + c)] = X[t, c]


def test_qk_and_pv_operands_read_back_the_logical_matrices():
    rng = np.random.default_rng(3)
    N = 16
    Kc = rng.integers(0, 256, (TILE, 128), dtype=np.uint8)      # codes [token][d]
    Vc = rng.integers(0, 256, (TILE, 128), dtype=np.uint8)
    Kc[(VAL[Kc] != VAL[Kc])] = 0                                # no NaN codes in a cache
    Vc[(VAL[Vc] != VAL[Vc])] = 0
    Qp = rng.integers(0, 120, (N, 128), dtype=np.uint8)         # q parts [n][d]
    Pp = rng.integers(0, 120, (N, TILE), dtype=np.uint8)        # P parts [n][token]
    st = 1                                                      # stage 1 of the ring
    kQp, kPp = 3 * STAGE, 3 * STAGE + N * 128
    sm = np.zeros(kPp + 2 * N * 128, np.uint8)
    tma_tile(sm, st * STAGE, [Kc[16 * k:16 * k + 16] for k in range(8)])
    tma_tile(sm, st * STAGE + TILE * 128, [Vc[16 * k:16 * k + 16] for k in range(8)])
    for n in range(N):
        for c in range(128):
            sm[kQp + sw128_byte(n, c)] = Qp[n, c]
            sm[kPp + N * 128 + sw128_byte(n, c)] = Pp[n, c]     # P buffer 1
    # S^T = K Qp^T: A (K-major) at stage + kk * 32, B (K-major) at kQp + kk * 32
    S = np.zeros((TILE, N))
    for kk in range(4):
        A = read_kmajor8(sm, st * STAGE + kk * 32, 1024, TILE)
        B = read_kmajor8(sm, kQp + kk * 32, 1024, N)
        assert np.array_equal(A, Kc[:, 32 * kk:32 * kk + 32])
        assert np.array_equal(B, Qp[:, 32 * kk:32 * kk + 32])
        S += VAL[A] @ VAL[B].T
    assert np.array_equal(S, VAL[Kc] @ VAL[Qp].T)
    # O^T = V^T Pp^T: A (MN-major) at stage + 16 KiB + kk * 4096, B (K-major) at P buffer + kk * 32
    O = np.zeros((128, N))
    for kk in range(4):
        A = read_mnmajor8(sm, st * STAGE + TILE * 128 + kk * 4096, 16, 1024, 128)   # [32 tok][128 d]
        B = read_kmajor8(sm, kPp + N * 128 + kk * 32, 1024, N)                       # [N][32 tok]
        assert np.array_equal(A, Vc[32 * kk:32 * kk + 32, :])
        assert np.array_equal(B, Pp[:, 32 * kk:32 * kk + 32])
        O += VAL[A].T @ VAL[B].T
    assert np.array_equal(O, VAL[Vc].T @ VAL[Pp].T)


def test_emulation_catches_a_wrong_k_step():
    rng = np.random.default_rng(4)
    Vc = rng.integers(0, 100, (TILE, 128), dtype=np.uint8)
    sm = np.zeros(STAGE, np.uint8)
    tma_tile(sm, TILE * 128, [Vc[16 * k:16 * k + 16] for k in range(8)])
    A = read_mnmajor8(sm, TILE * 128 + 1 * 2048, 16, 1024, 128)   # a k-step of 2 KiB instead of 4 KiB
    assert not np.array_equal(A, Vc[32:64, :])


def test_three_parts_hold_q_and_p():
    rng = np.random.default_rng(5)
    # q: bf16-valued, scaled so max |x| in [128, 256)
    q = torch.from_numpy(rng.standard_normal((64, 128)).astype(np.float32)).to(torch.bfloat16).float().numpy()
    e = 7 - np.floor(np.log2(np.abs(q).max(axis=1, keepdims=True)))
    x = (q * 2.0 ** e).astype(np.float32)
    c = split3(x)
    back = VAL[c[0]] + VAL[c[1]] / 16 + VAL[c[2]] / 256
    err = np.abs(back - x.astype(np.float64))
    assert (err <= 2.0 ** -12 * np.abs(x) + 2.0 ** -17).all()
    # P in (0, 1] scaled by 256, including tiny weights
    p = np.concatenate([rng.random(4000), 2.0 ** -rng.uniform(0, 30, 4000), [1.0]]).astype(np.float32)
    c = split3(p * np.float32(256))
    back = (VAL[c[0]] + VAL[c[1]] / 16 + VAL[c[2]] / 256) / 256
    err = np.abs(back - p.astype(np.float64))
    assert (err <= 2.0 ** -12 * p + 2.0 ** -25).all()


def _kernel_arith(q, Kc, Vc, k_scale, v_scale, scale):
    """One CTA's arithmetic as the kernel orders it; returns out [G][128]."""
    G = q.shape[0]
    L = Kc.shape[0]
    c_log2 = np.float32(scale * np.log2(np.e) * k_scale)
    mx = np.abs(q).max(axis=1)
    e = np.where(mx > 0, 7 - np.floor(np.log2(mx)), 0)
    ch = (c_log2 * 2.0 ** -e).astype(np.float32)
    qp = split3((q * 2.0 ** e[:, None]).astype(np.float32))      # 3 x [G][128]
    Kv, Vv = VAL[Kc], VAL[Vc]
    m_run = np.full(G, -np.inf)
    l_acc = np.zeros((TILE, G))                                 # per token lane
    o_acc = np.zeros((128, G))                                  # per d lane
    nt = -(-L // TILE)
    for i in range(nt):
        tok = np.arange(i * TILE, i * TILE + TILE)
        valid = tok < L
        Kt = np.zeros((TILE, 128))
        Vt = np.zeros((TILE, 128))
        Kt[valid] = Kv[tok[valid]]
        Vt[valid] = Vv[tok[valid]]
        S = [Kt @ VAL[qp[j]].T for j in range(3)]               # exact sums of exact products
        x = (S[0] + S[1] / 16 + S[2] / 256) * ch[None, :]
        x[~valid] = -np.inf
        mn = np.maximum(m_run, x.max(axis=0))
        alpha = np.exp2(m_run - mn)
        m_run = mn
        pw = np.exp2(x - mn[None, :])
        l_acc = l_acc * alpha[None, :] + pw
        pp = split3((pw * 256).astype(np.float32))
        O = [Vt.T @ VAL[pp[j]] for j in range(3)]                # [128 d][G]
        o_acc = o_acc * alpha[None, :] + (O[0] + O[1] / 16 + O[2] / 256)
    l = l_acc.sum(axis=0)
    return (o_acc * (v_scale / 256) / l[None, :]).T


def test_kernel_arithmetic_within_the_decode_tolerance():
    rng = np.random.default_rng(6)
    G, k_scale, v_scale = 4, 0.0125, 0.0125
    scale = 1 / np.sqrt(128)
    for L in (1, 37, 128, 300, 1024):
        q = torch.from_numpy(rng.standard_normal((G, 128)).astype(np.float32)).to(torch.bfloat16).float().numpy()
        Kc = e4m3_rn(np.clip(rng.standard_normal((L, 128)) / k_scale, -448, 448))
        Vc = e4m3_rn(np.clip(rng.standard_normal((L, 128)) / v_scale, -448, 448))
        got = _kernel_arith(q, Kc, Vc, k_scale, v_scale, scale)
        K = VAL[Kc] * k_scale
        V = VAL[Vc] * v_scale
        s = (q.astype(np.float64) @ K.T) * scale
        w = np.exp(s - s.max(axis=1, keepdims=True))
        ref = (w / w.sum(axis=1, keepdims=True)) @ V
        err = np.abs(got - ref)
        assert (err <= 0.1 * (2e-3 + 1e-2 * np.abs(ref))).all(), (L, err.max())
