"""The paged-prefill kernel's operand layouts, emulated on the CPU.

csrc/pa_prefill.cuh stages Q with generic 16-byte stores that apply the
128-byte swizzle themselves, lands K and V tiles with TMA boxes (one 128-byte
half of 16 token rows per cache block, hardware swizzle), and hands the tensor
cores shared-memory descriptors (start address, leading / stride byte offsets)
for S = Q K^T (both operands K-major) and O += P V (V MN-major).  The 128-byte
swizzle exchanges the 16-byte chunks of each 128-byte row by the row's index
within its 1024-byte atom.  Tile elements here are unique 16-bit identifiers,
so every operand the descriptors describe must read back exactly the matrix
the product needs.  Also checked: where P's fp16 pairs land in tensor
memory for the products that read them, and the accuracy of P and V in fp16.
"""
import numpy as np

ROWS, KV, HALF_ROWS = 128, 64, 128 * 128       # query rows, KV tile tokens, bytes of one Q half
KV_HALF = KV * 128                              # bytes of one 64-element half of a KV tile


def swz(a):
    """Physical address of logical address a under the 128-byte swizzle (1024-byte atoms)."""
    return a ^ (((a >> 7) & 7) << 4)


def read16(sm, addr):
    addr = np.asarray(addr)
    return sm[addr].astype(np.uint32) | (sm[addr + 1].astype(np.uint32) << 8)


def read_kmajor(sm, start, sbo, rows):
    """A K-major operand of `rows` x 16 elements: 8-row groups sbo bytes apart, 128-byte rows."""
    r = np.arange(rows)[:, None]
    k = np.arange(16)[None, :]
    return read16(sm, swz(start + (r % 8) * 128 + (r // 8) * sbo + 2 * k))


def read_mnmajor(sm, start, lbo, sbo, nmn):
    """An MN-major operand of 16 (K) x nmn elements: 64-element MN groups lbo bytes apart,
    consecutive K in consecutive 128-byte rows, 8-row K groups sbo bytes apart."""
    k = np.arange(16)[:, None]
    mn = np.arange(nmn)[None, :]
    return read16(sm, swz(start + (mn % 64) * 2 + (mn // 64) * lbo + (k % 8) * 128 + (k // 8) * sbo))


def ids(rows, cols, base):
    return (base + np.arange(rows * cols, dtype=np.uint32).reshape(rows, cols)) & 0xFFFF


def put16(sm, addr, v):
    sm[addr], sm[addr + 1] = v & 0xFF, v >> 8


def test_q_staging_and_qk_descriptors():
    Q = ids(ROWS, 128, 1)
    sm = np.zeros(2 * HALF_ROWS, np.uint8)
    for row in range(ROWS):                         # the kernel's Q store: chunk c of a row, swizzled by hand
        for c in range(16):
            base = (c >> 3) * HALF_ROWS + row * 128 + (((c & 7) ^ (row & 7)) << 4)
            for e in range(8):
                put16(sm, base + 2 * e, Q[row, 8 * c + e])
    for kk in range(8):                             # a_qk + ((kk >> 2) * half + (kk & 3) * 32)
        start = (kk >> 2) * HALF_ROWS + (kk & 3) * 32
        assert np.array_equal(read_kmajor(sm, start, 1024, ROWS), Q[:, 16 * kk:16 * kk + 16])


def _tma_tile(X_blocks):
    """A KV tile from 4 cache blocks (16 tokens x 128 elements each) placed as the TMA
    boxes do: half h of block bi at h * KV_HALF + bi * 16 * 128, rows of 128 bytes, swizzled."""
    sm = np.zeros(2 * KV_HALF, np.uint8)
    for bi, X in enumerate(X_blocks):
        for h in range(2):
            dst = h * KV_HALF + bi * 16 * 128
            for t in range(16):
                for e in range(64):
                    put16(sm, swz(dst + t * 128 + 2 * e), X[t, 64 * h + e])
    return sm


def test_kv_tiles_and_product_descriptors():
    blocks_k = [ids(16, 128, 1000 * (i + 1)) for i in range(4)]
    blocks_v = [ids(16, 128, 7000 + 1000 * i) for i in range(4)]
    K, V = np.vstack(blocks_k), np.vstack(blocks_v)            # logical 64 x 128 tiles
    smk, smv = _tma_tile(blocks_k), _tma_tile(blocks_v)
    for kk in range(8):                                        # QK: B = K tile, K-major, N = 64
        start = (kk >> 2) * KV_HALF + (kk & 3) * 32
        assert np.array_equal(read_kmajor(smk, start, 1024, KV), K[:, 16 * kk:16 * kk + 16])
    for kk in range(KV // 16):                                 # PV: B = V tile, MN-major, N = 128 (head_dim)
        got = read_mnmajor(smv, kk * 16 * 128, KV_HALF, 1024, 128)
        assert np.array_equal(got, V[16 * kk:16 * kk + 16, :])


def test_p_columns_in_tensor_memory():
    """The softmax stores P(j) over S(j) as fp16 pairs (tokens 2k, 2k+1) at
    column k, the lower token in the low half.  The product for tokens
    16kk..16kk+15 reads columns 8kk .. 8kk + 7."""
    col_of = {}
    for k in range(32):
        for h in range(2):
            col_of[2 * k + h] = (k, h)
    for kk in range(KV // 16):
        cols = [kk * 8 + c for c in range(8)]
        tokens = [c * 2 + h for c in cols for h in range(2)]
        assert tokens == list(range(16 * kk, 16 * kk + 16))
        assert all(col_of[t][0] in cols for t in tokens)


def test_fp16_p_and_v_conversion():
    """P in fp16 (nearest): relative rounding <= 2^-11 over the lazy-rescale
    range (0, 2^8], and absolute <= 2^-25 where it is subnormal.  bf16 V
    times 2^-8 in fp16: exact for every bf16 value with 2^-6 <= |v| < 2^24,
    within 2^-17 absolute below that, and out of range (inf) from 2^24 up."""
    rng = np.random.default_rng(5)
    p = np.concatenate([rng.uniform(0, 1, 200000), rng.uniform(1, 256, 50000),
                        2.0 ** rng.uniform(-40, 0, 50000)]).astype(np.float32)
    h = p.astype(np.float16).astype(np.float64)
    err = np.abs(h - p.astype(np.float64))
    assert (err <= np.maximum(2.0 ** -11 * p, 2.0 ** -25)).all()
    # every bf16 bit pattern: exponent fields 1..254 (finite, normal), both signs
    bits = np.arange(1 << 16, dtype=np.uint32)
    v = (bits << 16).view(np.float32)
    v = v[np.isfinite(v)]
    with np.errstate(over="ignore"):
        scaled = (v * np.float32(2.0 ** -8)).astype(np.float16)
    back = scaled.astype(np.float64) * 256.0
    a = np.abs(v.astype(np.float64))
    exact = (a >= 2.0 ** -6) & (a < 2.0 ** 24)
    assert np.array_equal(back[exact], v.astype(np.float64)[exact])
    small = a < 2.0 ** -6
    assert (np.abs(back[small] - v.astype(np.float64)[small]) <= 2.0 ** -17).all()
    assert np.isinf(back[a >= 2.0 ** 24 + 2.0 ** 17]).all()


def test_emulation_catches_a_wrong_stride():
    """The V operand read with the K-major stride (lbo = 16) is wrong."""
    blocks_v = [ids(16, 128, 7000 + 1000 * i) for i in range(4)]
    V, smv = np.vstack(blocks_v), _tma_tile(blocks_v)
    assert not np.array_equal(read_mnmajor(smv, 0, 16, 1024, 128), V[0:16, :])


def _bank_degree(byte_addrs):
    """Wavefronts of one warp's 16-byte shared-memory accesses: the largest
    number of distinct 4-byte words any of the 32 banks must serve."""
    words = {(a // 4 + i) for a in byte_addrs for i in range(4)}
    per_bank = {}
    for wd in words:
        per_bank[wd % 32] = per_bank.get(wd % 32, 0) + 1
    return max(per_bank.values())


def stage_addr(r, ch):
    """Epilogue staging in the Q buffer: 16-byte chunk ch of output row r."""
    return r * 256 + ((ch ^ (r & 15)) << 4)


def test_epilogue_staging_and_copy_out():
    """O / l goes through the tile's 32 KiB Q buffer: thread r (the row) writes
    its 16 chunks at stage_addr(r, ch); the warpgroup then copies unit u (row
    u >> 4, chunk u & 15) from there to the output row of query r // G, head
    g*G + r % G.  Checked: the staging is a permutation of the buffer, every
    warp access takes the minimum 4 wavefronts, the copy reads back exactly
    what each row wrote, and a warp store covers at most 4 128-byte lines
    (the row-per-thread store it replaces covers 32)."""
    addrs = sorted(stage_addr(r, ch) for r in range(128) for ch in range(16))
    assert addrs == list(range(0, 32768, 16))
    for q in range(4):                      # warp q of the warpgroup writes rows 32q .. 32q + 31
        for ch in range(16):
            assert _bank_degree([stage_addr(32 * q + l, ch) for l in range(32)]) == 4
    for G in (1, 2, 4, 8):
        Hq, g, qs, q0 = 32, 1, 5, 0
        QT = 128 // G
        for nq in (QT, 1, QT - 1 if QT > 1 else 1):
            stage = {}
            for r in range(128):
                for ch in range(16):
                    stage[stage_addr(r, ch)] = (r, ch)
            units = nq * G * 16
            seen = set()
            for base in range(0, units, 32):    # one warp instruction: 32 consecutive units
                lanes = range(base, min(base + 32, units))
                assert _bank_degree([stage_addr(u >> 4, u & 15) for u in lanes]) <= 4
                lines = set()
                for u in lanes:
                    rr, ch = u >> 4, u & 15
                    assert stage[stage_addr(rr, ch)] == (rr, ch)
                    elem = ((qs + q0 + rr // G) * Hq + g * G + rr % G) * 128 + ch * 8
                    seen.add((rr, ch))
                    lines.add(elem * 2 // 128)
                assert len(lines) <= 4
            assert seen == {(r, ch) for r in range(nq * G) for ch in range(16)}
    # the store it replaces: each lane its own row, one 16-byte chunk per instruction
    old = {(((r // 4) * 32 + 4 + r % 4) * 128 * 2) // 128 for r in range(32)}
    assert len(old) == 32
