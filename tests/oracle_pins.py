"""Pins that tie the CPU oracle to things other than itself.

Each ``pin_*`` function takes an ``oracle.Oracle`` and raises AssertionError when
the oracle disagrees with what the pages or the mathematics fix:

* a library routine: torch's ``scaled_dot_product_attention`` (fp64, dense,
  unpaged, with its own grouped-query head mapping) on the logical K/V that the
  generator drew before placing them in blocks; numpy/torch dtype conversions;
* invariants: physical block placement does not matter; weights sum to 1;
  a copy-on-write copy leaves every output unchanged;
* closed forms on 1-3 tokens: L=1 gives V exactly; two tokens give
  V0 + sigmoid(s1-s0) (V1-V0); equal scores give the mean of V; a dominant
  score gives its row; an empty context gives zeros;
* the cache layout as the generator placed the step's token and the copies.

The same functions run against deliberately broken builds of the oracle
(tests/test_oracle_mutants.py) to show that each plausible mistake is caught.
"""
from __future__ import annotations

import math

import numpy as np
import torch
import torch.nn.functional as F

from paged_kv_cache_464_b200 import inputs

SMALL_LENS = {
    "tiny": None,                                # the workload itself
    "llama2_7b": [64, 1, 77, 200, 2048 - 1000],
    "llama3_8b_gqa": [128, 250, 17, 5],
    "shared_prefix": [1024 + 16, 1024 + 100, 1024 + 512, 1024 + 33, 1030, 1024 + 1, 1200, 1300],
    "long_context": [700, 1536],
}


def small_case(name, **kw):
    lens = SMALL_LENS[name]
    return inputs.make_case(name, lens=lens, keep_logical=True, **kw)


def sdpa_reference(case) -> np.ndarray:
    """Dense attention with torch's library routine, in fp64, per sequence."""
    c = case.cfg
    out = np.zeros((c.num_seqs, c.num_heads, c.head_dim))
    q = case.q.to(torch.float64)
    for b in range(c.num_seqs):
        K = torch.from_numpy(case.k_logical[b]).permute(1, 0, 2)[None]   # [1, Hkv, L, D]
        V = torch.from_numpy(case.v_logical[b]).permute(1, 0, 2)[None]
        if K.shape[2] == 0:
            continue
        o = F.scaled_dot_product_attention(q[b][None, :, None, :], K, V, scale=float(np.float32(case.scale)),
                                           enable_gqa=True)
        out[b] = o[0, :, 0, :].numpy()
    return out


def _bytes(t: torch.Tensor) -> torch.Tensor:
    return t.contiguous().view(torch.uint8)


# ---------------------------------------------------------------------------
def pin_widening(o):
    bits = torch.arange(0, 65536, dtype=torch.int32).to(torch.int16)
    h = bits.view(torch.float16)
    got = o.widen(h)
    ref = h.numpy().astype(np.float64)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan), "fp16 NaN positions"
    assert np.array_equal(got[~nan], ref[~nan]), "fp16 widening"
    bf = bits.view(torch.bfloat16)
    got = o.widen(bf)
    ref = bf.to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan), "bf16 NaN positions"
    assert np.array_equal(got[~nan], ref[~nan]), "bf16 widening"
    f = torch.from_numpy(np.random.default_rng(1).standard_normal(4096).astype(np.float32))
    assert np.array_equal(o.widen(f), f.numpy().astype(np.float64)), "fp32 widening"


def pin_dense_equivalence(o, names=None, tol=1e-12):
    for name in names or inputs.BASE_WORKLOADS:
        case = small_case(name)
        got = o.decode_case(case)
        ref = sdpa_reference(case)
        err = np.abs(got - ref).max()
        assert err <= tol * max(1.0, np.abs(ref).max()), f"{name}: paged oracle vs dense SDPA max err {err}"


def pin_gqa_mapping(o):
    """Grouped heads read KV head h // G; a case where that differs from h % Hkv."""
    case = inputs.make_case(inputs.DecodeConfig("gqa", 9, 3, 8, 2, 128, "bf16"), lens=[40, 3, 70],
                            keep_logical=True)
    got = o.decode_case(case)
    ref = sdpa_reference(case)
    assert np.abs(got - ref).max() <= 1e-12, "GQA head mapping vs SDPA enable_gqa"
    # MHA on K/V heads repeated per group is the same computation
    G = case.cfg.group
    k_rep = case.k_cache_post.repeat_interleave(G, dim=2).contiguous()
    v_rep = case.v_cache_post.repeat_interleave(G, dim=2).contiguous()
    mha = o.paged_decode(case.q, k_rep, v_rep, case.block_tables, case.context_lens, case.scale)
    assert np.array_equal(got, mha), "GQA vs MHA on repeated heads"


def pin_block_permutation(o, names=("tiny", "llama3_8b_gqa", "shared_prefix")):
    for name in names:
        case = small_case(name)
        a = o.decode_case(case)
        for s in (7, 8):
            pc = inputs.permute_blocks(case, seed=s)
            b = o.decode_case(pc)
            assert np.array_equal(a, b), f"{name}: outputs depend on physical block ids"


def pin_length_one(o):
    for name in ("tiny", "llama2_7b", "llama3_8b_gqa"):
        case = inputs.make_case(name, lens=[1, 1, 2, 1], keep_logical=True)
        out = o.decode_case(case)
        G = case.cfg.group
        for b in range(case.cfg.num_seqs):
            if int(case.context_lens[b]) != 1:
                continue
            for h in range(case.cfg.num_heads):
                v = case.v_logical[b][0, h // G]
                assert np.array_equal(out[b, h], v), f"{name}: L=1 must return V exactly"


def pin_weights(o):
    for name in ("tiny", "llama3_8b_gqa", "long_context"):
        case = small_case(name)
        _, w = o.decode_case(case, return_weights=True)
        L = case.context_lens.numpy()
        for b in range(case.cfg.num_seqs):
            ws = w[b, :, :L[b]]
            assert np.all(ws >= 0.0)
            assert np.abs(ws.sum(axis=1) - 1.0).max() <= 1e-14, f"{name}: weights must sum to 1"
            assert np.all(w[b, :, L[b]:] == 0.0)


def _manual_case(qv, Ks, Vs, scale, dtype=torch.float32):
    """One sequence, one head, D = len(qv); tokens placed in blocks 3, 1 (bs=16) reversed."""
    D = len(qv)
    L = len(Ks)
    bs = 16
    NB = 4
    k = torch.full((NB, bs, 1, D), float("nan"), dtype=dtype)
    v = torch.full((NB, bs, 1, D), float("nan"), dtype=dtype)
    table = [3, 1]
    for t in range(L):
        k[table[t // bs], t % bs, 0] = torch.tensor(Ks[t], dtype=dtype)
        v[table[t // bs], t % bs, 0] = torch.tensor(Vs[t], dtype=dtype)
    q = torch.tensor([[qv]], dtype=dtype)
    bt = torch.tensor([table], dtype=torch.int32)
    cl = torch.tensor([L], dtype=torch.int32)
    return q, k, v, bt, cl


def pin_closed_forms(o):
    # two tokens: out = V0 + sigmoid(s1 - s0) (V1 - V0)
    qv = [0.5, -1.0]
    Ks = [[1.0, 0.25], [-0.75, 2.0]]
    Vs = [[1.0, -2.0], [0.5, 3.0]]
    scale = 0.5
    q, k, v, bt, cl = _manual_case(qv, Ks, Vs, scale)
    out = o.paged_decode(q, k, v, bt, cl, scale)[0, 0]
    s0 = scale * (qv[0] * Ks[0][0] + qv[1] * Ks[0][1])
    s1 = scale * (qv[0] * Ks[1][0] + qv[1] * Ks[1][1])
    sig = 1.0 / (1.0 + math.exp(-(s1 - s0)))
    ref = np.array(Vs[0]) + sig * (np.array(Vs[1]) - np.array(Vs[0]))
    assert np.abs(out - ref).max() <= 1e-15, f"two-token closed form {out} vs {ref}"

    # three tokens with identical keys: equal weights -> mean of V
    Ks = [[0.25, -0.5]] * 3
    Vs = [[1.0, 2.0], [4.0, -8.0], [-2.0, 0.5]]
    q, k, v, bt, cl = _manual_case([3.0, 1.0], Ks, Vs, 0.125)
    out = o.paged_decode(q, k, v, bt, cl, 0.125)[0, 0]
    assert np.abs(out - np.mean(Vs, axis=0)).max() <= 1e-15, "identical keys -> mean of V"

    # q = 0 -> mean of V whatever the keys
    Ks = [[1.0, 2.0], [-3.0, 0.5], [7.0, -1.0]]
    q, k, v, bt, cl = _manual_case([0.0, 0.0], Ks, Vs, 0.125)
    out = o.paged_decode(q, k, v, bt, cl, 0.125)[0, 0]
    assert np.abs(out - np.mean(Vs, axis=0)).max() <= 1e-15, "q = 0 -> mean of V"

    # scale = 0 -> mean of V
    q, k, v, bt, cl = _manual_case([1.0, -2.0], Ks, Vs, 0.0)
    out = o.paged_decode(q, k, v, bt, cl, 0.0)[0, 0]
    assert np.abs(out - np.mean(Vs, axis=0)).max() <= 1e-15, "scale = 0 -> mean of V"

    # a dominant score selects its row exactly (others underflow to weight 0)
    Ks = [[1.0, 0.0], [1000.0, 0.0], [-1000.0, 0.0]]
    q, k, v, bt, cl = _manual_case([1.0, 0.0], Ks, Vs, 1.0)
    out = o.paged_decode(q, k, v, bt, cl, 1.0)[0, 0]
    assert np.array_equal(out, np.array(Vs[1])), "dominant score -> its V row"

    # 20 tokens spanning two blocks; closed-form softmax with numpy for a check on the gather order
    rng = np.random.default_rng(5)
    Ks = [[float(x) for x in rng.integers(-4, 5, 2) / 4] for _ in range(20)]
    Vs = [[float(x) for x in rng.integers(-8, 9, 2) / 8] for _ in range(20)]
    q, k, v, bt, cl = _manual_case([0.5, -0.25], Ks, Vs, 0.5)
    out = o.paged_decode(q, k, v, bt, cl, 0.5)[0, 0]
    s = 0.5 * (np.array(Ks) @ np.array([0.5, -0.25]))
    w = np.exp(s - s.max())
    w /= w.sum()
    ref = w @ np.array(Vs)
    assert np.abs(out - ref).max() <= 1e-14, "two-block brute force"

    # empty context -> zeros
    q, k, v, bt, cl = _manual_case([1.0, 1.0], [[1.0, 1.0]], [[2.0, 2.0]], 1.0)
    cl[0] = 0
    out = o.paged_decode(q, k, v, bt, cl, 1.0)
    assert np.array_equal(out, np.zeros_like(out)), "empty context -> zeros"


def pin_slot_rule(o):
    for name in inputs.BASE_WORKLOADS:
        case = small_case(name)
        L = case.context_lens.numpy()
        for b in range(case.cfg.num_seqs):
            s = o.slot_for_position(case.block_tables[b], int(L[b]) - 1, case.cfg.block_size)
            assert s == int(case.slot_mapping[b]), f"{name}: slot of the new token"


def pin_cache_writes(o):
    for name in inputs.BASE_WORKLOADS:
        case = small_case(name)
        k = case.k_cache.clone()
        v = case.v_cache.clone()
        assert o.copy_blocks(k, v, case.block_mapping) == 0
        assert o.reshape_and_cache(k, v, case.key, case.value, case.slot_mapping) == 0
        assert torch.equal(_bytes(k), _bytes(case.k_cache_post)), f"{name}: K cache after step"
        assert torch.equal(_bytes(v), _bytes(case.v_cache_post)), f"{name}: V cache after step"
    # negative slots write nothing; an out-of-range slot is reported and skipped
    case = small_case("tiny")
    k = case.k_cache.clone()
    v = case.v_cache.clone()
    sm = case.slot_mapping.clone()
    sm[0] = -1
    sm[1] = case.num_blocks * case.cfg.block_size
    rc = o.reshape_and_cache(k, v, case.key, case.value, sm)
    assert rc == 3, "out-of-range slot must be reported"
    kk = case.k_cache.clone()
    vv = case.v_cache.clone()
    o.reshape_and_cache(kk, vv, case.key[2:], case.value[2:], case.slot_mapping[2:])
    assert torch.equal(_bytes(k), _bytes(kk)) and torch.equal(_bytes(v), _bytes(vv))


def pin_copy_blocks(o):
    g = torch.Generator().manual_seed(3)
    NB, bs, Hkv, D = 12, 16, 2, 64
    k0 = torch.randn(NB, bs, Hkv, D, generator=g)
    v0 = torch.randn(NB, bs, Hkv, D, generator=g)

    def run(pairs):
        k, v = k0.clone(), v0.clone()
        rc = o.copy_blocks(k, v, torch.tensor(pairs, dtype=torch.int64).reshape(-1, 2))
        return rc, k, v

    rc, k, v = run([[1, 5], [1, 6], [2, 7]])
    assert rc == 0
    exp_k, exp_v = k0.clone(), v0.clone()
    for s, d in [[1, 5], [1, 6], [2, 7]]:
        exp_k[d] = k0[s]
        exp_v[d] = v0[s]
    assert torch.equal(k, exp_k) and torch.equal(v, exp_v), "block copies"
    # duplicate destination: both pairs skipped; others done
    rc, k, v = run([[1, 5], [2, 5], [3, 8]])
    exp_k, exp_v = k0.clone(), v0.clone()
    exp_k[8], exp_v[8] = k0[3], v0[3]
    assert rc == 4 and torch.equal(k, exp_k) and torch.equal(v, exp_v), "duplicate destination"
    # a destination that another pair reads (a chain) and a self copy: skipped
    rc, k, v = run([[1, 5], [5, 9], [4, 4]])
    exp_k, exp_v = k0.clone(), v0.clone()
    exp_k[9], exp_v[9] = k0[5], v0[5]
    assert rc == 4 and torch.equal(k, exp_k) and torch.equal(v, exp_v), "chain / self copy"
    # out of range
    rc, k, v = run([[1, NB], [-1, 3]])
    assert rc == 2 and torch.equal(k, k0) and torch.equal(v, v0), "out-of-range ids"
    rc, k, v = run([])
    assert rc == 0 and torch.equal(k, k0)


def pin_copy_on_write_invariant(o):
    """Sequences that copied the shared block read the same values: outputs equal
    the outputs through the shared tables, bit for bit."""
    case = small_case("shared_prefix")
    out, k, v = o.step(case)
    ref = o.paged_decode(case.q, k, v, case.shared_block_tables, case.context_lens, case.scale)
    assert np.array_equal(out, ref), "copy-on-write changed an output"
    assert case.block_mapping.shape[0] == (case.cfg.num_seqs + 3) // 4


def pin_errors(o):
    case = small_case("tiny")
    bt = case.block_tables.clone()
    bt[1, 0] = case.num_blocks
    try:
        o.paged_decode(case.q, case.k_cache_post, case.v_cache_post, bt, case.context_lens, case.scale)
    except RuntimeError as e:
        assert getattr(e, "code", None) == 2
    else:
        raise AssertionError("out-of-range block id not reported")


# ---------------------------------------------------------------------------- FP8 (E4M3) cache
def pin_e4m3_decode(o):
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    got = o.e4m3_decode(codes)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan), "E4M3 NaN codes"
    assert np.array_equal(got[~nan], ref[~nan]), "E4M3 values"


def pin_e4m3_quantize(o):
    g = torch.Generator().manual_seed(11)
    x = torch.cat([torch.randn(20000, generator=g) * 30,
                   torch.randn(5000, generator=g) * 2 ** -8,                 # subnormal range
                   (torch.arange(-256, 256, dtype=torch.float32) + 0.5) * 2 ** -9,   # exact ties
                   torch.tensor([0.0, -0.0, 447.9, 448.0, 463.9, 464.0, -464.0, 479.9])])
    for scale in (1.0, 0.037, 2.5):
        got = o.e4m3_quantize(x, scale)
        q = x / torch.tensor(scale, dtype=torch.float32)
        inside = q.abs() <= 464          # torch's cast overflows to NaN beyond the 448/480 midpoint
        ref = q[inside].to(torch.float8_e4m3fn).view(torch.uint8)
        assert torch.equal(got[inside], ref), f"E4M3 rounding (scale {scale})"
    big = torch.tensor([464.01, 480.0, 1e6, -500.0, float("inf"), float("-inf")])
    assert o.e4m3_quantize(big, 1.0).tolist() == [0x7E, 0x7E, 0x7E, 0xFE, 0x7E, 0xFE], "saturation to +-448"
    assert o.e4m3_quantize(torch.tensor([float("nan")]), 1.0).tolist() == [0x7F]


def _fp8_case(name, lens, k_scale, v_scale, o):
    """A 16-bit case whose logical K/V are written into 1-byte caches by the oracle."""
    case = inputs.make_case(name, lens=lens, keep_logical=True)
    NB, bs, Hkv, D = case.k_cache.shape
    kc = torch.zeros((NB, bs, Hkv, D), dtype=torch.uint8)
    vc = torch.zeros_like(kc)
    rows_k, rows_v, slots = [], [], []
    bt = case.block_tables
    for b in range(case.cfg.num_seqs):
        L = int(case.context_lens[b])
        pos = torch.arange(L)
        slots.append(bt[b, pos // bs].to(torch.int64) * bs + pos % bs)
        rows_k.append(torch.from_numpy(case.k_logical[b]).to(case.k_cache.dtype))
        rows_v.append(torch.from_numpy(case.v_logical[b]).to(case.k_cache.dtype))
    sm, K, V = torch.cat(slots), torch.cat(rows_k), torch.cat(rows_v)
    assert o.reshape_and_cache_fp8(kc, vc, K, V, sm, k_scale, v_scale) == 0
    return case, kc, vc, K, V, sm


def pin_fp8_cache_layout(o):
    case, kc, vc, K, V, sm = _fp8_case("llama3_8b_gqa", [40, 17, 3], 0.02, 0.03, o)
    NB, bs, Hkv, D = kc.shape
    flat_k, flat_v = kc.view(NB * bs, Hkv, D), vc.view(NB * bs, Hkv, D)
    assert torch.equal(flat_k[sm], o.e4m3_quantize(K, 0.02)), "K rows at their slots"
    assert torch.equal(flat_v[sm], o.e4m3_quantize(V, 0.03)), "V rows at their slots"
    untouched = torch.ones(NB * bs, dtype=torch.bool)
    untouched[sm] = False
    assert int(flat_k[untouched].abs().sum()) == 0 and int(flat_v[untouched].abs().sum()) == 0


def pin_fp8_decode_vs_sdpa(o):
    for name, lens, ks, vs in (("llama3_8b_gqa", [128, 250, 17, 5], 0.011, 0.013),
                               ("llama2_7b", [64, 1, 77], 0.02, 0.05)):
        case, kc, vc, K, V, sm = _fp8_case(name, lens, ks, vs, o)
        got = o.paged_decode_fp8(case.q, kc, vc, ks, vs, case.block_tables, case.context_lens, case.scale)
        # dense reference on the dequantised logical rows
        dk = o.e4m3_decode(o.e4m3_quantize(K, ks)) * float(np.float32(ks))
        dv = o.e4m3_decode(o.e4m3_quantize(V, vs)) * float(np.float32(vs))
        c = case.cfg
        ref = np.zeros_like(got)
        start = 0
        for b in range(c.num_seqs):
            L = int(case.context_lens[b])
            Kb = torch.from_numpy(dk[start:start + L]).permute(1, 0, 2)[None]
            Vb = torch.from_numpy(dv[start:start + L]).permute(1, 0, 2)[None]
            start += L
            qb = case.q[b].to(torch.float64)[None, :, None, :]
            ref[b] = F.scaled_dot_product_attention(qb, Kb, Vb, scale=float(np.float32(case.scale)),
                                                    enable_gqa=True)[0, :, 0, :].numpy()
        assert np.abs(got - ref).max() <= 1e-12 * max(1.0, np.abs(ref).max()), f"{name}: fp8 decode vs SDPA"


# ---------------------------------------------------------------------------- prefill
def _prefill_sdpa(case):
    c = case.cfg
    out = np.zeros((case.num_tokens, c.num_heads, c.head_dim))
    for b in range(c.num_seqs):
        q0, q1 = int(case.query_start_loc[b]), int(case.query_start_loc[b + 1])
        n, L = q1 - q0, int(case.context_lens[b])
        if n == 0:
            continue
        K = torch.from_numpy(case.k_logical[b]).permute(1, 0, 2)[None]
        V = torch.from_numpy(case.v_logical[b]).permute(1, 0, 2)[None]
        qb = case.q[q0:q1].to(torch.float64).permute(1, 0, 2)[None]         # [1, Hq, n, D]
        mask = torch.arange(L)[None, :] <= (L - n + torch.arange(n))[:, None]  # query i sees tokens <= L-n+i
        o = F.scaled_dot_product_attention(qb, K, V, attn_mask=mask, scale=float(np.float32(case.scale)),
                                           enable_gqa=True)
        out[q0:q1] = o[0].permute(1, 0, 2).numpy()
    return out


def pin_prefill_vs_sdpa(o):
    cfg = inputs.PREFILL_CONFIGS["llama3_8b_prefill"]
    for chunks, prefixes in (([5, 16, 17, 1, 40], [0, 3, 31, 100, 0]), ([64, 33], [200, 1])):
        case = inputs.make_prefill_case(cfg, chunk_lens=chunks, prefix_lens=prefixes, keep_logical=True)
        got = o.paged_prefill(case.q, case.k_cache, case.v_cache, case.block_tables, case.context_lens,
                              case.query_start_loc, case.scale)
        ref = _prefill_sdpa(case)
        assert np.abs(got - ref).max() <= 1e-12 * max(1.0, np.abs(ref).max()), "prefill vs SDPA with causal mask"


def pin_prefill_causality(o):
    cfg = inputs.PREFILL_CONFIGS["llama3_8b_prefill"]
    case = inputs.make_prefill_case(cfg, chunk_lens=[20], prefix_lens=[30])
    a = o.paged_prefill(case.q, case.k_cache, case.v_cache, case.block_tables, case.context_lens,
                        case.query_start_loc, case.scale)
    k, v = case.k_cache.clone(), case.v_cache.clone()
    last = int(case.context_lens[0]) - 1
    blk, off = int(case.block_tables[0, last // 16]), last % 16
    k[blk, off] = -k[blk, off]
    v[blk, off] = v[blk, off] + 1
    b = o.paged_prefill(case.q, k, v, case.block_tables, case.context_lens, case.query_start_loc, case.scale)
    assert np.array_equal(a[:-1], b[:-1]), "earlier queries must not see a later token"
    assert not np.array_equal(a[-1], b[-1]), "the last query sees the last token"


def pin_prefill_one_query_is_decode(o):
    cfg = inputs.PREFILL_CONFIGS["llama3_8b_prefill"]
    case = inputs.make_prefill_case(cfg, chunk_lens=[1, 1, 1], prefix_lens=[0, 16, 700])
    a = o.paged_prefill(case.q, case.k_cache, case.v_cache, case.block_tables, case.context_lens,
                        case.query_start_loc, case.scale)
    b = o.paged_decode(case.q, case.k_cache, case.v_cache, case.block_tables, case.context_lens, case.scale)
    assert np.array_equal(a, b)


ALL_PINS = [pin_widening, pin_dense_equivalence, pin_gqa_mapping, pin_block_permutation,
            pin_length_one, pin_weights, pin_closed_forms, pin_slot_rule, pin_cache_writes,
            pin_copy_blocks, pin_copy_on_write_invariant, pin_errors, pin_e4m3_decode, pin_e4m3_quantize,
            pin_fp8_cache_layout, pin_fp8_decode_vs_sdpa, pin_prefill_vs_sdpa, pin_prefill_causality,
            pin_prefill_one_query_is_decode]
