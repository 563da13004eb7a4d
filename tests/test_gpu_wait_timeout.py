"""The bounded-wait error path, made to run on purpose (no fault, no hang).

Every wait of the decode and prefill kernels on a tile copy gives up after a
time limit, records PA_DEV_WAIT_TIMEOUT with the CTA's linear index, lets the
copies it still has in flight land, and returns without writing its output.
pa_test_stall_next_launch arms the next launch so that one chosen CTA leaves
one copy unissued (no copy and no barrier arrival: nothing is in flight for
it) and waits at most 1 ms; its wait on that tile therefore runs out.

Each test checks: the error word holds the timeout and that CTA's index; the
stalled CTA's output rows keep the sentinel they were filled with; every other
row is within the decode tolerance of the fp64 oracle; and the next ordinary
launch on the same stream is correct and records no error (the context is
still usable).
"""
import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_464_b200 import inputs

pytestmark = [pytest.mark.gpu, pytest.mark.expects_device_error]

PA_DEV_WAIT_TIMEOUT = 5
SENTINEL = 12288.0   # 3 * 2^12: exactly representable in bf16 and fp16


@pytest.fixture(scope="module")
def pa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from paged_kv_cache_464_b200 import capi
    capi.test_stall_next_launch("decode", -1)
    capi.test_stall_next_launch("prefill", -1)
    capi.get_device_error(clear=True)
    yield capi
    capi.test_stall_next_launch("decode", -1)
    capi.test_stall_next_launch("prefill", -1)
    capi.get_device_error(clear=True)


@pytest.fixture(scope="module")
def orc():
    return oracle.get()


def _close(g: np.ndarray, ref: np.ndarray, what: str):
    assert np.isfinite(g).all(), f"{what}: non-finite output"
    err = np.abs(g - ref)
    bad = err > 2e-3 + 1e-2 * np.abs(ref)
    assert not bad.any(), f"{what}: {bad.sum()} elements out of tolerance, max abs {err.max():.3e}"


def test_decode_wait_runs_out_in_one_cta(pa, orc):
    # four sequences, none longer than one partition (1024 tokens for the
    # grouped-query tensor-core path), so every CTA writes its rows itself
    case = inputs.make_case("llama3_8b_gqa", lens=[128, 700, 1000, 33])
    cfg = case.cfg
    G, Hkv = cfg.group, cfg.num_kv_heads
    P = pa.decode_partition_size(cfg.num_seqs, cfg.num_heads, Hkv, cfg.head_dim, case.max_context_len, 0)
    assert P >= case.max_context_len
    ref = orc.decode_case(case)
    dev = "cuda"
    q, k, v = case.q.to(dev), case.k_cache_post.to(dev), case.v_cache_post.to(dev)
    bt, cl = case.block_tables.to(dev), case.context_lens.to(dev)
    b, g = 1, 3                      # 700 tokens: 44 blocks, so warp 0 owns 11 of them
    cta = (b * Hkv + g) * 1 + 0      # grid = (sequence, KV head, partition); one partition
    out = torch.full_like(q, SENTINEL)
    pa.get_device_error(clear=True)
    pa.test_stall_next_launch("decode", cta)
    pa.decode(q, k, v, bt, cl, case.scale, out, max_context_len=case.max_context_len)
    code, detail = pa.get_device_error(clear=True)
    assert (code, detail) == (PA_DEV_WAIT_TIMEOUT, cta)
    got = out.to(torch.float64).cpu().numpy()
    heads = slice(g * G, (g + 1) * G)
    assert (got[b, heads] == SENTINEL).all(), "the stalled CTA wrote its rows"
    mask = np.ones(got.shape[:2], dtype=bool)
    mask[b, heads] = False
    _close(got[mask], ref[mask], "other rows of the stalled launch")

    # the next ordinary launch on the same stream: correct, no error
    out2 = pa.decode(q, k, v, bt, cl, case.scale, max_context_len=case.max_context_len)
    code, detail = pa.get_device_error(clear=True)
    assert code == 0, (code, detail)
    _close(out2.to(torch.float64).cpu().numpy(), ref, "next launch")


def test_decode_wait_runs_out_in_a_split_sequence(pa, orc):
    # a partition CTA of a split sequence: its partial is never written, so only
    # the other (sequence, KV head) rows are checked; the error names the CTA
    case = inputs.make_case("long_context", lens=[2048, 700, 1500])
    cfg = case.cfg
    G, Hkv = cfg.group, cfg.num_kv_heads
    P = 512
    np_max = -(-case.max_context_len // P)
    ref = orc.decode_case(case)
    dev = "cuda"
    q, k, v = case.q.to(dev), case.k_cache_post.to(dev), case.v_cache_post.to(dev)
    bt, cl = case.block_tables.to(dev), case.context_lens.to(dev)
    b, g, part = 0, 5, 2
    cta = (b * Hkv + g) * np_max + part
    out = torch.full_like(q, SENTINEL)
    pa.get_device_error(clear=True)
    pa.test_stall_next_launch("decode", cta)
    pa.decode(q, k, v, bt, cl, case.scale, out, max_context_len=case.max_context_len, partition_size=P)
    code, detail = pa.get_device_error(clear=True)
    assert (code, detail) == (PA_DEV_WAIT_TIMEOUT, cta)
    got = out.to(torch.float64).cpu().numpy()
    mask = np.ones(got.shape[:2], dtype=bool)
    mask[b, g * G:(g + 1) * G] = False
    _close(got[mask], ref[mask], "other rows of the stalled launch")
    out2 = pa.decode(q, k, v, bt, cl, case.scale, max_context_len=case.max_context_len, partition_size=P)
    code, detail = pa.get_device_error(clear=True)
    assert code == 0, (code, detail)
    _close(out2.to(torch.float64).cpu().numpy(), ref, "next launch")


def test_prefill_wait_runs_out_in_one_cta(pa, orc):
    cfg = inputs.DecodeConfig("stall_prefill", 77, 3, 8, 2, 128, "bf16")
    pc = inputs.make_prefill_case(cfg, chunk_lens=[70, 5, 129], prefix_lens=[40, 0, 300])
    G = cfg.group
    ref = orc.paged_prefill(pc.q, pc.k_cache, pc.v_cache, pc.block_tables, pc.context_lens, pc.query_start_loc,
                            pc.scale)
    dev = "cuda"
    args = [pc.q.to(dev), pc.k_cache.to(dev), pc.v_cache.to(dev), pc.block_tables.to(dev), pc.context_lens.to(dev),
            pc.query_start_loc.to(dev), pc.scale]
    # grid: x = query-tile pair, counted from the end (x = gx - 1 holds chunk
    # queries 0 .. 63), y = KV head, z = sequence; 64 chunk queries per CTA at G = 4
    qt = 2 * 128 // G
    gx, gy = -(-pc.max_query_len // qt), cfg.num_kv_heads
    b, g = 0, 1
    x = gx - 1
    cta = x + gx * (g + gy * b)
    out = torch.full_like(args[0], SENTINEL)
    pa.get_device_error(clear=True)
    pa.test_stall_next_launch("prefill", cta)
    pa.prefill(*args, out, max_query_len=pc.max_query_len)
    code, detail = pa.get_device_error(clear=True)
    assert (code, detail) == (PA_DEV_WAIT_TIMEOUT, cta)
    got = out.to(torch.float64).cpu().numpy()
    r0 = int(pc.query_start_loc[b])
    n = int(pc.query_start_loc[b + 1]) - r0
    rows = slice(r0, r0 + min(n, qt))
    heads = slice(g * G, (g + 1) * G)
    assert (got[rows, heads] == SENTINEL).all(), "the stalled CTA wrote its rows"
    mask = np.ones(got.shape[:2], dtype=bool)
    mask[rows, heads] = False
    _close(got[mask], ref[mask], "other rows of the stalled launch")
    out2 = pa.prefill(*args, max_query_len=pc.max_query_len)
    code, detail = pa.get_device_error(clear=True)
    assert code == 0, (code, detail)
    _close(out2.to(torch.float64).cpu().numpy(), ref, "next launch")


def _fp8_codes(orc, case, k_scale, v_scale):
    """1-byte caches holding every attended token of a 16-bit case (quantised by the oracle)."""
    NB, bs, Hkv, D = case.k_cache_post.shape
    sm = torch.cat([case.block_tables[b, torch.arange(int(L)) // bs].to(torch.int64) * bs + torch.arange(int(L)) % bs
                    for b, L in enumerate(case.context_lens.tolist())])
    K = case.k_cache_post.view(NB * bs, Hkv, D)[sm].contiguous()
    V = case.v_cache_post.view(NB * bs, Hkv, D)[sm].contiguous()
    kc = torch.zeros((NB, bs, Hkv, D), dtype=torch.uint8)
    vc = torch.zeros_like(kc)
    assert orc.reshape_and_cache_fp8(kc, vc, K, V, sm, k_scale, v_scale) == 0
    return kc, vc


def test_fp8_decode_wait_runs_out_in_one_cta(pa, orc):
    # the tensor-core E4M3 kernel: the stalled CTA's TMA warp leaves its first
    # tile unissued, so the issuer's wait on it runs out and every role stops
    case = inputs.make_case("llama3_8b_gqa", lens=[128, 700, 1000, 33])
    cfg = case.cfg
    G, Hkv = cfg.group, cfg.num_kv_heads
    ks, vs = 0.0125, 0.011
    kc, vc = _fp8_codes(orc, case, ks, vs)
    ref = orc.paged_decode_fp8(case.q, kc, vc, ks, vs, case.block_tables, case.context_lens, case.scale)
    dev = "cuda"
    args = [case.q.to(dev), kc.to(dev), vc.to(dev), ks, vs, case.block_tables.to(dev), case.context_lens.to(dev),
            case.scale]
    b, g = 2, 6
    cta = b * Hkv + g                # one partition a sequence (P = 1024)
    out = torch.full_like(args[0], SENTINEL)
    pa.get_device_error(clear=True)
    pa.test_stall_next_launch("decode", cta)
    pa.decode_fp8(*args, out, max_context_len=case.max_context_len)
    code, detail = pa.get_device_error(clear=True)
    assert (code, detail) == (PA_DEV_WAIT_TIMEOUT, cta)
    got = out.to(torch.float64).cpu().numpy()
    heads = slice(g * G, (g + 1) * G)
    assert (got[b, heads] == SENTINEL).all(), "the stalled CTA wrote its rows"
    mask = np.ones(got.shape[:2], dtype=bool)
    mask[b, heads] = False
    _close(got[mask], ref[mask], "other rows of the stalled launch")
    out2 = pa.decode_fp8(*args, max_context_len=case.max_context_len)
    code, detail = pa.get_device_error(clear=True)
    assert code == 0, (code, detail)
    _close(out2.to(torch.float64).cpu().numpy(), ref, "next launch")
