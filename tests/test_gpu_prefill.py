"""Paged chunked prefill on the GPU (tcgen05 kernel) against the CPU oracle.

Tolerance: that of the 16-bit decode, |gpu - ref| <= 2e-3 + 1e-2 |ref|, with
ref the oracle's fp64 result on the same rounded inputs.  Stale cache slots
(rows no context covers) are filled with NaN, so that reading one shows up.
"""
import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_464_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from paged_kv_cache_464_b200 import capi
    capi.get_device_error(clear=True)
    return capi


@pytest.fixture(scope="module")
def orc():
    return oracle.get()


def _close(out, ref, what=""):
    g = out.to(torch.float64).cpu().numpy()
    assert np.isfinite(g).all(), f"{what}: non-finite output"
    err = np.abs(g - ref)
    bad = err > 2e-3 + 1e-2 * np.abs(ref)
    assert not bad.any(), f"{what}: {bad.sum()} of {bad.size} out of tolerance, max abs {err.max():.3e}"


def _poison(case):
    """NaN in every cache row outside all contexts."""
    NB, bs, Hkv, D = case.k_cache.shape
    used = torch.zeros(NB * bs, dtype=torch.bool)
    for b in range(case.cfg.num_seqs):
        L = int(case.context_lens[b])
        pos = torch.arange(L)
        used[case.block_tables[b, pos // bs].long() * bs + pos % bs] = True
    for c in (case.k_cache, case.v_cache):
        c.view(NB * bs, Hkv, D)[~used] = float("nan")
    return case


def _gpu(pa, case, **kw):
    out = pa.prefill(case.q.cuda(), case.k_cache.cuda(), case.v_cache.cuda(), case.block_tables.cuda(),
                     case.context_lens.cuda(), case.query_start_loc.cuda(), case.scale,
                     max_query_len=kw.pop("max_query_len", case.max_query_len), **kw)
    torch.cuda.synchronize()
    return out


def _ref(orc, case):
    return orc.paged_prefill(case.q, case.k_cache, case.v_cache, case.block_tables, case.context_lens,
                             case.query_start_loc, case.scale)


def _no_device_error(pa):
    code, detail = pa.get_device_error(clear=True)
    assert code == 0, (code, detail)


CHUNKS = [37, 5, 70, 1, 128, 200]
PREFIX = [50, 0, 13, 600, 0, 333]


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
@pytest.mark.parametrize("group", [1, 2, 4, 8])
def test_prefill_small(pa, orc, dtype, group):
    cfg = inputs.DecodeConfig(f"prefill_g{group}", 21 + group, len(CHUNKS), 2 * group, 2, 128, dtype)
    case = _poison(inputs.make_prefill_case(cfg, chunk_lens=CHUNKS, prefix_lens=PREFIX))
    _close(_gpu(pa, case), _ref(orc, case), f"G={group} {dtype}")
    _no_device_error(pa)


def test_prefill_chunk_is_whole_prompt_and_ragged_tiles(pa, orc):
    # no prefix: the chunk is the whole prompt; lengths around the 64-token KV tile
    # and the 32-query tile of G=4 (ragged tails on both axes)
    chunks = [1, 15, 16, 17, 31, 32, 33, 63, 64, 65, 127, 129]
    cfg = inputs.DecodeConfig("prefill_ragged", 31, len(chunks), 8, 2, 128, "bf16")
    case = _poison(inputs.make_prefill_case(cfg, chunk_lens=chunks, prefix_lens=[0] * len(chunks)))
    _close(_gpu(pa, case), _ref(orc, case), "ragged")
    _no_device_error(pa)


def test_prefill_one_token_chunks_equal_decode(pa, orc):
    # a chunk of one token is a decode step: the two kernels agree with each other
    # (and with the oracle) on the same cache
    lens = [1, 16, 77, 300, 1024, 2049]
    cfg = inputs.DecodeConfig("prefill_decode", 41, len(lens), 32, 8, 128, "bf16")
    case = inputs.make_prefill_case(cfg, chunk_lens=[1] * len(lens), prefix_lens=[n - 1 for n in lens])
    out = _gpu(pa, case)
    dec = pa.decode(case.q.cuda(), case.k_cache.cuda(), case.v_cache.cuda(), case.block_tables.cuda(),
                    case.context_lens.cuda(), case.scale, max_context_len=max(lens))
    torch.cuda.synchronize()
    ref = _ref(orc, case)
    _close(out, ref, "prefill n=1")
    _close(dec, ref, "decode")
    _no_device_error(pa)


def test_prefill_block_permutation_invariance(pa, orc):
    cfg = inputs.DecodeConfig("prefill_perm", 51, 4, 16, 4, 128, "bf16")
    case = inputs.make_prefill_case(cfg, chunk_lens=[100, 3, 64, 250], prefix_lens=[20, 400, 0, 90])
    a = _gpu(pa, case)
    # move every physical block (and its table entries) through a seeded permutation
    NB = case.k_cache.shape[0]
    sigma = torch.randperm(NB, generator=torch.Generator().manual_seed(3))
    k2 = torch.empty_like(case.k_cache)
    v2 = torch.empty_like(case.v_cache)
    k2[sigma] = case.k_cache
    v2[sigma] = case.v_cache
    bt2 = torch.where(case.block_tables >= 0, sigma[case.block_tables.clamp(min=0).long()].to(torch.int32),
                      case.block_tables)
    import dataclasses
    case2 = dataclasses.replace(case, k_cache=k2, v_cache=v2, block_tables=bt2)
    b = _gpu(pa, case2)
    assert torch.equal(a.cpu(), b.cpu()), "output depends on where the blocks sit"
    _close(a, _ref(orc, case), "perm")


def test_prefill_garbage_table_tail(pa, orc):
    # table entries past each context's last block are never read
    cfg = inputs.DecodeConfig("prefill_tail", 61, 3, 32, 8, 128, "bf16")
    case = inputs.make_prefill_case(cfg, chunk_lens=[40, 7, 90], prefix_lens=[10, 33, 0])
    ref = _ref(orc, case)
    bt = case.block_tables.clone()
    for b in range(3):
        L = int(case.context_lens[b])
        bt[b, (L + 15) // 16:] = -7 if b % 2 else 10 ** 6
    import dataclasses
    out = _gpu(pa, dataclasses.replace(case, block_tables=bt))
    _close(out, ref, "garbage tail")
    _no_device_error(pa)


def test_prefill_full_size_all_sequences(pa, orc):
    """The Llama-3-8B-shaped chunked-prefill workload in the launch the bench
    times; the oracle checks every query row of all 16 sequences."""
    case = _poison(inputs.make_prefill_case("llama3_8b_prefill"))
    out = _gpu(pa, case).cpu()
    _no_device_error(pa)
    qsl = case.query_start_loc
    for b in range(case.cfg.num_seqs):
        sub = inputs.prefill_subcase(case, [b])
        ref = _ref(orc, sub)
        _close(out[int(qsl[b]):int(qsl[b + 1])], ref, f"full size, sequence {b}")


def test_prefill_bad_context_len_and_block_id(pa):
    cfg = inputs.DecodeConfig("prefill_err", 71, 2, 8, 2, 128, "bf16")
    case = inputs.make_prefill_case(cfg, chunk_lens=[20, 20], prefix_lens=[5, 5])
    pa.get_device_error(clear=True)
    # chunk longer than the context: sequence 1 is skipped and reported
    cl = case.context_lens.clone()
    cl[1] = 10
    pa.prefill(case.q.cuda(), case.k_cache.cuda(), case.v_cache.cuda(), case.block_tables.cuda(), cl.cuda(),
               case.query_start_loc.cuda(), case.scale, max_query_len=20)
    code, detail = pa.get_device_error(clear=True)
    assert (code, detail) == (4, 1)
    # a block id outside the pool: reported, read as zeros, no fault
    bt = case.block_tables.clone()
    bt[0, 0] = 10 ** 6
    pa.prefill(case.q.cuda(), case.k_cache.cuda(), case.v_cache.cuda(), bt.cuda(), case.context_lens.cuda(),
               case.query_start_loc.cuda(), case.scale, max_query_len=20)
    code, detail = pa.get_device_error(clear=True)
    assert (code, detail) == (1, 10 ** 6)


def test_prefill_v_out_of_range_reported(pa, orc):
    # bf16 caches: V enters P V as fp16 times 2^-8, which holds every |v| < 2^24.
    # One attended V element of sequence 1 at 2^25 is reported (detail = the
    # sequence); sequence 0's rows stay within tolerance of the oracle.
    cfg = inputs.DecodeConfig("prefill_range", 73, 2, 8, 2, 128, "bf16")
    case = inputs.make_prefill_case(cfg, chunk_lens=[20, 20], prefix_lens=[5, 30])
    vc = case.v_cache.clone()
    blk = int(case.block_tables[1, 0])
    vc[blk, 3, 1, 7] = 2.0 ** 25
    ref = orc.paged_prefill(case.q, case.k_cache, vc, case.block_tables, case.context_lens, case.query_start_loc,
                            case.scale)
    pa.get_device_error(clear=True)
    out = pa.prefill(case.q.cuda(), case.k_cache.cuda(), vc.cuda(), case.block_tables.cuda(),
                     case.context_lens.cuda(), case.query_start_loc.cuda(), case.scale, max_query_len=20)
    code, detail = pa.get_device_error(clear=True)
    assert (code, detail) == (6, 1)
    rows0 = slice(0, int(case.query_start_loc[1]))
    _close(out[rows0], ref[rows0], "sequence 0")


def test_prefill_empty_chunks(pa, orc):
    # sequences with no query rows in this step are skipped; others unaffected
    cfg = inputs.DecodeConfig("prefill_empty", 81, 4, 8, 2, 128, "f16")
    case = inputs.make_prefill_case(cfg, chunk_lens=[0, 33, 0, 2], prefix_lens=[40, 1, 0, 70])
    _close(_gpu(pa, case), _ref(orc, case), "empty chunks")
    _no_device_error(pa)
