"""FP8 (E4M3) KV cache on the GPU against the CPU oracle.

The quantising slot write must reproduce the oracle's codes byte for byte; the
decode over 1-byte caches must match the oracle's fp64 decode of the same codes
within the 16-bit decode tolerance (|gpu - ref| <= 2e-3 + 1e-2 |ref|).
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
    assert np.isfinite(g).all(), what
    err = np.abs(g - ref)
    bad = err > 2e-3 + 1e-2 * np.abs(ref)
    assert not bad.any(), f"{what}: {bad.sum()} out of tolerance, max abs {err.max():.3e}"


def fp8_caches(pa, orc, case, k_scale, v_scale):
    """Quantise every attended token of a 16-bit case into 1-byte caches, on both sides."""
    NB, bs, Hkv, D = case.k_cache_post.shape
    slots = []
    for b in range(case.cfg.num_seqs):
        L = int(case.context_lens[b])
        pos = torch.arange(L)
        slots.append(case.block_tables[b, pos // bs].to(torch.int64) * bs + pos % bs)
    sm = torch.cat(slots)
    K = case.k_cache_post.view(NB * bs, Hkv, D)[sm].contiguous()
    V = case.v_cache_post.view(NB * bs, Hkv, D)[sm].contiguous()
    kc = torch.zeros((NB, bs, Hkv, D), dtype=torch.uint8)
    vc = torch.zeros_like(kc)
    assert orc.reshape_and_cache_fp8(kc, vc, K, V, sm, k_scale, v_scale) == 0
    kg = torch.zeros_like(kc).cuda()
    vg = torch.zeros_like(vc).cuda()
    pa.reshape_and_cache_fp8(K.cuda(), V.cuda(), kg, vg, sm.cuda(), k_scale, v_scale)
    torch.cuda.synchronize()
    assert torch.equal(kg.cpu(), kc), "K codes differ from the oracle's"
    assert torch.equal(vg.cpu(), vc), "V codes differ from the oracle's"
    return kc, vc, kg, vg


@pytest.mark.parametrize("name", ["llama3_8b_gqa", "llama2_7b", "long_context"])
def test_fp8_write_and_decode_small(pa, orc, name):
    lens = {"llama3_8b_gqa": [128, 250, 17, 5, 4096, 1024, 1, 16, 33],
            "llama2_7b": [64, 1, 77, 2048, 513],
            "long_context": [700, 1536, 32768]}[name]
    case = inputs.make_case(name, lens=lens)
    ks, vs = 0.0125, 0.011
    kc, vc, kg, vg = fp8_caches(pa, orc, case, ks, vs)
    ref = orc.paged_decode_fp8(case.q, kc, vc, ks, vs, case.block_tables, case.context_lens, case.scale)
    for P in (0, 64, 512):
        out = pa.decode_fp8(case.q.cuda(), kg, vg, ks, vs, case.block_tables.cuda(), case.context_lens.cuda(),
                            case.scale, max_context_len=case.max_context_len, partition_size=P)
        torch.cuda.synchronize()
        _close(out, ref, f"{name} P={P}")


@pytest.mark.parametrize("qdtype", ["bf16", "f16"])
@pytest.mark.parametrize("group", [1, 2, 4, 8])
def test_fp8_group_sizes(pa, orc, qdtype, group):
    cfg = inputs.DecodeConfig(f"fp8_g{group}", 8, 5, 2 * group, 2, 128, qdtype)
    case = inputs.make_case(cfg, lens=[1, 16, 100, 700, 37])
    kc, vc, kg, vg = fp8_caches(pa, orc, case, 0.02, 0.015)
    ref = orc.paged_decode_fp8(case.q, kc, vc, 0.02, 0.015, case.block_tables, case.context_lens, case.scale)
    out = pa.decode_fp8(case.q.cuda(), kg, vg, 0.02, 0.015, case.block_tables.cuda(), case.context_lens.cuda(),
                        case.scale, max_context_len=case.max_context_len)
    torch.cuda.synchronize()
    _close(out, ref, f"G={group} {qdtype}")


def test_fp8_full_size_gqa(pa, orc):
    cfg = inputs.CONFIGS["llama3_8b_gqa_fp8"]
    case = inputs.make_case(cfg)
    s = cfg.kv_scale
    kc, vc, kg, vg = fp8_caches(pa, orc, case, s, s)
    ref = orc.paged_decode_fp8(case.q, kc, vc, s, s, case.block_tables, case.context_lens, case.scale)
    out = pa.decode_fp8(case.q.cuda(), kg, vg, s, s, case.block_tables.cuda(), case.context_lens.cuda(), case.scale,
                        max_context_len=case.max_context_len)
    torch.cuda.synchronize()
    _close(out, ref, "llama3_8b_gqa_fp8 full size")


def test_fp8_saturation_and_signed_zero(pa, orc):
    # one token, one head: values beyond +-448*scale saturate, -0 and tiny negatives keep the sign
    vals = torch.tensor([0.0, -0.0, -1e-9, 1e9, -1e9, 447.0, 448.0, 465.0, 3 * 2 ** -10, 2 ** -10] + [0.5] * 118,
                        dtype=torch.float32)
    key = vals.to(torch.bfloat16).view(1, 1, 128)
    kc = torch.zeros((1, 16, 1, 128), dtype=torch.uint8)
    vc = torch.zeros_like(kc)
    sm = torch.tensor([5], dtype=torch.int64)
    assert orc.reshape_and_cache_fp8(kc, vc, key, key, sm, 1.0, 1.0) == 0
    kg, vg = kc.clone().cuda() * 0, vc.clone().cuda() * 0
    pa.reshape_and_cache_fp8(key.cuda(), key.cuda(), kg, vg, sm.cuda(), 1.0, 1.0)
    torch.cuda.synchronize()
    assert torch.equal(kg.cpu(), kc)
    assert kc[0, 5, 0, :8].tolist() == [0x00, 0x80, 0x80, 0x7E, 0xFE, 0x7E, 0x7E, 0x7E]


def test_fp8_copy_blocks(pa, orc):
    g = torch.Generator().manual_seed(5)
    k0 = torch.randint(0, 255, (12, 16, 2, 128), dtype=torch.uint8, generator=g)
    v0 = torch.randint(0, 255, (12, 16, 2, 128), dtype=torch.uint8, generator=g)
    pairs = torch.tensor([[1, 5], [1, 6], [2, 7]], dtype=torch.int64)
    kc, vc = k0.clone(), v0.clone()
    # the oracle copies blocks of bytes; view the 1-byte rows as 2-byte elements of half the width
    assert orc.copy_blocks(kc.view(torch.bfloat16), vc.view(torch.bfloat16), pairs) == 0
    kg, vg = k0.cuda(), v0.cuda()
    pa.copy_blocks(kg, vg, pairs.cuda())
    torch.cuda.synchronize()
    assert torch.equal(kg.cpu(), kc) and torch.equal(vg.cpu(), vc)
    code, _ = pa.get_device_error(clear=True)
    assert code == 0
