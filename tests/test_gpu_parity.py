"""GPU path (through the C ABI) against the CPU oracle on the same seeded inputs.

Bars: cache writes and block copies bit-exact over the whole cache; decode
within 1e-5 max-abs for fp32 caches and |gpu - ref| <= 2e-3 + 1e-2 |ref| for
fp16/bf16 caches (ref = fp64 oracle on the same rounded inputs).
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_464_b200 import inputs

pytestmark = pytest.mark.gpu

TOL_F32_ABS = 1e-5
TOL_16_ABS, TOL_16_REL = 2e-3, 1e-2


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


@pytest.fixture(autouse=True)
def no_device_error(request):
    """Every test that does not expect one must leave the device error word clean."""
    yield
    if "pa" in request.fixturenames and "expects_device_error" not in request.keywords:
        from paged_kv_cache_464_b200 import capi
        code, detail = capi.get_device_error(clear=True)
        assert code == 0, f"device error {capi.DEVICE_ERRORS.get(code)} detail {detail}"


def assert_decode_close(gpu: torch.Tensor, ref: np.ndarray, dtype: str, what: str = ""):
    g = gpu.detach().to(torch.float64).cpu().numpy()
    assert g.shape == ref.shape
    assert np.isfinite(g).all(), f"{what}: non-finite GPU output"
    err = np.abs(g - ref)
    if dtype == "f32":
        assert err.max() <= TOL_F32_ABS, f"{what}: max abs err {err.max():.3e}"
    else:
        bound = TOL_16_ABS + TOL_16_REL * np.abs(ref)
        bad = err > bound
        assert not bad.any(), (f"{what}: {bad.sum()} elements out of tolerance; max abs {err.max():.3e}, "
                               f"max rel {(err / np.maximum(np.abs(ref), 1e-30)).max():.3e}")


def to_dev(case):
    dev = "cuda"
    return dict(q=case.q.to(dev), k=case.k_cache.to(dev), v=case.v_cache.to(dev), key=case.key.to(dev),
                value=case.value.to(dev), slots=case.slot_mapping.to(dev), pairs=case.block_mapping.to(dev),
                bt=case.block_tables.to(dev), cl=case.context_lens.to(dev))


def gpu_step(pa, case, partition_size=None):
    d = to_dev(case)
    if case.block_mapping.numel():
        pa.copy_blocks(d["k"], d["v"], d["pairs"])
    pa.reshape_and_cache(d["key"], d["value"], d["k"], d["v"], d["slots"])
    P = case.cfg.partition_size if partition_size is None else partition_size
    out = pa.decode(d["q"], d["k"], d["v"], d["bt"], d["cl"], case.scale, max_context_len=case.max_context_len,
                    partition_size=P)
    torch.cuda.synchronize()
    return out, d


def _bytes(t):
    return t.contiguous().cpu().view(torch.uint8)


SMALL = {
    "tiny": None,
    "llama2_7b": [64, 1, 77, 200, 1000, 2048, 513, 16, 17],
    "llama3_8b_gqa": [128, 250, 17, 5, 4096, 1024, 511, 512, 513],
    "shared_prefix": [1040, 1124, 1536, 1057, 1030, 1025, 1200, 1300],
    "long_context": [700, 1536, 32768],
}


@pytest.mark.parametrize("name", inputs.BASE_WORKLOADS)
def test_step_small(pa, orc, name):
    """copy-on-write copies, new-token write and decode on small cases of every workload."""
    case = inputs.make_case(name, lens=SMALL[name])
    out, d = gpu_step(pa, case)
    ref, k_ref, v_ref = orc.step(case)
    assert torch.equal(_bytes(d["k"]), _bytes(k_ref)), "K cache after the step"
    assert torch.equal(_bytes(d["v"]), _bytes(v_ref)), "V cache after the step"
    assert_decode_close(out, ref, case.cfg.dtype, name)


@pytest.mark.parametrize("name", inputs.BASE_WORKLOADS)
def test_step_full_size(pa, orc, name):
    """Every workload at its full size, all outputs, in the launch configuration the benchmark times."""
    case = inputs.make_case(name, with_post=False)
    out, d = gpu_step(pa, case)
    ref, k_ref, v_ref = orc.step(case)
    assert torch.equal(_bytes(d["k"]), _bytes(k_ref))
    assert torch.equal(_bytes(d["v"]), _bytes(v_ref))
    assert_decode_close(out, ref, case.cfg.dtype, name)


@pytest.mark.parametrize("P", [16, 32, 64, 512, 4096, 0])
def test_split_k_partition_sizes(pa, orc, P):
    case = inputs.make_case("llama3_8b_gqa", lens=[1, 15, 16, 17, 31, 32, 33, 511, 512, 513, 1000, 2500])
    out, _ = gpu_step(pa, case, partition_size=P)
    ref = orc.decode_case(case)
    assert_decode_close(out, ref, "bf16", f"P={P}")


@pytest.mark.parametrize("np_max", [2, 3, 5, 9, 17, 33, 65])
@pytest.mark.parametrize("dtype,D", [("f32", 64), ("bf16", 128)])
def test_split_k_reduce_paths(pa, orc, np_max, dtype, D):
    """Every way the reduce splits a row's partitions over warps (1, 2, 4 or 8
    warps a row, chosen from the longest context's partition count), with rows
    of 1 .. np_max partitions side by side; odd partition counts leave each
    row's partials at every alignment."""
    P = 64
    lens = [P * np_max, P * np_max - 5, P + 1, P, 1, P * (np_max // 2) + 3, 2 * P + 7, max(1, P * np_max - 63)]
    cfg = inputs.DecodeConfig(f"reduce_{dtype}", 9, len(lens), 8, 2, D, dtype)
    case = inputs.make_case(cfg, lens=lens)
    out, _ = gpu_step(pa, case, partition_size=P)
    assert_decode_close(out, orc.decode_case(case), dtype, f"{np_max} partitions, {dtype}")


@pytest.mark.parametrize("dtype,D", [("f32", 64), ("f16", 128), ("bf16", 128)])
@pytest.mark.parametrize("group", [1, 2, 4, 8])
def test_group_sizes_and_dtypes(pa, orc, dtype, D, group):
    cfg = inputs.DecodeConfig(f"g{group}_{dtype}", 7, 5, 2 * group, 2, D, dtype)
    case = inputs.make_case(cfg, lens=[1, 16, 100, 700, 37])
    for P in (0, 64):
        out, _ = gpu_step(pa, case, partition_size=P)
        ref = orc.decode_case(case)
        assert_decode_close(out, ref, dtype, f"G={group} {dtype} P={P}")


@pytest.mark.parametrize("name", ["tiny", "llama2_7b", "llama3_8b_gqa"])
def test_length_one_returns_v_exactly(pa, name):
    case = inputs.make_case(name, lens=[1, 1, 1, 1])
    out, d = gpu_step(pa, case)
    G = case.cfg.group
    v = case.v_cache_post.view(-1, case.cfg.num_kv_heads, case.cfg.head_dim)[case.slot_mapping]  # [S, Hkv, D]
    expect = v.repeat_interleave(G, dim=1)
    assert torch.equal(out.cpu(), expect), "L=1 must return V bit-exactly"


def test_block_permutation_bit_identical(pa):
    case = inputs.make_case("llama3_8b_gqa", lens=[300, 1000, 17, 4096])
    a, _ = gpu_step(pa, case)
    b, _ = gpu_step(pa, inputs.permute_blocks(case, seed=11))
    assert torch.equal(a.cpu(), b.cpu()), "outputs must not depend on physical block ids"


def test_copy_on_write_invariant_bit_identical(pa):
    """Sequences that copied the shared block must read what the shared block holds."""
    case = inputs.make_case("shared_prefix", lens=SMALL["shared_prefix"])
    out, d = gpu_step(pa, case)
    out_shared = pa.decode(d["q"], d["k"], d["v"], case.shared_block_tables.cuda(), d["cl"], case.scale,
                           max_context_len=case.max_context_len)
    assert torch.equal(out.cpu(), out_shared.cpu())


def test_empty_context_gives_zeros(pa, orc):
    case = inputs.make_case("llama3_8b_gqa", lens=[5, 40, 7])
    d = to_dev(case)
    k, v = case.k_cache_post.cuda(), case.v_cache_post.cuda()
    cl = d["cl"].clone()
    cl[1] = 0
    out = torch.full_like(d["q"], float("nan"))
    pa.decode(d["q"], k, v, d["bt"], cl, case.scale, out=out, max_context_len=40, partition_size=16)
    torch.cuda.synchronize()
    assert torch.equal(out[1].cpu(), torch.zeros_like(out[1].cpu()))
    ref = orc.paged_decode(case.q, case.k_cache_post, case.v_cache_post, case.block_tables, cl.cpu(), case.scale)
    assert_decode_close(out, ref, "bf16")


def test_noncontiguous_free_blocks_and_garbage_table_tail(pa, orc):
    """Entries past a sequence's last block are never read, whatever they hold."""
    case = inputs.make_case("llama2_7b", lens=[17, 300, 64])
    bt = case.block_tables.clone()
    bt[bt < 0] = 2 ** 31 - 1
    out, _ = gpu_step(pa, dataclasses.replace(case, block_tables=bt))
    assert_decode_close(out, orc.decode_case(case), "f16")


@pytest.mark.expects_device_error
def test_bad_block_id_is_recorded_not_faulted(pa):
    case = inputs.make_case("tiny")
    d = to_dev(case)
    bt = d["bt"].clone()
    bt[2, 1] = case.num_blocks + 5
    pa.get_device_error(clear=True)
    pa.decode(d["q"], d["k"], d["v"], bt, d["cl"], case.scale, max_context_len=case.max_context_len)
    code, detail = pa.get_device_error(clear=True)
    assert code == 1 and detail == case.num_blocks + 5


@pytest.mark.expects_device_error
def test_bad_slot_is_recorded_and_skipped(pa):
    case = inputs.make_case("tiny")
    d = to_dev(case)
    slots = d["slots"].clone()
    slots[0] = case.num_blocks * 16 + 3
    slots[1] = -1
    k0 = d["k"].clone()
    pa.get_device_error(clear=True)
    pa.reshape_and_cache(d["key"], d["value"], d["k"], d["v"], slots)
    code, detail = pa.get_device_error(clear=True)
    assert code == 2 and detail == case.num_blocks * 16 + 3
    # only tokens 2 and 3 were written
    expect = k0.clone()
    flat = expect.view(-1, case.cfg.num_kv_heads, case.cfg.head_dim)
    flat[d["slots"][2:]] = d["key"][2:]
    assert torch.equal(_bytes(d["k"]), _bytes(expect))


@pytest.mark.expects_device_error
def test_copy_conflicts_match_oracle(pa, orc):
    g = torch.Generator().manual_seed(3)
    k0 = torch.randn(12, 16, 2, 128, generator=g).to(torch.bfloat16)
    v0 = torch.randn(12, 16, 2, 128, generator=g).to(torch.bfloat16)
    for pairs, expect_code in [([[1, 5], [1, 6], [2, 7]], 0), ([[1, 5], [2, 5], [3, 8]], 3),
                               ([[1, 5], [5, 9], [4, 4]], 3), ([[1, 12], [-1, 3], [2, 3]], 1)]:
        bm = torch.tensor(pairs, dtype=torch.int64)
        kc, vc = k0.clone(), v0.clone()
        orc.copy_blocks(kc, vc, bm)
        kg, vg = k0.cuda(), v0.cuda()
        pa.get_device_error(clear=True)
        pa.copy_blocks(kg, vg, bm.cuda())
        code, _ = pa.get_device_error(clear=True)
        assert code == expect_code, pairs
        assert torch.equal(_bytes(kg), _bytes(kc)) and torch.equal(_bytes(vg), _bytes(vc)), pairs


@pytest.mark.expects_device_error
def test_context_len_beyond_bound_is_recorded(pa):
    case = inputs.make_case("tiny")
    d = to_dev(case)
    pa.get_device_error(clear=True)
    pa.decode(d["q"], d["k"], d["v"], d["bt"], d["cl"], case.scale, max_context_len=50)
    code, detail = pa.get_device_error(clear=True)
    assert code == 4 and detail == 3


def test_streams_and_repeat_determinism(pa):
    case = inputs.make_case("llama3_8b_gqa", lens=[900, 33, 4000])
    d = to_dev(case)
    k, v = case.k_cache_post.cuda(), case.v_cache_post.cuda()
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        a = pa.decode(d["q"], k, v, d["bt"], d["cl"], case.scale, max_context_len=4000)
        b = pa.decode(d["q"], k, v, d["bt"], d["cl"], case.scale, max_context_len=4000)
    s.synchronize()
    assert torch.equal(a.cpu(), b.cpu())


def gpu_step_append(pa, case, partition_size=None):
    """The step through the fused entry point: copies, then write + decode in one launch."""
    d = to_dev(case)
    if case.block_mapping.numel():
        pa.copy_blocks(d["k"], d["v"], d["pairs"])
    P = case.cfg.partition_size if partition_size is None else partition_size
    out = pa.decode_append(d["q"], d["key"], d["value"], d["k"], d["v"], d["bt"], d["cl"], case.scale,
                           max_context_len=case.max_context_len, partition_size=P)
    torch.cuda.synchronize()
    return out, d


@pytest.mark.parametrize("name", inputs.BASE_WORKLOADS)
def test_append_step_small(pa, orc, name):
    case = inputs.make_case(name, lens=SMALL[name])
    out, d = gpu_step_append(pa, case)
    ref, k_ref, v_ref = orc.step(case)
    assert torch.equal(_bytes(d["k"]), _bytes(k_ref)), "K cache after the fused step"
    assert torch.equal(_bytes(d["v"]), _bytes(v_ref)), "V cache after the fused step"
    assert_decode_close(out, ref, case.cfg.dtype, name)
    # the fused launch computes exactly what the two separate calls compute
    out2, _ = gpu_step(pa, case)
    assert torch.equal(out.cpu(), out2.cpu())


@pytest.mark.parametrize("name", inputs.BASE_WORKLOADS)
def test_append_step_full_size(pa, orc, name):
    case = inputs.make_case(name, with_post=False)
    out, d = gpu_step_append(pa, case)
    ref, k_ref, v_ref = orc.step(case)
    assert torch.equal(_bytes(d["k"]), _bytes(k_ref))
    assert torch.equal(_bytes(d["v"]), _bytes(v_ref))
    assert_decode_close(out, ref, case.cfg.dtype, name)


@pytest.mark.parametrize("P", [16, 64, 1024])
def test_append_partition_sizes_and_edges(pa, orc, P):
    case = inputs.make_case("llama3_8b_gqa", lens=[1, 15, 16, 17, 31, 32, 33, 1023, 1024, 1025, 3000])
    out, d = gpu_step_append(pa, case, partition_size=P)
    ref, k_ref, v_ref = orc.step(case)
    assert torch.equal(_bytes(d["k"]), _bytes(k_ref))
    assert_decode_close(out, ref, "bf16", f"P={P}")
