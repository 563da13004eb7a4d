"""Many decode steps driven by the C++ block manager through the C ABI, against
the oracle manager + the CPU oracle on the same seeded operations.

Per step: the manager appends one token to every live sequence (slots and
copy-on-write pairs), the GPU runs pa_copy_blocks then pa_decode_append; the
oracle side makes the same decisions with its own manager and runs copies,
slot writes and fp64 decode.  Decisions must be identical, outputs within the
decode tolerance, and the caches bit-identical at the end.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle.block_manager import PagedBlockManager

pytestmark = pytest.mark.gpu

DT = {"bf16": torch.bfloat16, "f16": torch.float16, "f32": torch.float32}


def _close(out, ref, dtype):
    g = out.to(torch.float64).cpu().numpy()
    err = np.abs(g - ref)
    assert np.isfinite(g).all()
    if dtype == "f32":
        assert err.max() <= 1e-5, err.max()
    else:
        assert (err <= 2e-3 + 1e-2 * np.abs(ref)).all(), err.max()


@pytest.mark.parametrize("dtype,Hq,Hkv,D", [("bf16", 8, 2, 128), ("f16", 4, 4, 128), ("f32", 4, 2, 64)])
def test_managed_decode_steps(dtype, Hq, Hkv, D):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from paged_kv_cache_464_b200 import capi
    from paged_kv_cache_464_b200.block_manager import BlockManager
    capi.get_device_error(clear=True)
    orc = oracle.get()
    rng = np.random.default_rng(7)
    gen = torch.Generator().manual_seed(7)
    tdt = DT[dtype]
    NB, bs, MBS = 96, 16, 16
    scale = float(np.float32(1 / np.sqrt(D)))

    k_cpu = torch.full((NB, bs, Hkv, D), float("nan"), dtype=tdt)
    v_cpu = torch.full_like(k_cpu, float("nan"))
    k_gpu, v_gpu = k_cpu.cuda(), v_cpu.cuda()
    mgr, ref = BlockManager(NB, bs), PagedBlockManager(NB, bs)

    def rows(n):
        return (torch.randn((n, Hkv, D), generator=gen).to(tdt), torch.randn((n, Hkv, D), generator=gen).to(tdt))

    def write(slots, kr, vr):
        if not slots:
            return
        s = torch.tensor(slots, dtype=torch.int64)
        assert orc.reshape_and_cache(k_cpu, v_cpu, kr, vr, s) == 0
        capi.reshape_and_cache(kr.cuda(), vr.cuda(), k_gpu, v_gpu, s.cuda())

    def allocate(seq, n):
        slots = mgr.allocate(seq, n)
        assert slots == ref.allocate(seq, n)
        write(slots, *rows(n))

    def share(seq, src, n):
        slots = mgr.share_prefix(seq, src, n)
        assert slots == ref.share_prefix(seq, src, n)
        # the unshared prefix tokens get the source's rows
        src_slots = torch.tensor(ref.slots(src, n - len(slots), n), dtype=torch.int64)
        flat_k, flat_v = k_cpu.view(-1, Hkv, D), v_cpu.view(-1, Hkv, D)
        write(slots, flat_k[src_slots].clone(), flat_v[src_slots].clone())

    def free(seq):
        mgr.free(seq)
        ref.free(seq)

    allocate(0, 50)          # a system prompt ending in a partial block
    for s in (1, 2, 3):
        share(s, 0, 50)      # all four blocks shared, the partial one too
    allocate(4, int(rng.integers(1, 90)))
    allocate(5, 0)
    share(6, 4, int(rng.integers(0, ref.context_lens[4] + 1)))
    next_seq = 7
    total_pairs = 0
    for step in range(40):
        if step == 15:
            free(2)
            allocate(next_seq, 33)
            next_seq += 1
        if step == 25:
            share(next_seq, 1, ref.context_lens[1] - 5)
            next_seq += 1
        live = ref.block_tables and sorted(ref.block_tables)
        slots, pairs, done = mgr.append_batch(live)
        assert done == len(live)
        exp_slots, exp_pairs = [], []
        for s in live:
            slot, cow = ref.append(s)
            exp_slots.append(slot)
            if cow:
                exp_pairs.append(list(cow))
        assert slots.tolist() == exp_slots and pairs.tolist() == exp_pairs
        total_pairs += len(exp_pairs)
        tables, lens = mgr.tables(live, MBS)
        # the manager's slot is the append rule applied to its own table
        for i, s in enumerate(live):
            L = int(lens[i])
            assert slots[i] == tables[i, (L - 1) // bs] * bs + (L - 1) % bs
        S = len(live)
        q = torch.randn((S, Hq, D), generator=gen).to(tdt)
        kn, vn = rows(S)
        bt = torch.from_numpy(np.ascontiguousarray(tables))
        cl = torch.from_numpy(np.ascontiguousarray(lens))
        # GPU: copies, then new-token write + decode in one launch
        if len(pairs):
            capi.copy_blocks(k_gpu, v_gpu, torch.from_numpy(np.ascontiguousarray(pairs)).cuda())
        out = capi.decode_append(q.cuda(), kn.cuda(), vn.cuda(), k_gpu, v_gpu, bt.cuda(), cl.cuda(), scale,
                                 max_context_len=int(lens.max()), partition_size=32)
        # oracle
        if exp_pairs:
            assert orc.copy_blocks(k_cpu, v_cpu, torch.tensor(exp_pairs, dtype=torch.int64)) == 0
        assert orc.reshape_and_cache(k_cpu, v_cpu, kn, vn, torch.tensor(exp_slots, dtype=torch.int64)) == 0
        expect = orc.paged_decode(q, k_cpu, v_cpu, bt, cl, scale)
        torch.cuda.synchronize()
        _close(out, expect, dtype)
    assert total_pairs >= 3                      # the shared partial block was copied on write
    assert torch.equal(k_gpu.cpu().view(torch.uint8), k_cpu.view(torch.uint8))
    assert torch.equal(v_gpu.cpu().view(torch.uint8), v_cpu.view(torch.uint8))
    assert mgr.stats() == ref.stats()
    code, detail = capi.get_device_error(clear=True)
    assert code == 0, (code, detail)
