"""The seeded input recipe: the workloads' length draws (totals as stated in
the design notes), seeds, and the structure every case carries -- a shuffled
pool 1.25x the blocks needed, NaN in every slot no sequence owns, -1 past each
table's last block, the new token's slot poisoned before the step, and
copy-on-write destinations poisoned and owned by the one sequence whose shared
block they replace."""
import math

import numpy as np
import pytest
import torch

from paged_kv_cache_464_b200 import inputs

TOTALS = {"tiny": 200, "llama2_7b": 64352, "llama3_8b_gqa": 294533, "shared_prefix": 165789,
          "long_context": 262144, "llama3_8b_gqa_fp8": 297258}
BOUNDS = {"llama2_7b": (64, 2048), "llama3_8b_gqa": (128, 4096), "shared_prefix": (1040, 1536),
          "long_context": (32768, 32768), "llama3_8b_gqa_fp8": (128, 4096)}


@pytest.mark.parametrize("name", sorted(TOTALS))
def test_full_size_length_draws(name):
    cfg = inputs.CONFIGS[name]
    assert cfg.seed == 1000 + list(inputs.CONFIGS).index(name) + 1
    L = inputs._draw_lens(cfg, np.random.Generator(np.random.PCG64(cfg.seed)))
    assert len(L) == cfg.num_seqs and int(L.sum()) == TOTALS[name]
    if name in BOUNDS:
        lo, hi = BOUNDS[name]
        assert lo <= L.min() and L.max() <= hi


@pytest.mark.parametrize("name,lens", [("llama3_8b_gqa", [128, 250, 17, 5, 33]), ("tiny", None),
                                       ("shared_prefix", [1040, 1300, 1536, 1100]),
                                       ("llama2_7b", [64, 1, 77, 513])])
def test_case_structure(name, lens):
    case = inputs.make_case(name, lens=lens)
    bs = case.cfg.block_size
    L = case.context_lens.tolist()
    nb = case.k_cache.shape[0]
    need = sum(math.ceil(x / bs) for x in L)
    shared = case.cfg.name == "shared_prefix"
    if name == "tiny":
        assert nb == 64
    elif not shared:
        assert nb == math.ceil(1.25 * need)
    owners = {}
    for b, x in enumerate(L):
        row = case.block_tables[b].tolist()
        nblk = math.ceil(x / bs)
        assert all(i >= 0 for i in row[:nblk]) and all(i == -1 for i in row[nblk:]), "table tail must be -1"
        for lb, blk in enumerate(row[:nblk]):
            owners.setdefault(blk, set()).add((b, lb))
        # the new token (position L-1) is poisoned before the step and carried in key/value
        pos = x - 1
        slot = row[pos // bs] * bs + pos % bs
        assert int(case.slot_mapping[b]) == slot
        assert torch.isnan(case.k_cache.view(nb * bs, -1)[slot].float()).all()
    for blk, users in owners.items():
        if len(users) > 1:
            assert shared and all(lb < 1024 // bs for _, lb in users), "only prefix blocks are shared"
    # every slot no sequence owns holds NaN (stale), in both caches
    owned = torch.zeros(nb * bs, dtype=torch.bool)
    for b, x in enumerate(L):
        for pos in range(x):
            owned[int(case.block_tables[b, pos // bs]) * bs + pos % bs] = True
    for c in (case.k_cache, case.v_cache):
        rows = c.view(nb * bs, -1).float()
        assert torch.isnan(rows[~owned]).all()
    # copy-on-write: block_tables already point at the copy (shared_block_tables at the
    # source); a destination is poisoned before the step and owned by exactly one sequence,
    # in the place the shared source holds in its pre-copy table
    for src, dst in case.block_mapping.tolist():
        assert torch.isnan(case.k_cache[dst].float()).all() and torch.isnan(case.v_cache[dst].float()).all()
        (b, lb), = owners[dst]
        assert int(case.shared_block_tables[b, lb]) == src
        assert sum(int(r[lb]) == src for r in case.shared_block_tables.tolist()) > 1


def test_prefill_recipe_and_flop_count():
    """16 chunks of 512 tokens after prefixes drawn U[0, 1536] (seed 1007); the
    metric's unit, 4*Hq*D per causally visible (query, key) pair, from its
    closed form: a chunk of n queries after L-n cached tokens sees
    n(L-n) + n(n+1)/2 pairs."""
    case = inputs.make_prefill_case("llama3_8b_prefill")
    cfg = case.cfg
    assert cfg.seed == 1007 and cfg.num_seqs == 16
    qsl = case.query_start_loc.tolist()
    assert qsl == [512 * i for i in range(17)] and case.max_query_len == 512 and case.num_tokens == 8192
    L = case.context_lens.tolist()
    assert all(512 <= x <= 512 + 1536 for x in L) and (min(L), max(L)) == (595, 1888)
    pairs = sum(512 * (x - 512) + 512 * 513 // 2 for x in L)
    assert case.flops() == 4 * cfg.num_heads * cfg.head_dim * pairs == 130291859456
    assert case.kv_bytes_attended() == sum(L) * cfg.num_kv_heads * cfg.head_dim * 2 * 2


KV_BYTES = {"tiny": 409600, "llama2_7b": 1054343168, "llama3_8b_gqa": 1206407168, "shared_prefix": 679071744,
            "long_context": 1073741824, "llama3_8b_gqa_fp8": 608784384}


@pytest.mark.parametrize("name", sorted(KV_BYTES))
def test_decode_metric_bytes(name):
    """The decode metric's algorithmic bytes: every attended token's K and V
    rows once, sum_b L_b * Hkv * 2 * D * element size (1 byte for E4M3)."""
    cfg = inputs.CONFIGS[name]
    es = 1 if cfg.kv_dtype == "fp8_e4m3" else {"f32": 4, "f16": 2, "bf16": 2}[cfg.dtype]
    assert TOTALS[name] * cfg.num_kv_heads * 2 * cfg.head_dim * es == KV_BYTES[name]
    lens = {"tiny": None, "shared_prefix": [1040, 1100, 1300]}.get(name, [1, 16, 17, 300])
    small = inputs.make_case(name, lens=lens, with_post=False)
    assert small.kv_bytes() == int(small.context_lens.sum()) * cfg.num_kv_heads * 2 * cfg.head_dim * es
