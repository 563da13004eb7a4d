"""The pages' worked examples (fixtures under tests/golden/, each citing its
page and section) through the oracle's block managers and the native one."""
import json
import os

import pytest

from oracle.block_manager import PagedBlockManager, StaticKVManager

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _native(num_blocks, block_size):
    from paged_kv_cache_464_b200.block_manager import BlockManager
    return BlockManager(num_blocks, block_size)


@pytest.mark.parametrize("make", [PagedBlockManager, _native], ids=["oracle", "native"])
def test_paged_manager_example(make):
    g = _load("paged_manager_example.json")
    exp = g["expected"]
    m = make(g["num_blocks"], g["block_size"])
    appended = []
    for op in g["ops"]:
        if op[0] == "allocate":
            first, last = exp["allocate_slots"][str(op[1])]
            assert list(m.allocate(op[1], op[2])) == list(range(first, last + 1))
        elif op[0] == "share_prefix":
            assert list(m.share_prefix(op[1], op[2], op[3])) == exp["share_prefix_new_slots"]
        elif op[0] == "append":
            slot, cow = m.append(op[1])
            appended.append([slot, list(cow) if cow is not None else None])
    assert appended == exp["append"]
    assert {str(k): list(v) for k, v in m.block_tables.items()} == exp["block_tables"]
    assert {str(k): v for k, v in m.context_lens.items()} == exp["context_lens"]
    rc = list(m.ref_count)
    assert {str(b): r for b, r in enumerate(rc) if r > 0} == exp["ref_count_nonzero"]
    st = m.stats()
    for k, v in exp["stats"].items():
        assert st[k] == v, (k, st[k], v)


def test_static_allocator_example():
    g = _load("static_allocator_example.json")
    exp = g["expected"]
    m = StaticKVManager(g["max_batch_size"] * g["max_seq_len"], g["max_seq_len"])
    for seq, n in g["requests"]:
        m.allocate(seq, n)
    st = m.stats()
    assert st["reserved_tokens"] == exp["reserved_tokens"]
    assert st["used_tokens"] == exp["used_tokens"]
    assert st["reserved_tokens"] - st["used_tokens"] == exp["wasted_tokens"]
    assert st["allocated_utilization"] == exp["allocated_utilization"]
    gib = g["bytes_per_token"] / 2 ** 30
    assert st["reserved_tokens"] * gib == exp["reserved_gib"]
    assert st["used_tokens"] * gib == exp["used_gib"]
    assert (st["reserved_tokens"] - st["used_tokens"]) * gib == exp["wasted_gib"]
