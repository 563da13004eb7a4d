"""The C++ block manager (through the C ABI; host code, no GPU) against the
same pins as the oracle, and step by step against the oracle itself."""
import random

import numpy as np
import pytest

import block_manager_pins as pins
from oracle.block_manager import NoSpace as OracleNoSpace
from oracle.block_manager import PagedBlockManager


@pytest.fixture(scope="module")
def BM():
    from paged_kv_cache_464_b200 import build
    build.build()
    from paged_kv_cache_464_b200.block_manager import BlockManager
    return BlockManager


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda f: f.__name__)
def test_cpp_manager_pin(BM, pin):
    pin(BM)


def _state(m):
    return (m.free_blocks, m.block_tables, m.context_lens, m.ref_count)


@pytest.mark.parametrize("seed", range(8))
def test_cpp_manager_matches_oracle_step_by_step(BM, seed):
    rng = random.Random(seed)
    nb = rng.choice([16, 40, 128])
    a, b = BM(nb, 16), PagedBlockManager(nb, 16)
    live, next_seq = [], 0
    for _ in range(500):
        op = rng.random()
        n = rng.randint(0, 60)
        src = rng.choice(live) if live else None
        share_n = rng.randint(0, b.context_lens[src]) if src is not None else 0
        target = rng.choice(live) if live else None
        res = []
        for m, exc in ((a, a.NoSpace), (b, OracleNoSpace)):
            try:
                if op < 0.2 or not live:
                    r = ("alloc", m.allocate(next_seq, n))
                elif op < 0.35:
                    r = ("share", m.share_prefix(next_seq, src, share_n))
                elif op < 0.85:
                    r = ("append", m.append(target))
                else:
                    m.free(target)
                    r = ("free",)
            except exc:
                r = ("nospace",)
            res.append(r)
        assert res[0] == res[1], (res[0], res[1])
        assert _state(a) == _state(b)
        if res[0][0] in ("alloc", "share"):
            live.append(next_seq)
            next_seq += 1
        elif res[0][0] == "free":
            live.remove(target)
    assert a.stats() == b.stats()


def test_batch_step_and_tables(BM):
    a, b = BM(64, 16), PagedBlockManager(64, 16)
    for m in (a, b):
        m.allocate(0, 50)
        m.share_prefix(1, 0, 50)
        m.share_prefix(2, 0, 40)
        m.allocate(3, 16)
    slots, pairs, done = a.append_batch([1, 0, 2, 3])
    exp_slots, exp_pairs = [], []
    for s in [1, 0, 2, 3]:
        slot, cow = b.append(s)
        exp_slots.append(slot)
        if cow:
            exp_pairs.append(cow)
    assert done == 4 and slots.tolist() == exp_slots and pairs.tolist() == [list(p) for p in exp_pairs]
    tables, lens = a.tables([3, 0, 1, 2], 6)
    for row, s in zip(tables.tolist(), [3, 0, 1, 2]):
        t = b.block_tables[s]
        assert row == t + [-1] * (6 - len(t))
    assert lens.tolist() == [b.context_lens[s] for s in [3, 0, 1, 2]]
    with pytest.raises(Exception):
        a.tables([0], 2)       # a 4-block table does not fit 2 entries


def test_batch_stops_at_no_space(BM):
    a = BM(3, 16)
    a.allocate(0, 16)
    a.allocate(1, 16)
    a.allocate(2, 15)
    slots, pairs, done = a.append_batch([2, 0, 1])
    assert done == 1 and len(slots) == 1     # seq 2 had room; seq 0 needs a block and there is none
    assert a.context_lens == {0: 16, 1: 16, 2: 16}
