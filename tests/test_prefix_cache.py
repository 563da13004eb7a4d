"""The C++ prefix-caching manager (through its binding) against the pins and,
decision by decision, against the oracle ("vLLM 原理与源码阅读", Prefix Caching)."""
import functools
import random

import pytest

from oracle.prefix_cache import PrefixCachingBlockManager
from paged_kv_cache_464_b200.block_manager import BlockManager
from tests import prefix_cache_pins as pins

Native = functools.partial(BlockManager, prefix_caching=True)
Native.NoSpace = BlockManager.NoSpace


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda f: f.__name__)
def test_native_pin(pin):
    pin(Native)


def _state(m):
    return (m.free_blocks, m.evictable, m.ref_count, m.block_tables, m.context_lens, m.prefix_stats())


@pytest.mark.parametrize("seed", range(4))
def test_native_matches_oracle_step_by_step(seed):
    """Random streams of prompts sharing system prefixes, decode appends and frees
    on a small pool: every slot, cached-token count, table, reference count, free
    list, evictable list and counter equal the oracle's after every operation."""
    rng = random.Random(100 + seed)
    nb = rng.choice([24, 48, 96])
    a, b = Native(nb, 16), PrefixCachingBlockManager(nb, 16)
    systems = [[rng.randrange(500) for _ in range(rng.choice([16, 40, 64, 100]))] for _ in range(3)]
    live = []
    for step in range(600):
        op = rng.random()
        if op < 0.45 or not live:
            seq = step
            toks = list(rng.choice(systems)[:rng.randrange(0, 101)]) + [rng.randrange(500) for _ in range(rng.randrange(0, 40))]
            if not toks:
                toks = [7]
            ra = rb = None
            try:
                ra = a.allocate_prompt(seq, toks)
            except a.NoSpace:
                ra = "nospace"
            try:
                rb = b.allocate_prompt(seq, toks)
            except b.NoSpace:
                rb = "nospace"
            assert ra == (rb if rb == "nospace" else (rb[0], rb[1])), (step, ra, rb)
            if ra != "nospace":
                live.append(seq)
        elif op < 0.75:
            seq = rng.choice(live)
            try:
                ra = a.append(seq)
            except a.NoSpace:
                ra = "nospace"
            try:
                rb = b.append(seq)
            except b.NoSpace:
                rb = "nospace"
            assert ra == rb, (step, ra, rb)
        else:
            seq = live.pop(rng.randrange(len(live)))
            a.free(seq)
            b.free(seq)
        assert _state(a) == _state(b), step
    st = b.prefix_stats()
    assert st["hit_blocks"] > 20 and st["evictions"] > 0 and st["queried_blocks"] > st["hit_blocks"], st


def test_plain_manager_allocate_prompt_caches_nothing():
    m = BlockManager(8, 16)
    slots, cached = m.allocate_prompt(0, list(range(40)))
    assert cached == 0 and slots == [b * 16 + p % 16 for p, b in ((p, m.table(0)[p // 16]) for p in range(40))]
    _, cached = m.allocate_prompt(2, list(range(40)))
    assert cached == 0 and m.prefix_stats()["cached_blocks"] == 0 and m.table(2) != m.table(0)
