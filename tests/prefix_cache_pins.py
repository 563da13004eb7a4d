"""Pins of the prefix-caching block manager ("vLLM 原理与源码阅读", Prefix Caching).

Each pin takes a manager class with the oracle's interface, so the same pins
check the oracle, planted mistakes (which must fail one of them) and, through
the binding, the C++ manager.
"""
from __future__ import annotations

import random
from typing import Dict, List


def _prompt(rng: random.Random, prefix: List[int], extra: int) -> List[int]:
    return list(prefix) + [rng.randrange(32000) for _ in range(extra)]


def _table(m, seq):
    return m.table(seq) if hasattr(m, "table") else m.block_tables[seq]


def _check_state(m, live: Dict[int, List[int]], contents: Dict[int, List[int]]):
    """Conservation, reference counts and content of every live sequence."""
    bs = m.block_size
    counts = [0] * m.num_blocks
    for seq, toks in live.items():
        t = _table(m, seq)
        assert len(t) == (len(toks) + bs - 1) // bs
        for i, b in enumerate(t):
            counts[b] += 1
            held = toks[i * bs:(i + 1) * bs]
            assert contents[b][:len(held)] == held, f"block {b} of seq {seq} holds other tokens"
    rc = list(m.ref_count)
    for b in range(m.num_blocks):
        assert rc[b] == counts[b], (b, rc[b], counts[b])
    free, evictable = list(m.free_blocks), list(m.evictable)
    in_use = [b for b in range(m.num_blocks) if counts[b] > 0]
    assert sorted(free + evictable + in_use) == list(range(m.num_blocks)), "a block is lost or counted twice"


def _allocate(m, seq, toks, contents):
    """allocate_prompt plus the content model: new blocks receive the tokens they cover."""
    bs = m.block_size
    rc = list(m.ref_count)
    before = set(b for b in range(m.num_blocks) if rc[b] > 0)
    slots, cached = m.allocate_prompt(seq, toks)
    t = _table(m, seq)
    assert cached % bs == 0 and cached <= len(toks)
    for i, b in enumerate(t):
        if i * bs < cached:
            continue                                   # shared: must already hold these tokens (checked later)
        contents[b] = toks[i * bs:(i + 1) * bs]
    for p, s in enumerate(slots):
        assert s == t[p // bs] * bs + p % bs
    return cached, before


def pin_longest_prefix_brute_force(cls):
    """Without evictions, the cached tokens of a prompt are the longest run of
    leading full blocks it shares with any earlier prompt still cached."""
    rng = random.Random(11)
    m = cls(1024, 16)
    system = [rng.randrange(32000) for _ in range(70)]
    prompts: List[List[int]] = []
    contents: Dict[int, List[int]] = {}
    live = {}
    for seq in range(40):
        kind = rng.random()
        if kind < 0.4:
            toks = _prompt(rng, system[:rng.randrange(0, 71)], rng.randrange(0, 60))
        elif kind < 0.7 and prompts:
            base = rng.choice(prompts)
            toks = _prompt(rng, base[:rng.randrange(0, len(base) + 1)], rng.randrange(0, 40))
        else:
            toks = _prompt(rng, [], rng.randrange(1, 90))
        expect = 0
        for p in prompts:
            k = 0
            while (k + 1) * 16 <= min(len(p), len(toks)) and p[k * 16:(k + 1) * 16] == toks[k * 16:(k + 1) * 16]:
                k += 1
            expect = max(expect, k * 16)
        cached, _ = _allocate(m, seq, toks, contents)
        assert cached == expect, (seq, cached, expect)
        prompts.append(toks)
        live[seq] = toks
        if rng.random() < 0.3:                          # freed prompts stay cached (no pressure)
            victim = rng.choice(list(live))
            m.free(victim)
            del live[victim]
        _check_state(m, live, contents)


def pin_sharing_is_exact_under_eviction(cls):
    """With a small pool (constant eviction), every live sequence's blocks hold
    exactly its own tokens, reference counts match the tables, and no block is
    lost; a request that does not fit changes nothing."""
    rng = random.Random(12)
    m = cls(40, 16)
    system = [rng.randrange(1000) for _ in range(64)]
    contents: Dict[int, List[int]] = {}
    live: Dict[int, List[int]] = {}
    for seq in range(400):
        toks = _prompt(rng, system[:rng.choice([0, 16, 32, 48, 64])], rng.randrange(0, 50))
        if not toks:
            toks = [1]
        state = (list(m.free_blocks), list(m.evictable), list(m.ref_count))
        try:
            _allocate(m, seq, toks, contents)
            live[seq] = toks
        except m.NoSpace:
            assert (list(m.free_blocks), list(m.evictable), list(m.ref_count)) == state, "failed allocation changed state"
        while live and (rng.random() < 0.5 or len(live) > 6):
            victim = rng.choice(list(live))
            m.free(victim)
            del live[victim]
        _check_state(m, live, contents)


def pin_cached_prefixes_are_closed(cls):
    """Every cached block's prefix is cached too: a sequence holding a block holds
    its parent, so a parent's last reference never goes before its child's, and
    a sequence releases its blocks last to first, so among evictable blocks a
    child is always evicted before its parent."""
    rng = random.Random(13)
    m = cls(24, 16)
    base = [rng.randrange(50) for _ in range(80)]
    live = []
    for seq in range(300):
        toks = base[:rng.choice([16, 32, 48, 64, 80])] + [rng.randrange(50) for _ in range(rng.randrange(0, 20))]
        try:
            m.allocate_prompt(seq, toks)
            live.append(seq)
        except m.NoSpace:
            pass
        while live and (rng.random() < 0.5 or len(live) > 3):
            m.free(live.pop(rng.randrange(len(live))))
        entries = set(m.cache_entries())
        for parent, _tokens, _block in m.cache_items():
            assert parent == -1 or parent in entries, "a cached block outlived its prefix"


def pin_eviction_order(cls):
    """Free list first, then the least recently released cached block; a
    sequence releases its blocks last to first."""
    m = cls(4, 16)
    m.allocate_prompt(0, [1] * 32)                 # blocks b0, b1 (cached)
    t0 = list(_table(m, 0))
    m.allocate_prompt(1, [5] * 5)                  # a partial block, not cached
    m.free(0)                                      # released b1 then b0
    assert list(m.evictable) == [t0[1], t0[0]]
    m.allocate_prompt(2, [7] * 20)                 # needs 2: the free block first, then evicts b1
    t2 = _table(m, 2)
    assert t0[1] in t2 and t0[0] not in t2
    _, cached = m.allocate_prompt(3, [1] * 16)     # b0 is still cached: a hit
    assert cached == 16 and _table(m, 3)[0] == t0[0]


def pin_hit_revives_evictable(cls):
    """A hit on an evictable block takes it off the evictable list (it cannot be
    evicted while in use) and the capacity check counts that."""
    m = cls(2, 16)
    m.allocate_prompt(0, [4] * 16)
    b = _table(m, 0)[0]
    m.free(0)
    _, cached = m.allocate_prompt(1, [4] * 16 + [8] * 3)   # hit + one new block: fits exactly
    assert cached == 16 and b in _table(m, 1) and b not in list(m.evictable)
    try:
        m.allocate_prompt(2, [6] * 1)
        raise AssertionError("allocated past the pool")
    except m.NoSpace:
        pass
    # a hit that revives the only evictable block leaves one block for the rest
    m = cls(2, 16)
    m.allocate_prompt(0, [4] * 16)
    m.free(0)
    try:
        m.allocate_prompt(1, [4] * 16 + [8] * 20)   # needs 2 new blocks besides the hit: only 1 left
        raise AssertionError("allocated past the pool")
    except m.NoSpace:
        pass
    assert list(m.evictable) == [b] or len(list(m.evictable)) == 1


def pin_evicted_block_is_forgotten(cls):
    """An evicted block leaves the cache: once it holds other content, the prompt
    it used to hold misses."""
    m = cls(2, 16)
    a, x = [3] * 16, [5] * 32
    m.allocate_prompt(0, a)                   # block b0, cached
    b0 = _table(m, 0)[0]
    m.free(0)                                 # b0 evictable
    m.allocate_prompt(1, x)                   # the free block, then evicts b0 for x's second block
    assert b0 in _table(m, 1)
    m.free(1)
    _, cached = m.allocate_prompt(2, a)
    assert cached == 0, "an evicted block was still found in the cache"


def pin_stats(cls):
    m = cls(16, 16)
    m.allocate_prompt(0, [1] * 40)        # 2 full blocks queried, 0 hit
    m.allocate_prompt(1, [1] * 40)        # 2 queried, 2 hit
    m.free(0)
    st = m.prefix_stats()
    assert st["queried_blocks"] == 4 and st["hit_blocks"] == 2 and st["cached_blocks"] == 2
    assert st["evictable_blocks"] == 0     # the cached blocks are still used by seq 1


ALL_PINS = [pin_longest_prefix_brute_force, pin_sharing_is_exact_under_eviction, pin_cached_prefixes_are_closed,
            pin_eviction_order, pin_hit_revives_evictable, pin_evicted_block_is_forgotten, pin_stats]
