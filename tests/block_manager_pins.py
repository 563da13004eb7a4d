"""Pins for block managers (the Python oracle and, through the same functions,
the C++ manager in the library).

A manager is driven through ``allocate / share_prefix / append / free`` and
checked against what paging means, independently of how it is coded:

* content model: every sequence has a ground-truth token list; a slot-indexed
  "memory" receives tokens only at the slots the manager returns, and block
  copies only for the (src, dst) pairs it returns.  After every operation,
  reading each live sequence through its block table must give back its
  tokens -- a write into a block that another sequence still reads, a lost
  copy, a wrong slot or a freed block still in use all break this;
* conservation: free blocks + blocks in use = pool; every block's reference
  count = the number of tables that hold it; the free list has no duplicates;
* failure atomicity: an operation that runs out of blocks changes nothing;
* FIFO reuse: freed blocks go to the back of the free list;
* utilisation in closed form for requests without sharing.
"""
from __future__ import annotations

import copy
import math
import random



def snapshot(m):
    return (list(m.free_blocks), {k: list(v) for k, v in m.block_tables.items()}, dict(m.context_lens),
            list(m.ref_count))


def check_conservation(m):
    in_use = set()
    counts = [0] * m.num_blocks
    for table in m.block_tables.values():
        assert len(set(table)) == len(table), "a table holds a block twice"
        for b in table:
            counts[b] += 1
            in_use.add(b)
    free = list(m.free_blocks)
    assert len(set(free)) == len(free), "duplicate in the free list"
    assert not (set(free) & in_use), "a block is both free and in use"
    assert len(free) + len(in_use) == m.num_blocks, "blocks lost or invented"
    assert list(m.ref_count) == counts, "reference counts differ from table membership"
    for seq, table in m.block_tables.items():
        assert len(table) == math.ceil(m.context_lens[seq] / m.block_size), "table length vs context length"


class ContentModel:
    """Ground-truth tokens per sequence and a slot -> token memory."""

    def __init__(self, m):
        self.m = m
        self.tokens = {}
        self.memory = {}
        self.next_token = 1

    def new_tokens(self, n):
        t = list(range(self.next_token, self.next_token + n))
        self.next_token += n
        return t

    def write(self, slots, toks):
        for s, t in zip(slots, toks):
            self.memory[s] = t

    def copy_block(self, src, dst):
        bs = self.m.block_size
        for o in range(bs):
            if src * bs + o in self.memory:
                self.memory[dst * bs + o] = self.memory[src * bs + o]
            else:
                self.memory.pop(dst * bs + o, None)

    def check(self):
        bs = self.m.block_size
        for seq, toks in self.tokens.items():
            table = self.m.block_tables[seq]
            got = [self.memory.get(table[p // bs] * bs + p % bs) for p in range(len(toks))]
            assert got == toks, f"sequence {seq} reads {got[:8]}... expected {toks[:8]}..."

    # driven operations -------------------------------------------------------------
    def allocate(self, seq, n):
        toks = self.new_tokens(n)
        slots = self.m.allocate(seq, n)
        self.write(slots, toks)
        self.tokens[seq] = toks

    def share(self, seq, src, n):
        slots = self.m.share_prefix(seq, src, n)
        toks = self.tokens[src][:n]
        self.write(slots, toks[n - len(slots):])
        self.tokens[seq] = list(toks)

    def append(self, seq):
        slot, cow = self.m.append(seq)
        if cow is not None:
            self.copy_block(*cow)
        tok = self.new_tokens(1)
        self.write([slot], tok)
        self.tokens[seq] = self.tokens[seq] + tok

    def free(self, seq):
        self.m.free(seq)
        del self.tokens[seq]


def random_ops(make_manager, seed, num_blocks=64, steps=600, bs=16):
    """Random interleaving of the four operations; checks after each one."""
    rng = random.Random(seed)
    m = make_manager(num_blocks, bs)
    c = ContentModel(m)
    next_seq = 0
    failures = 0
    for _ in range(steps):
        live = list(c.tokens)
        op = rng.random()
        before = snapshot(m)
        try:
            if op < 0.2 or not live:
                c.allocate(next_seq, rng.randint(0, 70))
                next_seq += 1
            elif op < 0.35:
                src = rng.choice(live)
                n = rng.randint(0, len(c.tokens[src]))
                c.share(next_seq, src, n)
                next_seq += 1
            elif op < 0.85:
                c.append(rng.choice(live))
            else:
                c.free(rng.choice(live))
        except m.NoSpace:
            failures += 1
            assert snapshot(m) == before, "a failed operation changed the manager"
        check_conservation(m)
        c.check()
    return m, failures


# ---------------------------------------------------------------------------- pins
def pin_content_and_conservation(make_manager):
    for seed in range(6):
        m, failures = random_ops(make_manager, seed)
    m, failures = random_ops(make_manager, 99, num_blocks=12, steps=400)   # a tight pool: many failures
    assert failures > 0


def pin_pages_share_then_append(make_manager):
    """The pages' demo: request 1 holds a 50-token prompt, request 3 shares the
    same 50-token prefix (all four blocks, the partial one included), then
    request 3 appends: its partial block is copied first."""
    m = make_manager(16, 16)
    m.allocate(1, 50)
    assert m.block_tables[1] == [0, 1, 2, 3]
    unshared = m.share_prefix(3, 1, 50)
    assert unshared == [] and m.block_tables[3] == [0, 1, 2, 3]
    assert list(m.ref_count[:4]) == [2, 2, 2, 2]
    slot, cow = m.append(3)
    assert cow == (3, 4) and slot == 4 * 16 + 2
    assert m.block_tables[3] == [0, 1, 2, 4] and list(m.ref_count[:5]) == [2, 2, 2, 1, 1]
    slot, cow = m.append(1)      # request 1 now owns block 3 alone: no copy
    assert cow is None and slot == 3 * 16 + 2


def pin_fifo_free_list(make_manager):
    m = make_manager(8, 16)
    m.allocate(0, 32)      # blocks 0, 1
    m.allocate(1, 16)      # block 2
    m.free(0)              # 0 and 1 go to the back
    m.allocate(2, 48)      # takes 3, 4, 5
    assert m.block_tables[2] == [3, 4, 5]
    m.allocate(3, 48)      # takes 6, 7, then the freed 0
    assert m.block_tables[3] == [6, 7, 0]


def pin_utilisation_closed_form(make_manager):
    rng = random.Random(4)
    m = make_manager(1000, 16)
    lens = [rng.randint(1, 300) for _ in range(20)]
    for i, n in enumerate(lens):
        m.allocate(i, n)
    st = m.stats()
    blocks = sum(math.ceil(n / 16) for n in lens)
    assert st["used_blocks"] == blocks and st["used_tokens"] == sum(lens)
    assert st["free_blocks"] == 1000 - blocks
    assert abs(st["allocated_utilization"] - sum(lens) / (16 * blocks)) < 1e-12
    assert abs(st["pool_utilization"] - sum(lens) / 16000) < 1e-12


def pin_no_space_is_atomic(make_manager):
    m = make_manager(4, 16)
    m.allocate(0, 60)
    before = snapshot(m)
    try:
        m.allocate(1, 17)
    except m.NoSpace:
        pass
    else:
        raise AssertionError("allocation beyond the pool must fail")
    assert snapshot(m) == before
    m.allocate(1, 0)
    try:
        m.append(0)      # block 3 holds 12 tokens: room, no new block needed
    except m.NoSpace:
        raise AssertionError("append into a block with room must not need a free block")


ALL_PINS = [pin_content_and_conservation, pin_pages_share_then_append, pin_fifo_free_list,
            pin_utilisation_closed_form, pin_no_space_is_atomic]
