"""The block-manager oracle against its pins, and planted mistakes caught."""
import pytest

import block_manager_pins as pins
from oracle.block_manager import NoSpace, PagedBlockManager, StaticKVManager


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda f: f.__name__)
def test_oracle_pin(pin):
    pin(PagedBlockManager)


# ---- planted mistakes (in subclasses of the oracle, on the CPU) -------------------
class NoCopyOnWrite(PagedBlockManager):        # the sketch's behaviour: write into the shared block
    def append(self, seq):
        table = self.block_tables[seq]
        pos = self.context_lens[seq]
        if table and pos % self.block_size:
            self.context_lens[seq] = pos + 1
            return table[-1] * self.block_size + pos % self.block_size, None
        return super().append(seq)


class LifoFreeList(PagedBlockManager):         # pop() instead of pop(0)
    def allocate(self, seq, n):
        self.free_blocks.reverse()
        try:
            return super().allocate(seq, n)
        finally:
            self.free_blocks.reverse()


class FreeWithoutRefCount(PagedBlockManager):  # returns shared blocks while still referenced
    def free(self, seq):
        for b in self.block_tables.pop(seq):
            self.ref_count[b] = 0
            if b not in self.free_blocks:
                self.free_blocks.append(b)
        del self.context_lens[seq]


class CopyPairReversed(PagedBlockManager):
    def append(self, seq):
        slot, cow = super().append(seq)
        return slot, (cow[1], cow[0]) if cow else None


class NoFailureCheck(PagedBlockManager):       # partial allocation when the pool runs dry
    def allocate(self, seq, n):
        import math
        need = math.ceil(n / self.block_size)
        if need > len(self.free_blocks):
            self.block_tables[seq] = [self.free_blocks.pop(0) for _ in range(len(self.free_blocks))]
            self.context_lens[seq] = n
            raise NoSpace(seq)
        return super().allocate(seq, n)


@pytest.mark.parametrize("mutant", [NoCopyOnWrite, LifoFreeList, FreeWithoutRefCount, CopyPairReversed,
                                    NoFailureCheck], ids=lambda c: c.__name__)
def test_planted_mistake_is_caught(mutant):
    caught = []
    for pin in pins.ALL_PINS:
        try:
            pin(mutant)
        except (AssertionError, KeyError, IndexError, ValueError):
            caught.append(pin.__name__)
    assert caught, f"{mutant.__name__} passed every pin"


def test_static_allocator_utilisation():
    s = StaticKVManager(capacity_tokens=5 * 2048, max_seq_len=2048)
    lens = [100, 300, 512, 50, 1000]
    for i, n in enumerate(lens):
        s.allocate(i, n)
    with pytest.raises(NoSpace):
        s.allocate(9, 10)
    assert abs(s.stats()["allocated_utilization"] - sum(lens) / (5 * 2048)) < 1e-12
