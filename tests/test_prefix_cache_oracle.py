"""The prefix-caching oracle against its pins, and planted mistakes that a pin
must catch ("vLLM 原理与源码阅读", Prefix Caching)."""
import math

import pytest

from oracle.prefix_cache import PrefixCachingBlockManager
from tests import prefix_cache_pins as pins


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda f: f.__name__)
def test_oracle_pin(pin):
    pin(PrefixCachingBlockManager)


class PartialBlockHit(PrefixCachingBlockManager):
    """Mistake: the last, partial block of a prompt is matched and shared as well."""

    def longest_cached_prefix(self, tokens):
        hits = super().longest_cached_prefix(tokens)
        if len(tokens) % self.block_size and len(hits) == len(tokens) // self.block_size:
            for key, b in self.cache.items():
                if key[0] == (self.entry[hits[-1]] if hits else -1):
                    rest = tuple(tokens[len(hits) * self.block_size:])
                    if key[1][:len(rest)] == rest:
                        return hits + [b]
        return hits

    def allocate_prompt(self, seq, tokens):
        slots, cached = super().allocate_prompt(seq, tokens)
        return slots, min(len(tokens), len(self.block_tables[seq]) * self.block_size) if cached else cached


class NoRevive(PrefixCachingBlockManager):
    """Mistake: a hit on an evictable block leaves it on the evictable list."""

    def allocate_prompt(self, seq, tokens):
        hits = self.longest_cached_prefix(tokens)
        keep = [b for b in hits if self.ref_count[b] == 0]
        out = super().allocate_prompt(seq, tokens)
        for b in keep:
            if b not in self.evictable:
                self.evictable.append(b)
        return out


class MostRecentEviction(PrefixCachingBlockManager):
    """Mistake: evicts the most recently released cached block."""

    def _take(self):
        if self.free_blocks:
            return self.free_blocks.pop(0)
        b = self.evictable.pop()
        del self.cache[self.key_of.pop(b)]
        del self.entry[b]
        self.evictions += 1
        return b


class HeadFirstRelease(PrefixCachingBlockManager):
    """Mistake: a sequence releases its blocks first to last."""

    def free(self, seq):
        t = self.block_tables[seq]
        self.block_tables[seq] = list(reversed(t))
        super().free(seq)


class StaleEntry(PrefixCachingBlockManager):
    """Mistake: evicting a block keeps its cache entry."""

    def _take(self):
        if self.free_blocks:
            return self.free_blocks.pop(0)
        b = self.evictable.pop(0)
        self.key_of.pop(b)
        self.evictions += 1
        return b


class NoRevivedInCapacity(PrefixCachingBlockManager):
    """Mistake: the capacity check counts hit blocks that are evictable as free."""

    def _fits(self, need, hits):
        return need <= self._available()


@pytest.mark.parametrize("mutant", [PartialBlockHit, NoRevive, MostRecentEviction, HeadFirstRelease, StaleEntry,
                                    NoRevivedInCapacity], ids=lambda c: c.__name__)
def test_planted_mistake_is_caught(mutant):
    failed = []
    for pin in pins.ALL_PINS:
        try:
            pin(mutant)
        except Exception:
            failed.append(pin.__name__)
    assert failed, f"{mutant.__name__}: no pin fails"
