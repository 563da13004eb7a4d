"""Block manager oracle (test infrastructure only; plain Python, small sizes).

Restates the paged KV block manager of "vLLM推理引擎深度解析" §三
(PagedAttentionManager: block pool, free list, per-request block table,
allocate_request, append_token, free_request, share_prefix, get_stats) with
the readings this repository takes where the sketch is buggy or silent:

* one block table per sequence ("vLLM 原理与源码阅读", Block 管理器, item 1);
* a write into a block whose reference count is above one first copies the
  block (copy-on-write, same page, item 3) -- the sketch's share_prefix
  followed by append_token writes into the shared block without copying;
* allocation failure is reported (the sketch returns False / marks the request
  finished; "vLLM推理引擎深度实战" §1.2 raises MemoryError) and changes nothing;
* the free list is first-in first-out: blocks are taken from its front
  (``pop(0)`` in allocate_request and append_token) and returned to its back
  (``append`` in free_request).

Also restates TraditionalKVCacheManager (§二): a static allocator that
reserves ``max_seq_len`` token slots per request, for the utilisation
comparison.

Only tests, smoke() and the benchmark's CPU legs may import this module.
"""
from __future__ import annotations

import math
from typing import Dict, List, Optional, Tuple


class NoSpace(Exception):
    """The pool has no free block for the request (nothing was changed)."""


class PagedBlockManager:
    NoSpace = NoSpace

    def __init__(self, num_blocks: int, block_size: int = 16):
        self.num_blocks = num_blocks
        self.block_size = block_size
        self.ref_count = [0] * num_blocks
        self.num_tokens = [0] * num_blocks          # tokens stored in each block
        self.free_blocks: List[int] = list(range(num_blocks))
        self.block_tables: Dict[int, List[int]] = {}
        self.context_lens: Dict[int, int] = {}

    # -- helpers -----------------------------------------------------------------
    def _slot(self, seq: int, pos: int) -> int:
        """Position ``pos`` of ``seq`` lives in logical block pos // bs at offset pos % bs."""
        return self.block_tables[seq][pos // self.block_size] * self.block_size + pos % self.block_size

    def slots(self, seq: int, start: int, stop: int) -> List[int]:
        return [self._slot(seq, p) for p in range(start, stop)]

    def _available(self) -> int:
        """Blocks an allocation may take."""
        return len(self.free_blocks)

    def _take(self) -> int:
        """The next block to hand out: the front of the free list."""
        return self.free_blocks.pop(0)

    # -- allocate_request ------------------------------------------------------------
    def allocate(self, seq: int, num_tokens: int) -> List[int]:
        """Blocks for a new request's prompt: ceil(n / bs) blocks from the front of
        the free list, reference count 1.  Returns the slots of the n tokens."""
        assert seq not in self.block_tables
        need = math.ceil(num_tokens / self.block_size)
        if need > self._available():
            raise NoSpace(seq)
        table = []
        left = num_tokens
        for _ in range(need):
            b = self._take()
            self.ref_count[b] = 1
            self.num_tokens[b] = min(self.block_size, left)
            left -= self.num_tokens[b]
            table.append(b)
        self.block_tables[seq] = table
        self.context_lens[seq] = num_tokens
        return self.slots(seq, 0, num_tokens)

    # -- append_token ------------------------------------------------------------------
    def append(self, seq: int) -> Tuple[int, Optional[Tuple[int, int]]]:
        """Slot for the sequence's next token, and the (src, dst) block copy to issue
        first when the last block is shared.  The token goes into the last block if
        it has room, else into a new block from the front of the free list."""
        table = self.block_tables[seq]
        pos = self.context_lens[seq]
        offset = pos % self.block_size
        cow = None
        if table and offset != 0:
            last = table[-1]
            if self.ref_count[last] > 1:                        # shared: copy before writing
                if not self._available():
                    raise NoSpace(seq)
                new = self._take()
                self.ref_count[last] -= 1
                self.ref_count[new] = 1
                self.num_tokens[new] = offset
                table[-1] = new
                cow = (last, new)
                last = new
            self.num_tokens[last] = offset + 1
        else:
            if not self._available():
                raise NoSpace(seq)
            last = self._take()
            self.ref_count[last] = 1
            self.num_tokens[last] = 1
            table.append(last)
        self.context_lens[seq] = pos + 1
        return last * self.block_size + offset, cow

    # -- free_request -------------------------------------------------------------------
    def free(self, seq: int) -> None:
        for b in self.block_tables.pop(seq):
            self.ref_count[b] -= 1
            if self.ref_count[b] == 0:
                self.num_tokens[b] = 0
                self.free_blocks.append(b)
        del self.context_lens[seq]

    # -- share_prefix ---------------------------------------------------------------------
    def share_prefix(self, seq: int, src: int, num_tokens: int) -> List[int]:
        """A new request whose first ``num_tokens`` tokens equal those of ``src``:
        src's blocks are shared (reference count + 1) while the tokens they hold
        fit in the prefix; the rest of the prefix gets new blocks.  Returns the
        slots of the tokens that were not shared (the caller writes their K/V)."""
        assert seq not in self.block_tables and src in self.block_tables
        assert num_tokens <= self.context_lens[src]
        shared, covered = [], 0
        for b in self.block_tables[src]:
            held = min(self.block_size, self.context_lens[src] - covered)
            if covered + held <= num_tokens:
                shared.append(b)
                covered += held
            else:
                break
        need = math.ceil((num_tokens - covered) / self.block_size)
        if need > self._available():
            raise NoSpace(seq)
        for b in shared:
            self.ref_count[b] += 1
        table = list(shared)
        left = num_tokens - covered
        for _ in range(need):
            b = self._take()
            self.ref_count[b] = 1
            self.num_tokens[b] = min(self.block_size, left)
            left -= self.num_tokens[b]
            table.append(b)
        self.block_tables[seq] = table
        self.context_lens[seq] = num_tokens
        return self.slots(seq, covered, num_tokens)

    # -- get_stats --------------------------------------------------------------------------
    def stats(self) -> Dict[str, float]:
        used_blocks = sum(1 for r in self.ref_count if r > 0)
        used_tokens = sum(n for n, r in zip(self.num_tokens, self.ref_count) if r > 0)
        logical_tokens = sum(self.context_lens.values())
        cap = self.num_blocks * self.block_size
        return {
            "total_blocks": self.num_blocks,
            "free_blocks": len(self.free_blocks),
            "used_blocks": used_blocks,
            "used_tokens": used_tokens,
            "logical_tokens": logical_tokens,
            "pool_utilization": used_tokens / cap if cap else 0.0,
            "allocated_utilization": used_tokens / (used_blocks * self.block_size) if used_blocks else 0.0,
            "num_sequences": len(self.block_tables),
        }


class StaticKVManager:
    """§二 TraditionalKVCacheManager: every request reserves max_seq_len slots."""

    NoSpace = NoSpace

    def __init__(self, capacity_tokens: int, max_seq_len: int):
        self.capacity = capacity_tokens
        self.max_seq_len = max_seq_len
        self.lens: Dict[int, int] = {}

    def allocate(self, seq: int, num_tokens: int) -> None:
        if (len(self.lens) + 1) * self.max_seq_len > self.capacity or num_tokens > self.max_seq_len:
            raise NoSpace(seq)
        self.lens[seq] = num_tokens

    def append(self, seq: int) -> None:
        if self.lens[seq] + 1 > self.max_seq_len:
            raise NoSpace(seq)
        self.lens[seq] += 1

    def free(self, seq: int) -> None:
        del self.lens[seq]

    def stats(self) -> Dict[str, float]:
        reserved = len(self.lens) * self.max_seq_len
        used = sum(self.lens.values())
        return {"reserved_tokens": reserved, "used_tokens": used,
                "allocated_utilization": used / reserved if reserved else 0.0,
                "num_sequences": len(self.lens)}
