"""ctypes binding of the host block manager (include/pa_block_manager.h).

Marshalling only: every decision (free list, reference counts, copy-on-write,
slots) is made by the C++ manager in libpa_b200.so.
"""
from __future__ import annotations

import ctypes
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np

from .capi import _lib

_P, _I32, _I64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64


class _Stats(ctypes.Structure):
    _fields_ = [("total_blocks", ctypes.c_int64), ("free_blocks", ctypes.c_int64),
                ("used_blocks", ctypes.c_int64), ("used_tokens", ctypes.c_int64),
                ("logical_tokens", ctypes.c_int64), ("num_sequences", ctypes.c_int64)]


_lib.pa_bm_create.restype = _P
_lib.pa_bm_create.argtypes = [_I32, _I32]
_lib.pa_bm_destroy.restype = None
_lib.pa_bm_destroy.argtypes = [_P]
_lib.pa_bm_allocate.restype = ctypes.c_int
_lib.pa_bm_allocate.argtypes = [_P, _I64, _I32, _P]
_lib.pa_bm_share_prefix.restype = ctypes.c_int
_lib.pa_bm_share_prefix.argtypes = [_P, _I64, _I64, _I32, _P, ctypes.POINTER(_I32)]
_lib.pa_bm_append.restype = ctypes.c_int
_lib.pa_bm_append.argtypes = [_P, _I64, ctypes.POINTER(_I64), ctypes.POINTER(_I64), ctypes.POINTER(_I64)]
_lib.pa_bm_append_batch.restype = ctypes.c_int
_lib.pa_bm_append_batch.argtypes = [_P, _P, _I32, _P, _P, ctypes.POINTER(_I32), ctypes.POINTER(_I32)]
_lib.pa_bm_free.restype = ctypes.c_int
_lib.pa_bm_free.argtypes = [_P, _I64]
_lib.pa_bm_block_tables.restype = ctypes.c_int
_lib.pa_bm_block_tables.argtypes = [_P, _P, _I32, _P, _I32, _P]
_lib.pa_bm_context_len.restype = _I32
_lib.pa_bm_context_len.argtypes = [_P, _I64]
_lib.pa_bm_ref_count.restype = _I32
_lib.pa_bm_ref_count.argtypes = [_P, _I32]
_lib.pa_bm_free_list.restype = _I32
_lib.pa_bm_free_list.argtypes = [_P, _P, _I32]
_lib.pa_bm_sequences.restype = _I32
_lib.pa_bm_sequences.argtypes = [_P, _P, _I32]
_lib.pa_bm_table.restype = _I32
_lib.pa_bm_table.argtypes = [_P, _I64, _P, _I32]
_lib.pa_bm_stats.restype = None
_lib.pa_bm_stats.argtypes = [_P, ctypes.POINTER(_Stats)]


class _PrefixStats(ctypes.Structure):
    _fields_ = [("queried_blocks", ctypes.c_int64), ("hit_blocks", ctypes.c_int64),
                ("cached_blocks", ctypes.c_int64), ("evictable_blocks", ctypes.c_int64),
                ("evictions", ctypes.c_int64)]


_lib.pa_bm_create_prefix_caching.restype = _P
_lib.pa_bm_create_prefix_caching.argtypes = [_I32, _I32]
_lib.pa_bm_allocate_prompt.restype = ctypes.c_int
_lib.pa_bm_allocate_prompt.argtypes = [_P, _I64, _P, _I32, _P, ctypes.POINTER(_I32)]
_lib.pa_bm_evictable.restype = _I32
_lib.pa_bm_evictable.argtypes = [_P, _P, _I32]
_lib.pa_bm_cache_entry.restype = _I32
_lib.pa_bm_cache_entry.argtypes = [_P, _I32, ctypes.POINTER(_I64), ctypes.POINTER(_I64)]
_lib.pa_bm_prefix_stats.restype = None
_lib.pa_bm_prefix_stats.argtypes = [_P, ctypes.POINTER(_PrefixStats)]

EXPORTED = ["pa_bm_create", "pa_bm_destroy", "pa_bm_allocate", "pa_bm_share_prefix", "pa_bm_append",
            "pa_bm_append_batch", "pa_bm_free", "pa_bm_block_tables", "pa_bm_context_len", "pa_bm_ref_count",
            "pa_bm_free_list", "pa_bm_sequences", "pa_bm_table", "pa_bm_stats", "pa_bm_create_prefix_caching",
            "pa_bm_allocate_prompt", "pa_bm_evictable", "pa_bm_cache_entry", "pa_bm_prefix_stats"]

_STATUS = {0: "ok", 1: "no space", 2: "bad argument", 3: "unknown sequence", 4: "sequence exists",
           5: "table longer than max_blocks_per_seq"}


class NoSpace(Exception):
    """The pool has no free block for the request (nothing was changed)."""


class BlockManagerError(RuntimeError):
    pass


def _check(rc: int, what: str) -> None:
    if rc == 1:
        raise NoSpace(what)
    if rc != 0:
        raise BlockManagerError(f"{what}: {_STATUS.get(rc, rc)}")


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


class BlockManager:
    """A pool of ``num_blocks`` KV blocks of ``block_size`` tokens (with prefix
    caching of full prompt blocks when ``prefix_caching``)."""

    NoSpace = NoSpace

    def __init__(self, num_blocks: int, block_size: int = 16, prefix_caching: bool = False):
        create = _lib.pa_bm_create_prefix_caching if prefix_caching else _lib.pa_bm_create
        self._h = create(num_blocks, block_size)
        if not self._h:
            raise BlockManagerError("pa_bm_create failed")
        self.num_blocks = num_blocks
        self.block_size = block_size

    def __del__(self):
        h = getattr(self, "_h", None)
        if h:
            _lib.pa_bm_destroy(h)
            self._h = None

    # -- operations ---------------------------------------------------------------
    def allocate(self, seq: int, num_tokens: int) -> List[int]:
        slots = np.empty(max(num_tokens, 1), dtype=np.int64)
        _check(_lib.pa_bm_allocate(self._h, seq, num_tokens, _ptr(slots)), f"allocate({seq})")
        return slots[:num_tokens].tolist()

    def allocate_prompt(self, seq: int, tokens: Sequence[int]) -> Tuple[List[int], int]:
        """(slots of all prompt tokens, number of leading tokens already cached)."""
        t = np.ascontiguousarray(tokens, dtype=np.int32)
        n = len(t)
        slots = np.empty(max(n, 1), dtype=np.int64)
        cached = _I32(0)
        _check(_lib.pa_bm_allocate_prompt(self._h, seq, _ptr(t) if n else None, n, _ptr(slots), ctypes.byref(cached)),
               f"allocate_prompt({seq})")
        return slots[:n].tolist(), cached.value

    def share_prefix(self, seq: int, src: int, num_tokens: int) -> List[int]:
        slots = np.empty(max(num_tokens, 1), dtype=np.int64)
        n = _I32(0)
        _check(_lib.pa_bm_share_prefix(self._h, seq, src, num_tokens, _ptr(slots), ctypes.byref(n)),
               f"share_prefix({seq}, {src})")
        return slots[:n.value].tolist()

    def append(self, seq: int) -> Tuple[int, Optional[Tuple[int, int]]]:
        slot, src, dst = _I64(0), _I64(0), _I64(0)
        _check(_lib.pa_bm_append(self._h, seq, ctypes.byref(slot), ctypes.byref(src), ctypes.byref(dst)),
               f"append({seq})")
        return slot.value, ((src.value, dst.value) if src.value >= 0 else None)

    def append_batch(self, seqs: Sequence[int]):
        """One decode step: (slots [n] int64, copy pairs [P, 2] int64, number done)."""
        s = np.ascontiguousarray(seqs, dtype=np.int64)
        n = len(s)
        slots = np.empty(max(n, 1), dtype=np.int64)
        pairs = np.empty((max(n, 1), 2), dtype=np.int64)
        npairs, done = _I32(0), _I32(0)
        rc = _lib.pa_bm_append_batch(self._h, _ptr(s), n, _ptr(slots), _ptr(pairs), ctypes.byref(npairs),
                                     ctypes.byref(done))
        if rc not in (0, 1):
            _check(rc, "append_batch")
        return slots[:done.value], pairs[:npairs.value], done.value

    def free(self, seq: int) -> None:
        _check(_lib.pa_bm_free(self._h, seq), f"free({seq})")

    def tables(self, seqs: Sequence[int], max_blocks_per_seq: int):
        """(block_tables [n, max_blocks_per_seq] int32 (-1 padded), context_lens [n] int32)."""
        s = np.ascontiguousarray(seqs, dtype=np.int64)
        n = len(s)
        t = np.empty((max(n, 1), max(max_blocks_per_seq, 1)), dtype=np.int32)
        lens = np.empty(max(n, 1), dtype=np.int32)
        _check(_lib.pa_bm_block_tables(self._h, _ptr(s), n, _ptr(t), max_blocks_per_seq, _ptr(lens)),
               "block_tables")
        return t[:n, :max_blocks_per_seq], lens[:n]

    def stats(self) -> Dict[str, float]:
        st = _Stats()
        _lib.pa_bm_stats(self._h, ctypes.byref(st))
        cap = self.num_blocks * self.block_size
        return {
            "total_blocks": st.total_blocks, "free_blocks": st.free_blocks, "used_blocks": st.used_blocks,
            "used_tokens": st.used_tokens, "logical_tokens": st.logical_tokens,
            "pool_utilization": st.used_tokens / cap if cap else 0.0,
            "allocated_utilization": st.used_tokens / (st.used_blocks * self.block_size) if st.used_blocks else 0.0,
            "num_sequences": st.num_sequences,
        }

    # -- inspection (the oracle's attribute names) ------------------------------------
    @property
    def free_blocks(self) -> List[int]:
        n = _lib.pa_bm_free_list(self._h, None, 0)
        out = np.empty(max(n, 1), dtype=np.int32)
        _lib.pa_bm_free_list(self._h, _ptr(out), n)
        return out[:n].tolist()

    def sequences(self) -> List[int]:
        n = _lib.pa_bm_sequences(self._h, None, 0)
        out = np.empty(max(n, 1), dtype=np.int64)
        _lib.pa_bm_sequences(self._h, _ptr(out), n)
        return out[:n].tolist()

    def table(self, seq: int) -> List[int]:
        n = _lib.pa_bm_table(self._h, seq, None, 0)
        if n < 0:
            raise KeyError(seq)
        out = np.empty(max(n, 1), dtype=np.int32)
        _lib.pa_bm_table(self._h, seq, _ptr(out), n)
        return out[:n].tolist()

    @property
    def block_tables(self) -> Dict[int, List[int]]:
        return {s: self.table(s) for s in self.sequences()}

    @property
    def context_lens(self) -> Dict[int, int]:
        return {s: int(_lib.pa_bm_context_len(self._h, s)) for s in self.sequences()}

    @property
    def ref_count(self) -> List[int]:
        return [int(_lib.pa_bm_ref_count(self._h, b)) for b in range(self.num_blocks)]

    @property
    def evictable(self) -> List[int]:
        n = _lib.pa_bm_evictable(self._h, None, 0)
        out = np.empty(max(n, 1), dtype=np.int32)
        _lib.pa_bm_evictable(self._h, _ptr(out), n)
        return out[:n].tolist()

    def cache_items(self):
        """(parent entry, None, block) of every cached block (token ids stay in the manager)."""
        items = []
        e, pe = _I64(0), _I64(0)
        for b in range(self.num_blocks):
            if _lib.pa_bm_cache_entry(self._h, b, ctypes.byref(e), ctypes.byref(pe)) == 1:
                items.append((pe.value, None, b))
        return items

    def cache_entries(self) -> List[int]:
        e, pe = _I64(0), _I64(0)
        return [e.value for b in range(self.num_blocks)
                if _lib.pa_bm_cache_entry(self._h, b, ctypes.byref(e), ctypes.byref(pe)) == 1]

    def prefix_stats(self) -> Dict[str, int]:
        st = _PrefixStats()
        _lib.pa_bm_prefix_stats(self._h, ctypes.byref(st))
        return {"queried_blocks": st.queried_blocks, "hit_blocks": st.hit_blocks, "cached_blocks": st.cached_blocks,
                "evictable_blocks": st.evictable_blocks, "evictions": st.evictions}
