"""Seeded synthetic inputs for paged decode attention.

This module is shared by the CUDA path's tests and benchmark and by the CPU
oracle's tests.  It draws random numbers and places them in the cache layout;
it computes no attention, no softmax and no cache copy.  Every value comes from
numpy's PCG64 generator seeded per workload, is drawn in float32 and is rounded
once to the storage dtype, so both sides see identical stored bytes.

Cache layout (the boundary's): ``k_cache`` and ``v_cache`` are separate
``[num_blocks, block_size, num_kv_heads, head_dim]`` arrays, token-major inside a
block, as in the per-block ``(2, block_size, n_heads, head_dim)`` tensor of
``PagedAttention.forward`` ("vLLM推理引擎深度解析", §五 优化的注意力计算) with
the K/V axis split into two tensors.  A block table row maps a sequence's
logical block ``j`` (tokens ``j*bs .. j*bs+bs-1``) to one physical block
("vLLM 原理与源码阅读", Block 管理器, item 1).

Workloads (sizes, distributions):

* ``tiny``            fp32, 4 seqs, lens {17,33,50,100}, 4/4 heads, D=64, pool 64.
* ``llama2_7b``       fp16, 64 seqs, lens U[64,2048], 32/32 heads, D=128.
* ``llama3_8b_gqa``   bf16, 256 seqs, lens round(exp(N(ln 1024, 0.6^2))) clipped
                      to [128,4096], 32/8 heads, D=128.
* ``shared_prefix``   bf16, 128 seqs, 1024-token prefix in 64 shared blocks plus
                      private suffix U[16,512]; 32/8 heads, D=128; 25% of the
                      sequences copy-on-write the last prefix block.
* ``long_context``    bf16, 8 seqs, len 32768, 64/8 heads, D=128, partition 512.
* ``llama3_8b_gqa_fp8``  the GQA workload with an FP8 (E4M3) KV cache: the case
                      carries bf16 rows; a quantising slot write stores them as
                      1-byte codes with scale 0.0125 (k and v).

``context_lens`` are the lengths the decode call attends to.  The step's new
token sits at position ``context_len - 1``: the pre-step cache holds poison at
that slot and ``key``/``value`` carry the row that ``reshape_and_cache`` must
write there.  Slots that hold no token (unused pool blocks, the tail of a
sequence's last block) hold poison (NaN) so that a kernel that reads them
produces NaN.  Unused block-table entries are -1.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional

import numpy as np
import torch

DTYPES = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}
DTYPE_CODE = {"f32": 0, "f16": 1, "bf16": 2}
ELEM_BYTES = {"f32": 4, "f16": 2, "bf16": 2}


@dataclasses.dataclass(frozen=True)
class DecodeConfig:
    name: str
    index: int               # 1-based position in the workload list; seed = 1000 + index
    num_seqs: int
    num_heads: int
    num_kv_heads: int
    head_dim: int
    dtype: str
    block_size: int = 16
    partition_size: int = 0  # 0 = library's automatic choice
    description: str = ""
    kv_dtype: str = ""       # "" = dtype; "fp8_e4m3": caches hold 1-byte codes written from the dtype rows
    kv_scale: float = 1.0    # k_scale = v_scale for 1-byte caches

    @property
    def seed(self) -> int:
        return 1000 + self.index

    @property
    def group(self) -> int:
        return self.num_heads // self.num_kv_heads


CONFIGS: Dict[str, DecodeConfig] = {
    c.name: c for c in [
        DecodeConfig("tiny", 1, 4, 4, 4, 64, "f32",
                     description="tiny paged decode fp32, lens {17,33,50,100}, 4/4 heads, D=64, pool 64"),
        DecodeConfig("llama2_7b", 2, 64, 32, 32, 128, "f16",
                     description="Llama-2-7B-shaped decode fp16, 64 seqs, lens U[64,2048], 32/32 heads, D=128"),
        DecodeConfig("llama3_8b_gqa", 3, 256, 32, 8, 128, "bf16",
                     description="Llama-3-8B-shaped GQA decode bf16, 256 seqs, log-normal lens "
                                 "(median 1024, sigma 0.6, clip [128,4096]), 32/8 heads, D=128"),
        DecodeConfig("shared_prefix", 4, 128, 32, 8, 128, "bf16",
                     description="shared-prefix decode bf16, 128 seqs, 1024-token shared prefix + "
                                 "U[16,512] suffix, 32/8 heads, D=128, CoW of 32 seqs/step"),
        DecodeConfig("long_context", 5, 8, 64, 8, 128, "bf16", partition_size=512,
                     description="long-context split-K decode bf16, 8 seqs x 32768, 64/8 heads, "
                                 "D=128, partition 512"),
        DecodeConfig("llama3_8b_gqa_fp8", 6, 256, 32, 8, 128, "bf16", kv_dtype="fp8_e4m3", kv_scale=0.0125,
                     description="the Llama-3-8B-shaped GQA workload with an FP8 (E4M3) KV cache: bf16 q/out, "
                                 "K/V stored as 1-byte codes with scale 0.0125"),
    ]
}


# the workloads whose caches hold the storage dtype itself (the five of the target list)
BASE_WORKLOADS = [n for n, c in CONFIGS.items() if not c.kv_dtype]


def _round(x: np.ndarray, dtype: str) -> torch.Tensor:
    """float32 numpy -> torch tensor of the storage dtype (round to nearest even)."""
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(DTYPES[dtype])


def _draw_lens(cfg: DecodeConfig, rng: np.random.Generator) -> np.ndarray:
    S = cfg.num_seqs
    if cfg.name == "tiny":
        return np.array([17, 33, 50, 100], dtype=np.int64)
    if cfg.name == "llama2_7b":
        return rng.integers(64, 2048, size=S, endpoint=True).astype(np.int64)
    if cfg.name in ("llama3_8b_gqa", "llama3_8b_gqa_fp8"):
        x = np.exp(rng.normal(math.log(1024.0), 0.6, size=S))
        return np.clip(np.rint(x), 128, 4096).astype(np.int64)
    if cfg.name == "shared_prefix":
        return 1024 + rng.integers(16, 512, size=S, endpoint=True).astype(np.int64)
    if cfg.name == "long_context":
        return np.full(S, 32768, dtype=np.int64)
    raise KeyError(cfg.name)


@dataclasses.dataclass
class DecodeCase:
    """One workload instance.  All tensors are CPU tensors.

    q            [S, Hq, D]            storage dtype
    k_cache      [NB, bs, Hkv, D]      storage dtype, pre-step (new-token slots poisoned,
                                       copy-on-write destinations poisoned)
    v_cache      same
    k_cache_post / v_cache_post        the cache after the step's copies and writes
                                       (only when ``with_post`` was requested)
    key, value   [S, Hkv, D]           the step's new token rows
    slot_mapping [S] int64             where each new row goes (slot = block * bs + offset)
    block_mapping [P, 2] int64         copy-on-write (src, dst) pairs (may be empty)
    block_tables [S, MBS] int32        -1 past each sequence's last block
    context_lens [S] int32
    k_logical / v_logical              per-sequence [L_b, Hkv, D] float32 views of the
                                       stored values (only when ``keep_logical``)
    """
    cfg: DecodeConfig
    q: torch.Tensor
    k_cache: torch.Tensor
    v_cache: torch.Tensor
    key: torch.Tensor
    value: torch.Tensor
    slot_mapping: torch.Tensor
    block_mapping: torch.Tensor
    block_tables: torch.Tensor
    context_lens: torch.Tensor
    scale: float
    shared_block_tables: Optional[torch.Tensor] = None
    k_cache_post: Optional[torch.Tensor] = None
    v_cache_post: Optional[torch.Tensor] = None
    k_logical: Optional[List[np.ndarray]] = None
    v_logical: Optional[List[np.ndarray]] = None

    @property
    def num_blocks(self) -> int:
        return int(self.k_cache.shape[0])

    @property
    def max_context_len(self) -> int:
        return int(self.context_lens.max().item()) if self.context_lens.numel() else 0

    def kv_bytes(self) -> int:
        """Algorithmic KV bytes one decode call reads: sum_b L_b * Hkv * 2 * D * es."""
        c = self.cfg
        es = 1 if c.kv_dtype == "fp8_e4m3" else ELEM_BYTES[c.dtype]
        return int(self.context_lens.to(torch.int64).sum().item()) * c.num_kv_heads * 2 * c.head_dim * es


def make_case(name_or_cfg, *, seed: Optional[int] = None, num_seqs: Optional[int] = None,
              lens: Optional[List[int]] = None, pool_factor: float = 1.25,
              keep_logical: bool = False, with_post: bool = True) -> DecodeCase:
    """Build one seeded workload.

    ``num_seqs`` and ``lens`` override the workload's batch size and lengths (small
    parity cases with the same shapes); ``seed`` overrides 1000 + index.
    """
    cfg = CONFIGS[name_or_cfg] if isinstance(name_or_cfg, str) else name_or_cfg
    if num_seqs is not None or lens is not None:
        cfg = dataclasses.replace(cfg, num_seqs=len(lens) if lens is not None else num_seqs)
    rng = np.random.Generator(np.random.PCG64(cfg.seed if seed is None else seed))
    S, Hq, Hkv, D, bs = cfg.num_seqs, cfg.num_heads, cfg.num_kv_heads, cfg.head_dim, cfg.block_size
    base = CONFIGS.get(cfg.name, cfg)

    # 1. context lengths
    if lens is not None:
        L = np.asarray(lens, dtype=np.int64)
    else:
        L = _draw_lens(dataclasses.replace(base, num_seqs=S), rng)[:S]
        if len(L) < S:  # tiny workload with more sequences than its fixed list
            L = np.resize(L, S)
    nblk = (L + bs - 1) // bs

    shared = cfg.name == "shared_prefix"
    prefix_blocks = 1024 // bs if shared else 0
    if shared:
        assert (L > 1024).all(), "shared-prefix lengths must exceed the prefix"

    # 2. pool size and the shuffled physical ids
    if cfg.name == "tiny" and lens is None and pool_factor == 1.25:
        need = int(nblk.sum())
        NB = 64
    else:
        need = int(nblk.sum()) - (prefix_blocks * (S - 1) if shared else 0)
        NB = max(1, int(math.ceil(pool_factor * need)))
    n_cow = (S + 3) // 4 if shared else 0
    NB += n_cow
    perm = rng.permutation(NB).astype(np.int64)

    MBS = int(nblk.max()) if S else 1
    MBS = max(MBS, 1)
    tables = np.full((S, MBS), -1, dtype=np.int64)
    cursor = 0
    if shared:
        prefix_ids = perm[cursor:cursor + prefix_blocks]
        cursor += prefix_blocks
    for b in range(S):
        start = 0
        if shared:
            tables[b, :prefix_blocks] = prefix_ids
            start = prefix_blocks
        k = int(nblk[b]) - start
        tables[b, start:start + k] = perm[cursor:cursor + k]
        cursor += k
    shared_tables = tables.copy()
    cow_pairs = np.zeros((0, 2), dtype=np.int64)
    if shared:
        cow_seqs = np.sort(rng.choice(S, size=n_cow, replace=False))
        dst = perm[cursor:cursor + n_cow]
        cursor += n_cow
        src = np.full(n_cow, tables[0, prefix_blocks - 1], dtype=np.int64)
        tables[cow_seqs, prefix_blocks - 1] = dst
        cow_pairs = np.stack([src, dst], axis=1)
    assert cursor <= NB

    # 3. queries
    q = _round(rng.standard_normal((S, Hq, D), dtype=np.float32), cfg.dtype)

    # 4. logical K/V, drawn per sequence (the shared prefix once), then placed in the pool
    pool_k = np.full((NB * bs, Hkv, D), np.nan, dtype=np.float32)
    pool_v = np.full((NB * bs, Hkv, D), np.nan, dtype=np.float32)
    if shared:
        pk = rng.standard_normal((1024, Hkv, D), dtype=np.float32)
        pv = rng.standard_normal((1024, Hkv, D), dtype=np.float32)
        slots = (prefix_ids[:, None] * bs + np.arange(bs)[None, :]).reshape(-1)
        pool_k[slots] = pk
        pool_v[slots] = pv
    klog_f32, vlog_f32 = [], []
    for b in range(S):
        t0 = 1024 if shared else 0
        n = int(L[b]) - t0
        kb = rng.standard_normal((n, Hkv, D), dtype=np.float32)
        vb = rng.standard_normal((n, Hkv, D), dtype=np.float32)
        pos = np.arange(t0, int(L[b]))
        slots = shared_tables[b, pos // bs] * bs + pos % bs
        pool_k[slots] = kb
        pool_v[slots] = vb
        if keep_logical:
            klog_f32.append(kb)
            vlog_f32.append(vb)

    k_post = _round(pool_k.reshape(NB, bs, Hkv, D), cfg.dtype)
    v_post = _round(pool_v.reshape(NB, bs, Hkv, D), cfg.dtype)
    del pool_k, pool_v
    if shared and n_cow:
        # the copy-on-write destinations hold what the shared block holds
        k_post[cow_pairs[:, 1]] = k_post[cow_pairs[:, 0]]
        v_post[cow_pairs[:, 1]] = v_post[cow_pairs[:, 0]]

    # 5. the step's new token: position L_b - 1 of each sequence
    new_pos = L - 1
    slot_mapping = tables[np.arange(S), new_pos // bs] * bs + new_pos % bs if S else np.zeros(0, np.int64)
    kflat = k_post.view(NB * bs, Hkv, D)
    vflat = v_post.view(NB * bs, Hkv, D)
    sm_t = torch.from_numpy(slot_mapping.astype(np.int64))
    key = kflat[sm_t].clone()
    value = vflat[sm_t].clone()

    # 6. pre-step cache: new-token slots and copy destinations poisoned
    k_pre = k_post.clone()
    v_pre = v_post.clone()
    k_pre.view(NB * bs, Hkv, D)[sm_t] = float("nan")
    v_pre.view(NB * bs, Hkv, D)[sm_t] = float("nan")
    if n_cow:
        d = torch.from_numpy(cow_pairs[:, 1])
        k_pre[d] = float("nan")
        v_pre[d] = float("nan")

    k_logical = v_logical = None
    if keep_logical:
        k_logical, v_logical = [], []
        for b in range(S):
            pos = np.arange(int(L[b]))
            slots = torch.from_numpy(shared_tables[b, pos // bs] * bs + pos % bs)
            k_logical.append(kflat[slots].to(torch.float64).numpy())
            v_logical.append(vflat[slots].to(torch.float64).numpy())

    case = DecodeCase(
        cfg=cfg, q=q, k_cache=k_pre, v_cache=v_pre, key=key, value=value,
        slot_mapping=sm_t, block_mapping=torch.from_numpy(cow_pairs.astype(np.int64)),
        block_tables=torch.from_numpy(tables.astype(np.int32)),
        context_lens=torch.from_numpy(L.astype(np.int32)),
        scale=float(np.float32(1.0 / math.sqrt(D))),
        shared_block_tables=torch.from_numpy(shared_tables.astype(np.int32)) if shared else None,
        k_cache_post=k_post if with_post else None, v_cache_post=v_post if with_post else None,
        k_logical=k_logical, v_logical=v_logical)
    return case


def permute_blocks(case: DecodeCase, seed: int) -> DecodeCase:
    """The same logical case with its physical blocks moved to new ids.

    Block ``i`` moves to ``sigma[i]`` (data moved, tables, slots and copy pairs
    rewritten).  Used to check that outputs do not depend on physical placement.
    """
    rng = np.random.Generator(np.random.PCG64(seed))
    NB = case.num_blocks
    sigma = torch.from_numpy(rng.permutation(NB).astype(np.int64))

    def move(c):
        if c is None:
            return None
        out = torch.empty_like(c)
        out[sigma] = c
        return out

    def retab(t):
        if t is None:
            return None
        t64 = t.to(torch.int64)
        r = torch.where(t64 >= 0, sigma[t64.clamp(min=0)], t64)
        return r.to(t.dtype)

    bs = case.cfg.block_size
    sm = case.slot_mapping
    new_sm = torch.where(sm >= 0, sigma[(sm // bs).clamp(min=0)] * bs + sm % bs, sm)
    bm = case.block_mapping
    new_bm = sigma[bm] if bm.numel() else bm.clone()
    return dataclasses.replace(
        case, k_cache=move(case.k_cache), v_cache=move(case.v_cache),
        k_cache_post=move(case.k_cache_post), v_cache_post=move(case.v_cache_post),
        block_tables=retab(case.block_tables), shared_block_tables=retab(case.shared_block_tables),
        slot_mapping=new_sm, block_mapping=new_bm)


# ---------------------------------------------------------------------------- prefill
@dataclasses.dataclass
class PrefillCase:
    """A chunk of new tokens per sequence over a paged cache (all tokens already cached).

    q                [T, Hq, D]   the chunk tokens' queries, sequence after sequence
    query_start_loc  [S + 1] int32   sequence b's queries are rows qsl[b]:qsl[b+1];
                                     they are the last n_b tokens of its context
    k_cache, v_cache [NB, bs, Hkv, D]  every context token present
    """
    cfg: DecodeConfig
    q: torch.Tensor
    k_cache: torch.Tensor
    v_cache: torch.Tensor
    block_tables: torch.Tensor
    context_lens: torch.Tensor
    query_start_loc: torch.Tensor
    scale: float
    k_logical: Optional[List[np.ndarray]] = None
    v_logical: Optional[List[np.ndarray]] = None

    @property
    def num_tokens(self) -> int:
        return int(self.query_start_loc[-1])

    @property
    def max_query_len(self) -> int:
        q = self.query_start_loc
        return int((q[1:] - q[:-1]).max()) if len(q) > 1 else 0

    def kv_bytes_attended(self) -> int:
        """Bytes of the K and V rows the chunks attend to (every cached token of each sequence)."""
        c = self.cfg
        return int(self.context_lens.to(torch.int64).sum()) * c.num_kv_heads * 2 * c.head_dim * \
            self.k_cache.element_size()

    def flops(self) -> int:
        """Multiply-add flops of S = QK^T and O = PV over the causally visible keys."""
        c = self.cfg
        L = self.context_lens.to(torch.int64)
        n = (self.query_start_loc[1:] - self.query_start_loc[:-1]).to(torch.int64)
        visible = (n * (L - n) + n * (n + 1) // 2).sum().item()   # sum over queries of (position + 1)
        return int(4 * visible * c.num_heads * c.head_dim)


PREFILL_CONFIGS: Dict[str, DecodeConfig] = {
    c.name: c for c in [
        DecodeConfig("llama3_8b_prefill", 7, 16, 32, 8, 128, "bf16",
                     description="Llama-3-8B-shaped chunked prefill bf16: 16 sequences, 512-token chunks "
                                 "after a cached prefix U[0,1536], 32/8 heads, D=128"),
    ]
}


def make_prefill_case(name_or_cfg, *, chunk_lens=None, prefix_lens=None, seed=None,
                      keep_logical: bool = False) -> PrefillCase:
    """Context = prefix + chunk per sequence; every context token is drawn and
    placed in the cache (through make_case); q is drawn for the chunk tokens."""
    cfg = PREFILL_CONFIGS[name_or_cfg] if isinstance(name_or_cfg, str) else name_or_cfg
    rng = np.random.Generator(np.random.PCG64(cfg.seed if seed is None else seed))
    S = cfg.num_seqs if chunk_lens is None else len(chunk_lens)
    if chunk_lens is None:
        chunk_lens = [512] * S
    if prefix_lens is None:
        prefix_lens = rng.integers(0, 1536, size=S, endpoint=True).tolist()
    L = [int(a) + int(b) for a, b in zip(prefix_lens, chunk_lens)]
    base = make_case(dataclasses.replace(cfg, num_seqs=S), lens=L, seed=int(rng.integers(1 << 31)),
                     keep_logical=keep_logical)
    T = int(sum(chunk_lens))
    q = _round(rng.standard_normal((T, cfg.num_heads, cfg.head_dim), dtype=np.float32), cfg.dtype)
    qsl = torch.zeros(S + 1, dtype=torch.int32)
    qsl[1:] = torch.cumsum(torch.tensor(chunk_lens, dtype=torch.int32), 0)
    return PrefillCase(cfg=dataclasses.replace(cfg, num_seqs=S), q=q, k_cache=base.k_cache_post,
                       v_cache=base.v_cache_post, block_tables=base.block_tables, context_lens=base.context_lens,
                       query_start_loc=qsl, scale=base.scale, k_logical=base.k_logical, v_logical=base.v_logical)


def prefill_subcase(case: PrefillCase, seqs: List[int]) -> PrefillCase:
    """The sequences `seqs` of a prefill case over the same caches (for sampled checks)."""
    qsl = case.query_start_loc
    rows = [torch.arange(int(qsl[b]), int(qsl[b + 1])) for b in seqs]
    lens = torch.tensor([int(qsl[b + 1] - qsl[b]) for b in seqs], dtype=torch.int32)
    new_qsl = torch.zeros(len(seqs) + 1, dtype=torch.int32)
    new_qsl[1:] = torch.cumsum(lens, 0)
    idx = torch.tensor(seqs, dtype=torch.long)
    return dataclasses.replace(
        case, cfg=dataclasses.replace(case.cfg, num_seqs=len(seqs)), q=case.q[torch.cat(rows)].contiguous(),
        block_tables=case.block_tables[idx].contiguous(), context_lens=case.context_lens[idx].contiguous(),
        query_start_loc=new_qsl, k_logical=None, v_logical=None)
