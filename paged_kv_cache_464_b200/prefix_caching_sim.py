"""Prefill work saved by prefix caching, under continuous batching.

    python -m paged_kv_cache_464_b200.prefix_caching_sim [--requests N] [--pool-tokens T]

A seeded request stream in which most prompts start with one of a few shared
system prompts ("vLLM 原理与源码阅读", Prefix Caching: system prompts, few-shot
examples, RAG context shared by many requests) followed by the request's own
tokens, served with iteration-level batching as in kv_utilization.py: a
request joins when its prompt's blocks can be had, every step appends one token
to every running request, the newest request is preempted (freed, re-queued)
when the pool runs dry.  With prefix caching a joining request computes only
the prompt tokens after its longest cached prefix; without it, all of them.

Reported per mode: prompt tokens, prompt tokens computed, the share saved,
block hit rate, evictions, steps, mean running batch, preemptions.  Host-only.
"""
from __future__ import annotations

import argparse
import collections
import json
from typing import Callable, Dict, List, Tuple

import numpy as np


def draw_requests(num_requests: int, seed: int, system_lens=(256, 512, 1024, 1536), p_system: float = 0.9,
                  own=(16, 256), output=(16, 512), vocab: int = 32000) -> List[Tuple[List[int], int]]:
    """(prompt token ids, output tokens) per request."""
    rng = np.random.default_rng(seed)
    systems = [rng.integers(0, vocab, n).tolist() for n in system_lens]
    reqs = []
    for _ in range(num_requests):
        prefix = systems[int(rng.integers(len(systems)))] if rng.random() < p_system else []
        mine = rng.integers(0, vocab, int(rng.integers(own[0], own[1], endpoint=True))).tolist()
        reqs.append((prefix + mine, int(rng.integers(output[0], output[1], endpoint=True))))
    return reqs


def serve(requests, make_manager: Callable[[], object]) -> Dict[str, float]:
    m = make_manager()
    waiting = collections.deque(range(len(requests)))
    running, made = [], {}
    steps = preemptions = 0
    prompt_tokens = computed = 0
    batch_sum = 0.0
    while waiting or running:
        while waiting:                                   # join while the prompt fits
            r = waiting[0]
            toks = requests[r][0]
            try:
                _, cached = m.allocate_prompt(r, toks)
            except m.NoSpace:
                break
            waiting.popleft()
            running.append(r)
            made[r] = 0
            prompt_tokens += len(toks)
            computed += len(toks) - cached
        if not running:
            raise RuntimeError("a single request does not fit the pool")
        i = 0
        while i < len(running):                          # one decode step
            r = running[i]
            try:
                m.append(r)
                made[r] += 1
                i += 1
            except m.NoSpace:
                victim = running.pop()                   # newest request: free, start again later
                m.free(victim)
                made.pop(victim)
                waiting.appendleft(victim)
                preemptions += 1
        batch_sum += len(running)
        steps += 1
        for r in [r for r in running if made[r] >= requests[r][1]]:
            running.remove(r)
            m.free(r)
    st = m.prefix_stats()
    return {"prompt_tokens": prompt_tokens, "prompt_tokens_computed": computed,
            "saved": 1.0 - computed / prompt_tokens if prompt_tokens else 0.0,
            "block_hit_rate": st["hit_blocks"] / st["queried_blocks"] if st["queried_blocks"] else 0.0,
            "evictions": st["evictions"], "steps": steps, "mean_batch": batch_sum / steps,
            "preemptions": preemptions}


def compare(num_requests=400, pool_tokens=131072, block_size=16, seed=4321, managers=None):
    """Both modes on the same stream.  `managers` maps a mode to a factory
    (default: the C++ manager with and without prefix caching)."""
    if managers is None:
        from .block_manager import BlockManager
        nb = pool_tokens // block_size
        managers = {"no_caching": lambda: BlockManager(nb, block_size),
                    "prefix_caching": lambda: BlockManager(nb, block_size, prefix_caching=True)}
    reqs = draw_requests(num_requests, seed)
    return {"requests": num_requests, "pool_tokens": pool_tokens,
            **{mode: serve(reqs, make) for mode, make in managers.items()}}


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--requests", type=int, default=400)
    ap.add_argument("--pool-tokens", type=int, default=131072)
    ap.add_argument("--seed", type=int, default=4321)
    a = ap.parse_args(argv)
    print(json.dumps(compare(a.requests, a.pool_tokens, seed=a.seed)))


if __name__ == "__main__":
    main()
