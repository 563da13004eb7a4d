"""KV-memory utilisation of the paged block manager against a static allocator.

    python -m paged_kv_cache_464_b200.kv_utilization [--requests N] [--pool-tokens T] [--shared-prefix P]

Both serve the same seeded request stream under the same KV budget with
iteration-level batching ("vLLM推理引擎深度解析" §四 / "vLLM 原理与源码阅读"
Continuous Batching: finished requests leave and waiting ones join every
step):

* paged: the C++ block manager (libpa_b200.so).  A request joins when its
  prompt's blocks are free; every step appends one token to every running
  request (one pa_bm_append_batch); when the pool runs dry the newest request
  is preempted (its blocks freed, the request re-queued to start again).  With
  a shared system prompt, requests share its blocks (share_prefix) and write
  only their own tokens.
* static ("vLLM推理引擎深度解析" §二 TraditionalKVCacheManager): every request
  reserves max_seq_len token slots when it joins.

Reported per allocator: utilisation = tokens held / KV capacity reserved for
running requests (averaged over steps), mean and peak running batch, steps to
finish the stream, preemptions.  Host-only; no GPU is touched.
"""
from __future__ import annotations

import argparse
import collections
import json
from typing import Dict

import numpy as np


def draw_requests(num_requests: int, max_seq_len: int, seed: int, prompt=(32, 1024), output=(16, 1024)):
    rng = np.random.default_rng(seed)
    p = rng.integers(prompt[0], prompt[1], size=num_requests, endpoint=True)
    o = rng.integers(output[0], output[1], size=num_requests, endpoint=True)
    o = np.minimum(o, max_seq_len - p)
    return [(int(a), int(b)) for a, b in zip(p, o)]


def run_paged(requests, pool_tokens: int, block_size: int = 16, shared_prefix: int = 0) -> Dict[str, float]:
    from .block_manager import BlockManager
    num_blocks = pool_tokens // block_size
    m = BlockManager(num_blocks, block_size)
    PREFIX = -1
    if shared_prefix:
        m.allocate(PREFIX, shared_prefix)
    waiting = collections.deque(range(len(requests)))
    running, made = [], {}          # request ids in join order; tokens generated so far
    steps = preemptions = 0
    util_sum = batch_sum = 0.0
    peak = 0
    while waiting or running:
        # join while the prompt fits
        while waiting:
            r = waiting[0]
            plen = requests[r][0]
            try:
                if shared_prefix and plen >= shared_prefix:
                    m.share_prefix(r, PREFIX, shared_prefix)
                    for _ in range(plen - shared_prefix):
                        m.append(r)
                else:
                    m.allocate(r, plen)
            except m.NoSpace:
                if r in m.sequences():
                    m.free(r)
                break
            waiting.popleft()
            running.append(r)
            made[r] = 0
        if not running:
            raise RuntimeError("a single request does not fit the pool")
        # one decode step: one token for every running request
        todo, appended = list(running), []
        while todo:
            _, _, done = m.append_batch(todo)
            appended += todo[:done]
            if done == len(todo):
                break
            victim = running.pop()        # newest request: free and start again later
            m.free(victim)
            made.pop(victim)
            waiting.appendleft(victim)
            preemptions += 1
            todo = [r for r in todo[done:] if r != victim]
        for r in appended:
            if r in made:
                made[r] += 1
        st = m.stats()
        tokens = st["used_tokens"]
        util_sum += tokens / (st["used_blocks"] * block_size) if st["used_blocks"] else 0.0
        batch_sum += len(running)
        peak = max(peak, len(running))
        steps += 1
        for r in [r for r in running if made[r] >= requests[r][1]]:
            running.remove(r)
            m.free(r)
    return {"allocator": "paged", "steps": steps, "mean_batch": batch_sum / steps, "peak_batch": peak,
            "mean_utilization": util_sum / steps, "preemptions": preemptions,
            "blocks_left_in_use": m.stats()["used_blocks"]}


def run_static(requests, pool_tokens: int, max_seq_len: int) -> Dict[str, float]:
    slots = pool_tokens // max_seq_len
    waiting = collections.deque(range(len(requests)))
    running, made = [], {}
    steps = 0
    util_sum = batch_sum = 0.0
    peak = 0
    while waiting or running:
        while waiting and len(running) < slots:
            r = waiting.popleft()
            running.append(r)
            made[r] = 0
        for r in running:
            made[r] += 1
        held = sum(requests[r][0] + made[r] for r in running)
        util_sum += held / (len(running) * max_seq_len)
        batch_sum += len(running)
        peak = max(peak, len(running))
        steps += 1
        running = [r for r in running if made[r] < requests[r][1]]
    return {"allocator": "static", "steps": steps, "mean_batch": batch_sum / steps, "peak_batch": peak,
            "mean_utilization": util_sum / steps, "preemptions": 0}


def compare(num_requests=600, pool_tokens=131072, max_seq_len=2048, shared_prefix=0, seed=1234):
    reqs = draw_requests(num_requests, max_seq_len, seed)
    if shared_prefix:
        reqs = [(max(p, shared_prefix), o) for p, o in reqs]
    return {"requests": num_requests, "pool_tokens": pool_tokens, "max_seq_len": max_seq_len,
            "shared_prefix": shared_prefix,
            "paged": run_paged(reqs, pool_tokens, shared_prefix=shared_prefix),
            "static": run_static(reqs, pool_tokens, max_seq_len)}


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--requests", type=int, default=600)
    ap.add_argument("--pool-tokens", type=int, default=131072)
    ap.add_argument("--max-seq-len", type=int, default=2048)
    ap.add_argument("--shared-prefix", type=int, default=0)
    ap.add_argument("--seed", type=int, default=1234)
    a = ap.parse_args(argv)
    print(json.dumps(compare(a.requests, a.pool_tokens, a.max_seq_len, a.shared_prefix, a.seed)))


if __name__ == "__main__":
    main()
