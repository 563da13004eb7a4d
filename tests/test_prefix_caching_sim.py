"""The prefix-caching simulation: the C++ manager and the oracle give the same
numbers on the same stream; caching saves prefill work only when prompts share
full leading blocks ("vLLM 原理与源码阅读", Prefix Caching)."""
from oracle.prefix_cache import PrefixCachingBlockManager
from paged_kv_cache_464_b200 import prefix_caching_sim as sim
from paged_kv_cache_464_b200.block_manager import BlockManager


def test_native_equals_oracle():
    nb = 4096 // 16
    res = sim.compare(num_requests=60, pool_tokens=4096 * 4, seed=7, managers={
        "native": lambda: BlockManager(nb * 4, 16, prefix_caching=True),
        "oracle": lambda: PrefixCachingBlockManager(nb * 4, 16)})
    assert res["native"] == res["oracle"]
    assert res["native"]["saved"] > 0.3 and res["native"]["evictions"] > 0


def test_no_shared_prompts_saves_nothing():
    reqs = sim.draw_requests(40, seed=9, p_system=0.0)
    r = sim.serve(reqs, lambda: BlockManager(2048, 16, prefix_caching=True))
    assert r["saved"] == 0.0 and r["block_hit_rate"] == 0.0


def test_caching_saves_work_and_memory():
    res = sim.compare(num_requests=120, pool_tokens=32768, seed=11)
    a, b = res["no_caching"], res["prefix_caching"]
    assert a["saved"] == 0.0 and b["saved"] > 0.5
    assert b["mean_batch"] > a["mean_batch"] and b["steps"] < a["steps"]
