"""KV utilisation of the paged block manager vs static reservation (host only)."""
import pytest


@pytest.fixture(scope="module")
def kvu():
    from paged_kv_cache_464_b200 import build
    build.build()
    from paged_kv_cache_464_b200 import kv_utilization
    return kv_utilization


def test_paged_beats_static_reservation(kvu):
    r = kvu.compare(num_requests=200, pool_tokens=65536, max_seq_len=2048, seed=5)
    p, s = r["paged"], r["static"]
    assert p["blocks_left_in_use"] == 0                     # every block came back
    assert p["mean_utilization"] > 0.95                     # waste only in partial last blocks
    assert s["mean_utilization"] < 0.6                      # reservation for max_seq_len
    assert p["mean_batch"] > 1.5 * s["mean_batch"]
    assert p["steps"] < s["steps"]


def test_shared_prefix_packs_more_requests(kvu):
    plain = kvu.compare(num_requests=200, pool_tokens=65536, seed=6)
    shared = kvu.compare(num_requests=200, pool_tokens=65536, shared_prefix=512, seed=6)
    assert shared["paged"]["blocks_left_in_use"] == 512 // 16   # only the system prompt stays
    assert shared["paged"]["mean_batch"] > plain["paged"]["mean_batch"]


def test_static_closed_form(kvu):
    reqs = [(100, 10), (300, 5)]
    r = kvu.run_static(reqs, pool_tokens=4096, max_seq_len=2048)
    # both run together; step k holds (100+k) + (300+k) of 4096 reserved for 5 steps, then (100+k)/2048
    expect = [(400 + 2 * k) / 4096 for k in range(1, 6)] + [(100 + k) / 2048 for k in range(6, 11)]
    assert r["steps"] == 10 and abs(r["mean_utilization"] - sum(expect) / 10) < 1e-12
