"""bench.py host paths that need no GPU: the reference arm (the fp64 oracle on
the host cores) for the decode and chunked-prefill workloads, and the chunk
slot rule the prefill step writes through."""
import json
import os
import subprocess
import sys

import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from paged_kv_cache_464_b200 import inputs  # noqa: E402


def test_chunk_slots_follow_the_append_rule():
    cfg = inputs.DecodeConfig("slots", 5, 3, 8, 2, 128, "bf16")
    case = inputs.make_prefill_case(cfg, chunk_lens=[17, 1, 40], prefix_lens=[3, 0, 100])
    slots = bench.chunk_slots(case)
    assert slots.numel() == case.num_tokens
    i = 0
    for b in range(3):
        L = int(case.context_lens[b])
        n = int(case.query_start_loc[b + 1] - case.query_start_loc[b])
        for pos in range(L - n, L):
            blk = int(case.block_tables[b, pos // 16])
            assert int(slots[i]) == blk * 16 + pos % 16
            i += 1
    # the rows gathered through those slots are the chunk tokens' logical K rows
    NB, bs, Hkv, D = case.k_cache.shape
    case_l = inputs.make_prefill_case(cfg, chunk_lens=[17, 1, 40], prefix_lens=[3, 0, 100], keep_logical=True)
    k_rows = case_l.k_cache.view(NB * bs, Hkv, D)[slots]
    i = 0
    for b in range(3):
        L = int(case_l.context_lens[b])
        n = int(case_l.query_start_loc[b + 1] - case_l.query_start_loc[b])
        want = torch.from_numpy(case_l.k_logical[b][L - n:L]).to(k_rows.dtype)
        assert torch.equal(k_rows[i:i + n], want)
        i += n


def _reference_line(workload):
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", workload,
                        "--steps", "2", "--warmup", "3", "--ref-budget", "3"],
                       capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    return json.loads(r.stdout.strip().splitlines()[-1])


def test_reference_arm_prefill():
    d = _reference_line("llama3_8b_prefill")
    assert d["impl"] == "reference" and d["unit"] == "TFLOP/s" and d["metric"] == bench.PREFILL_METRIC
    assert d["value"] > 0 and d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"] == {"value": d["value"], "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert d["steps"] == 2 and d["warmup"] == 3 and d["gpu_launches"] == 0


def test_reference_arm_decode():
    d = _reference_line("tiny")
    assert d["impl"] == "reference" and d["unit"] == "GB/s" and d["metric"] == bench.METRIC
    assert d["value"] > 0 and d["config"]["workload"] == "tiny"


def test_cpu_baseline_reports_all_threads_and_one():
    case = inputs.make_case("tiny")
    d = bench.cpu_baseline(case, budget_s=2.0)
    assert d["kind"] == "oracle" and d["unit"] == "GB/s" and d["value"] > 0 and d["cores"] >= 1
    assert isinstance(d["cpu"], str) and d["cpu"]
    one = d["single_thread"]
    assert one["unit"] == "GB/s" and one["value"] > 0 and one["seqs_per_s"] > 0
    import oracle
    assert oracle.get().num_threads == d["cores"]   # thread count restored
