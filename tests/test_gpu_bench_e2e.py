"""The bench's end-to-end loop overlaps step k's host copies with step k-1's
kernels (two buffer sets, one copy stream per direction).  Its last host
output must equal the output of the same step run plainly: a missing stream
dependency would copy out a stale or half-written buffer."""
import os
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda", 0)


@pytest.mark.parametrize("workload", ["llama3_8b_gqa", "shared_prefix", "llama3_8b_gqa_fp8"])
def test_decode_e2e_output(dev, workload):
    import bench
    from paged_kv_cache_464_b200 import inputs
    case = inputs.make_case(inputs.CONFIGS[workload], num_seqs=16, with_post=False)
    step = bench.Step(case, dev)
    r = bench.run_e2e(case, step, steps=7, warmup=3, device=dev)
    step()
    torch.cuda.synchronize()
    assert torch.equal(r["last_out_host"], step.out.cpu())
    assert r["h2d"] > 0 and r["d2h"] == step.out.numel() * step.out.element_size()


def test_prefill_e2e_output(dev):
    import bench
    from paged_kv_cache_464_b200 import inputs
    case = inputs.make_prefill_case("llama3_8b_prefill", chunk_lens=[200, 37, 512], prefix_lens=[0, 900, 64])
    step = bench.PrefillStep(case, dev)
    r = bench.run_e2e_prefill(step, steps=5, warmup=3)
    step()
    torch.cuda.synchronize()
    assert torch.equal(r["last_out_host"], step.out.cpu())
