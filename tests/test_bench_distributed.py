"""The N>1 host path of bench.py on CPU: two gloo ranks, no GPU.

Each rank builds its own batch (same shape, seed offset by rank), the step
time is the maximum over ranks and the bytes/sequences are summed -- the
only collectives; there is no data-path exchange."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world), RANK=str(rank),
                      LOCAL_RANK=str(rank))
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import bench
    from paged_kv_cache_464_b200 import inputs
    w, r, _ = bench.dist_setup()
    try:
        cfg = inputs.CONFIGS["llama3_8b_gqa"]
        case = inputs.make_case(cfg, seed=bench.rank_seed(cfg, r), lens=None, num_seqs=8, with_post=False)
        t = 10.0 + r                       # pretend per-rank elapsed ms
        tmax = bench.all_reduce_max(t, w, "cpu")
        total = bench.all_reduce_sum(float(case.kv_bytes()), w, "cpu")
        bench.barrier(w)
        results[r] = (w, tmax, total, case.kv_bytes(), tuple(case.context_lens.tolist()), tuple(case.q.shape))
    finally:
        import torch.distributed as dist
        dist.destroy_process_group()


@pytest.mark.slow
def test_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    results = manager.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, results)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    r0, r1 = results[0], results[1]
    assert r0[0] == r1[0] == 2
    assert r0[1] == r1[1] == 11.0                  # max over ranks
    assert r0[2] == r1[2] == r0[3] + r1[3]         # bytes summed over ranks
    assert r0[5] == r1[5]                          # same shape per rank
    assert r0[4] != r1[4]                          # different batches (weak scaling)
