"""The library's calls inside a captured CUDA graph, as a serving loop runs them.

Every entry point takes its device buffers (split-K workspace included) from
the caller, allocates nothing and never synchronises, so a whole step can be
captured once and replayed.  Checked here: a decode step with the new-token
write and a split-K partition plus reduce (programmatic-launch edges inside
the graph), and a chunked-prefill call, each captured and replayed; every
replay must give the same bits as the eager call on the same inputs, the
caches included, and record no device error.
"""
import pytest
import torch

from paged_kv_cache_464_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from paged_kv_cache_464_b200 import capi
    capi.get_device_error(clear=True)
    return capi


def _capture(fn):
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()                      # warm-up outside the capture (attributes, tensor-map encoder)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    return g


def test_decode_step_replayed_from_a_graph(pa):
    case = inputs.make_case("long_context", lens=[2048, 700, 1500])   # split sequences: partition + reduce
    c = case.cfg
    d = "cuda"
    q, key, val = case.q.to(d), case.key.to(d), case.value.to(d)
    bt, cl = case.block_tables.to(d), case.context_lens.to(d)
    P = 512
    need = pa.decode_workspace_bytes(c.num_seqs, c.num_heads, c.num_kv_heads, c.head_dim, case.max_context_len, P)
    assert need > 0
    ws = torch.empty(need, dtype=torch.uint8, device=d)

    k1, v1 = case.k_cache.to(d), case.v_cache.to(d)
    out_eager = torch.empty_like(q)
    pa.decode_append(q, key, val, k1, v1, bt, cl, case.scale, out_eager, max_context_len=case.max_context_len,
                     partition_size=P, workspace=ws)
    torch.cuda.synchronize()

    k2, v2 = case.k_cache.to(d), case.v_cache.to(d)
    out_g = torch.empty_like(q)
    g = _capture(lambda: pa.decode_append(q, key, val, k2, v2, bt, cl, case.scale, out_g,
                                          max_context_len=case.max_context_len, partition_size=P, workspace=ws))
    for _ in range(5):
        out_g.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(out_g, out_eager)
        # the new token's slot write (idempotent); bits compared, the pool holds NaN in unused slots
        assert torch.equal(k2.view(torch.int16), k1.view(torch.int16))
        assert torch.equal(v2.view(torch.int16), v1.view(torch.int16))
    code, detail = pa.get_device_error(clear=True)
    assert code == 0, (code, detail)


def test_prefill_replayed_from_a_graph(pa):
    cfg = inputs.DecodeConfig("graph_prefill", 91, 3, 32, 8, 128, "bf16")
    pc = inputs.make_prefill_case(cfg, chunk_lens=[70, 200, 5], prefix_lens=[40, 300, 0])
    d = "cuda"
    args = [pc.q.to(d), pc.k_cache.to(d), pc.v_cache.to(d), pc.block_tables.to(d), pc.context_lens.to(d),
            pc.query_start_loc.to(d), pc.scale]
    out_eager = pa.prefill(*args, max_query_len=pc.max_query_len)
    torch.cuda.synchronize()
    out_g = torch.empty_like(out_eager)
    g = _capture(lambda: pa.prefill(*args, out_g, max_query_len=pc.max_query_len))
    for _ in range(3):
        out_g.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(out_g, out_eager)
    code, detail = pa.get_device_error(clear=True)
    assert code == 0, (code, detail)
