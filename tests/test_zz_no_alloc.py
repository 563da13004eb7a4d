"""pa_decode_static_workspace: decode for callers that cannot allocate device
memory (a plugin inside a process whose allocator owns all device memory, or
a loop that must not call cudaMalloc/cudaFree because they can synchronise the
device).  Its split-K scratch is the library's own fixed device array.

The GPU test calls it through the C ABI twice in a row (two different
workloads, both split into partitions so the scratch is used) and checks each
output against pa_decode with a caller-allocated workspace: both run the same
kernels on the same inputs, so the outputs must be bit-identical (and both are
within the decode tolerance of the fp64 oracle, which the parity tests check).
It needs nothing from other test files, so it passes alone in a fresh process
as well as after the rest of the suite.
"""
import numpy as np
import pytest
import torch

from paged_kv_cache_464_b200 import inputs

PA_ERR_WORKSPACE = 4


def _close(a: torch.Tensor, b: torch.Tensor, dtype: str):
    x = a.to(torch.float64).cpu().numpy()
    y = b.to(torch.float64).cpu().numpy()
    assert np.isfinite(x).all()
    err = np.abs(x - y)
    if dtype == "f32":
        assert err.max() <= 1e-5
    else:
        assert (err <= 2e-3 + 1e-2 * np.abs(y)).all(), err.max()


def test_oversized_request_is_rejected_before_any_launch():
    from paged_kv_cache_464_b200 import capi
    need = capi.decode_workspace_bytes(4096, 64, 8, 128, 32768, 16)
    assert need > capi.STATIC_WORKSPACE_BYTES
    # every argument valid for pa_decode, only the scratch need too large: rejected
    # before any launch (16 is a dummy, never dereferenced, device address)
    rc = capi.raw.pa_decode_static_workspace(16, 16, 16, 16, 16, 2048, 16, 4096, 64, 32768, 0.088, 16, 1 << 20,
                                             16, 8, 128, 2, None)
    assert rc == PA_ERR_WORKSPACE


@pytest.mark.gpu
def test_static_workspace_matches_caller_workspace_twice_in_a_row():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from paged_kv_cache_464_b200 import capi
    capi.get_device_error(clear=True)
    runs = [("llama3_8b_gqa", [128, 700, 4096, 33, 1500, 2049], 0),
            ("long_context", [32768, 9000, 513], 512)]
    for name, lens, P in runs:
        case = inputs.make_case(name, lens=lens)
        dev = "cuda"
        q, k, v = case.q.to(dev), case.k_cache_post.to(dev), case.v_cache_post.to(dev)
        bt, cl = case.block_tables.to(dev), case.context_lens.to(dev)
        maxL = case.max_context_len
        cfg = case.cfg
        need = capi.decode_workspace_bytes(cfg.num_seqs, cfg.num_heads, cfg.num_kv_heads, cfg.head_dim, maxL, P)
        assert 0 < need <= capi.STATIC_WORKSPACE_BYTES, "the case must use the split-K scratch"
        ref = capi.decode(q, k, v, bt, cl, case.scale, max_context_len=maxL, partition_size=P,
                          workspace=torch.empty(need, dtype=torch.uint8, device=dev))
        out = torch.full_like(q, float("nan"))
        rc = capi.raw.pa_decode_static_workspace(
            out.data_ptr(), q.data_ptr(), k.data_ptr(), v.data_ptr(), bt.data_ptr(), bt.shape[1], cl.data_ptr(),
            cfg.num_seqs, cfg.num_heads, maxL, case.scale, P, k.shape[0], 16, cfg.num_kv_heads, cfg.head_dim,
            capi.DTYPE_CODE[q.dtype], torch.cuda.current_stream().cuda_stream)
        assert rc == 0, capi.raw.pa_status_string(rc)
        torch.cuda.synchronize()
        _close(out, ref, cfg.dtype)
        assert torch.equal(out, ref), f"{name}: differs from pa_decode with a caller workspace"
    code, detail = capi.get_device_error(clear=True)
    assert code == 0, (code, detail)
