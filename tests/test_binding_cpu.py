"""The binding never computes on the host: every compute call given CPU
tensors of valid shapes raises before anything runs (no CPU fallback)."""
import pytest
import torch


@pytest.fixture(scope="module")
def capi():
    from paged_kv_cache_464_b200 import build
    build.build()
    from paged_kv_cache_464_b200 import capi
    return capi


def _case(dtype=torch.bfloat16):
    S, hq, hkv, d, nb = 2, 4, 1, 128, 8
    return dict(q=torch.zeros(S, hq, d, dtype=dtype), k=torch.zeros(nb, 16, hkv, d, dtype=dtype),
                v=torch.zeros(nb, 16, hkv, d, dtype=dtype), key=torch.zeros(S, hkv, d, dtype=dtype),
                value=torch.zeros(S, hkv, d, dtype=dtype), slots=torch.tensor([3, 40], dtype=torch.int64),
                bt=torch.tensor([[0, 1, -1, -1], [2, 3, -1, -1]], dtype=torch.int32),
                cl=torch.tensor([4, 20], dtype=torch.int32), pairs=torch.tensor([[0, 5]], dtype=torch.int64),
                qsl=torch.tensor([0, 1, 2], dtype=torch.int32))


def test_cpu_tensors_are_refused(capi):
    c = _case()
    k8 = torch.zeros(8, 16, 1, 128, dtype=torch.uint8)
    v8 = torch.zeros_like(k8)
    calls = {
        "reshape_and_cache": lambda: capi.reshape_and_cache(c["key"], c["value"], c["k"], c["v"], c["slots"]),
        "copy_blocks": lambda: capi.copy_blocks(c["k"], c["v"], c["pairs"]),
        "decode": lambda: capi.decode(c["q"], c["k"], c["v"], c["bt"], c["cl"], 0.088),
        "decode_split": lambda: capi.decode(c["q"], c["k"], c["v"], c["bt"], c["cl"], 0.088, partition_size=16),
        "decode_append": lambda: capi.decode_append(c["q"], c["key"], c["value"], c["k"], c["v"], c["bt"], c["cl"],
                                                    0.088),
        "reshape_and_cache_fp8": lambda: capi.reshape_and_cache_fp8(c["key"], c["value"], k8, v8, c["slots"], 0.1,
                                                                    0.1),
        "decode_fp8": lambda: capi.decode_fp8(c["q"], k8, v8, 0.1, 0.1, c["bt"], c["cl"], 0.088),
        "prefill": lambda: capi.prefill(c["q"], c["k"], c["v"], c["bt"], c["cl"], c["qsl"], 0.088),
    }
    for name, call in calls.items():
        with pytest.raises(ValueError, match="CUDA tensor"):
            call()
