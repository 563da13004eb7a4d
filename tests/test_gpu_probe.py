"""pa_stream_read, the plain streaming read that the bench uses for the
read-only bandwidth: it must read every byte exactly once (the XOR of all
8-byte words it returns equals the host's), including a ragged tail."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("nbytes", [16, 4096 + 48, (1 << 24) + 16 * 12345])
def test_stream_read_touches_every_word_once(nbytes):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from paged_kv_cache_464_b200 import capi
    g = torch.Generator().manual_seed(nbytes)
    host = torch.randint(0, 256, (nbytes,), dtype=torch.uint8, generator=g)
    buf = host.cuda()
    sink = torch.zeros(1, dtype=torch.int64, device="cuda")
    capi.stream_read(buf, sink)
    torch.cuda.synchronize()
    want = np.bitwise_xor.reduce(host.numpy().view(np.uint64))
    assert int(sink.cpu().numpy().view(np.uint64)[0]) == int(want)
