"""Prefix caching end to end on the GPU ("vLLM 原理与源码阅读", Prefix Caching):
a request whose prompt starts with cached full blocks computes and writes only
its suffix, and its chunked prefill over the shared blocks gives what the
oracle gives -- and bit for bit what a run without caching gives."""
import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu

BS, HKV, HQ, D = 16, 2, 8, 128


@pytest.fixture(scope="module")
def pa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from paged_kv_cache_464_b200 import capi
    capi.get_device_error(clear=True)
    return capi


def _rows(tokens, positions, which):
    """Stand-in for a model: the K (which=0) or V (which=1) rows of a token at a
    position, a seeded function of (token id, position) only."""
    out = np.empty((len(tokens), HKV, D), np.float32)
    for i, (t, p) in enumerate(zip(tokens, positions)):
        out[i] = np.random.default_rng([int(t), int(p), which]).standard_normal((HKV, D), dtype=np.float32)
    return torch.from_numpy(out).to(torch.bfloat16)


def _q(tokens, positions):
    out = np.empty((len(tokens), HQ, D), np.float32)
    for i, (t, p) in enumerate(zip(tokens, positions)):
        out[i] = np.random.default_rng([int(t), int(p), 7]).standard_normal((HQ, D), dtype=np.float32)
    return torch.from_numpy(out).to(torch.bfloat16)


def _run(pa, prefix_caching, prompts, nb=24):
    """Each prompt in turn: allocate (with or without caching), write the K/V of
    the tokens that are not cached, run the chunked prefill over those tokens.
    Returns the outputs of every prompt and the cached-token counts."""
    from paged_kv_cache_464_b200.block_manager import BlockManager
    m = BlockManager(nb, BS, prefix_caching=prefix_caching)
    kc = torch.zeros((nb, BS, HKV, D), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    outs, cached_counts, cpu_states = [], [], []
    for seq, toks in enumerate(prompts):
        slots, cached = m.allocate_prompt(seq, toks)
        cached_counts.append(cached)
        pos = list(range(cached, len(toks)))
        new = toks[cached:]
        pa.reshape_and_cache(_rows(new, pos, 0).cuda(), _rows(new, pos, 1).cuda(), kc, vc,
                             torch.tensor(slots[cached:], dtype=torch.int64, device="cuda"))
        bt, cl = m.tables([seq], (len(toks) + BS - 1) // BS)
        q = _q(new, pos)
        qsl = torch.tensor([0, len(new)], dtype=torch.int32)
        scale = float(np.float32(D ** -0.5))
        out = pa.prefill(q.cuda(), kc, vc, torch.from_numpy(bt).cuda(), torch.from_numpy(cl).cuda(), qsl.cuda(), scale,
                         max_query_len=len(new))
        torch.cuda.synchronize()
        outs.append(out.cpu())
        cpu_states.append((q, kc.cpu(), vc.cpu(), torch.from_numpy(bt.copy()), torch.from_numpy(cl.copy()), qsl, scale))
    return outs, cached_counts, cpu_states


def test_cached_prefix_computes_only_the_suffix(pa):
    rng = np.random.default_rng(3)
    system = rng.integers(0, 32000, 48).tolist()        # three full blocks
    prompts = [system + rng.integers(0, 32000, 20).tolist(),
               system + rng.integers(0, 32000, 30).tolist(),
               system[:32] + rng.integers(0, 32000, 9).tolist(),
               rng.integers(0, 32000, 40).tolist()]
    outs, cached, states = _run(pa, True, prompts)
    assert cached == [0, 48, 32, 0]
    orc = oracle.get()
    for i, (q, kc, vc, bt, cl, qsl, scale) in enumerate(states):
        ref = orc.paged_prefill(q, kc, vc, bt, cl, qsl, scale)
        g = outs[i].to(torch.float64).numpy()
        assert np.isfinite(g).all()
        assert (np.abs(g - ref) <= 2e-3 + 1e-2 * np.abs(ref)).all(), f"prompt {i}"
    # without caching every prompt is computed whole; the rows of the tokens the
    # cached run computed are bit-identical (same K/V, other physical blocks)
    outs_full, cached_full, _ = _run(pa, False, prompts)
    assert cached_full == [0, 0, 0, 0]
    for i, c in enumerate(cached):
        assert torch.equal(outs_full[i][c:], outs[i]), f"prompt {i}"
    code, detail = pa.get_device_error(clear=True)
    assert code == 0, (code, detail)
