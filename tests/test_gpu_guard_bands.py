"""Guard bands: every buffer a call writes (caches, outputs, the split-K
workspace) is a view into a larger allocation whose margins hold a sentinel
byte pattern.  After the call the margins must be untouched, and the results
must equal those of the same calls on plain buffers (so the calls really ran
on the guarded views)."""
import pytest
import torch

from paged_kv_cache_464_b200 import inputs

pytestmark = pytest.mark.gpu

SENTINEL = 0x5A
MARGIN_ROWS = 3   # rows of the first dimension on each side


@pytest.fixture(scope="module")
def pa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from paged_kv_cache_464_b200 import capi
    capi.get_device_error(clear=True)
    return capi


class Guarded:
    """A tensor living in rows [MARGIN_ROWS, MARGIN_ROWS + n) of a larger one."""

    def __init__(self, like: torch.Tensor):
        n = like.shape[0]
        self.big = torch.empty((n + 2 * MARGIN_ROWS,) + tuple(like.shape[1:]), dtype=like.dtype, device="cuda")
        self.big.view(torch.uint8).fill_(SENTINEL)
        self.t = self.big[MARGIN_ROWS:MARGIN_ROWS + n]
        self.t.copy_(like)
        assert self.t.is_contiguous() and self.t.data_ptr() % 256 == 0

    def margins_intact(self) -> bool:
        b = self.big.view(torch.uint8).view(self.big.shape[0], -1)
        return bool((b[:MARGIN_ROWS] == SENTINEL).all() and (b[-MARGIN_ROWS:] == SENTINEL).all())


def _same_bytes(a: torch.Tensor, b: torch.Tensor) -> bool:
    """Bitwise equality (the generated caches hold NaN-poisoned stale slots)."""
    return torch.equal(a.contiguous().view(torch.uint8), b.contiguous().view(torch.uint8))


def _raw_guard(nbytes: int) -> Guarded:
    return Guarded(torch.empty((nbytes // 256, 256), dtype=torch.uint8, device="cuda"))


@pytest.mark.parametrize("name,P", [("llama3_8b_gqa", 64), ("shared_prefix", 0), ("tiny", 16)])
def test_decode_step_writes_stay_in_bounds(pa, name, P):
    lens = {"llama3_8b_gqa": [128, 250, 17, 5, 1024, 33], "shared_prefix": [1040, 1300, 1536, 1100],
            "tiny": None}[name]
    case = inputs.make_case(name, lens=lens)
    dev = "cuda"
    q, bt, cl = case.q.to(dev), case.block_tables.to(dev), case.context_lens.to(dev)
    key, value, slots, pairs = case.key.to(dev), case.value.to(dev), case.slot_mapping.to(dev), case.block_mapping.to(dev)
    S, hq, d = q.shape
    hkv = case.k_cache.shape[2]
    need = pa.decode_workspace_bytes(S, hq, hkv, d, case.max_context_len, P)

    # plain buffers
    k, v = case.k_cache.to(dev), case.v_cache.to(dev)
    if pairs.numel():
        pa.copy_blocks(k, v, pairs)
    pa.reshape_and_cache(key, value, k, v, slots)
    out = pa.decode(q, k, v, bt, cl, case.scale, max_context_len=case.max_context_len, partition_size=P)

    # guarded buffers
    gk, gv = Guarded(case.k_cache.to(dev)), Guarded(case.v_cache.to(dev))
    gout = Guarded(torch.zeros_like(q))
    gws = _raw_guard(max(256, (need + 255) // 256 * 256))
    if pairs.numel():
        pa.copy_blocks(gk.t, gv.t, pairs)
    pa.reshape_and_cache(key, value, gk.t, gv.t, slots)
    pa.decode(q, gk.t, gv.t, bt, cl, case.scale, gout.t, max_context_len=case.max_context_len, partition_size=P,
              workspace=gws.t.view(-1) if need else None)
    torch.cuda.synchronize()
    for what, g in (("k_cache", gk), ("v_cache", gv), ("out", gout), ("workspace", gws)):
        assert g.margins_intact(), f"{name}: a write left {what}"
    assert _same_bytes(gk.t, k) and _same_bytes(gv.t, v)
    assert _same_bytes(gout.t, out)
    code, detail = pa.get_device_error(clear=True)
    assert code == 0, (code, detail)


def test_fp8_writes_stay_in_bounds(pa):
    case = inputs.make_case("llama3_8b_gqa_fp8", lens=[130, 1, 700, 33])
    sc = case.cfg.kv_scale
    dev = "cuda"
    nb, bs, hkv, d = case.k_cache.shape
    pool = torch.arange(nb * bs, dtype=torch.int64, device=dev)
    k16, v16 = case.k_cache.to(dev).view(nb * bs, hkv, d), case.v_cache.to(dev).view(nb * bs, hkv, d)
    q, bt, cl = case.q.to(dev), case.block_tables.to(dev), case.context_lens.to(dev)
    zeros = torch.zeros((nb, bs, hkv, d), dtype=torch.uint8, device=dev)

    k8, v8 = zeros.clone(), zeros.clone()
    pa.reshape_and_cache_fp8(k16, v16, k8, v8, pool, sc, sc)
    out = pa.decode_fp8(q, k8, v8, sc, sc, bt, cl, case.scale, max_context_len=case.max_context_len,
                        partition_size=64)

    gk, gv, gout = Guarded(zeros), Guarded(zeros), Guarded(torch.zeros_like(q))
    pa.reshape_and_cache_fp8(k16, v16, gk.t, gv.t, pool, sc, sc)
    pa.decode_fp8(q, gk.t, gv.t, sc, sc, bt, cl, case.scale, gout.t, max_context_len=case.max_context_len,
                  partition_size=64)
    torch.cuda.synchronize()
    for what, g in (("k_cache", gk), ("v_cache", gv), ("out", gout)):
        assert g.margins_intact(), f"fp8: a write left {what}"
    assert _same_bytes(gk.t, k8) and _same_bytes(gv.t, v8) and _same_bytes(gout.t, out)
    code, detail = pa.get_device_error(clear=True)
    assert code == 0, (code, detail)


def test_prefill_writes_stay_in_bounds(pa):
    cfg = inputs.DecodeConfig("guard_prefill", 78, 3, 8, 2, 128, "bf16")
    pc = inputs.make_prefill_case(cfg, chunk_lens=[70, 5, 129], prefix_lens=[40, 0, 300])
    dev = "cuda"
    args = (pc.q.to(dev), pc.k_cache.to(dev), pc.v_cache.to(dev), pc.block_tables.to(dev), pc.context_lens.to(dev),
            pc.query_start_loc.to(dev), pc.scale)
    out = pa.prefill(*args, max_query_len=pc.max_query_len)
    gout = Guarded(torch.zeros_like(pc.q.to(dev)))
    pa.prefill(*args, gout.t, max_query_len=pc.max_query_len)
    torch.cuda.synchronize()
    assert gout.margins_intact(), "prefill: a write left out"
    assert _same_bytes(gout.t, out)
    code, detail = pa.get_device_error(clear=True)
    assert code == 0, (code, detail)
