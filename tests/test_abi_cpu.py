"""C-ABI checks that need no GPU: the library loads, exports every function
include/pa.h declares, and host-side validation returns the documented codes
before any CUDA call is made."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pa.h")
HEADERS = sorted(os.path.join(ROOT, "include", f) for f in os.listdir(os.path.join(ROOT, "include"))
                 if f.endswith(".h"))


@pytest.fixture(scope="module")
def capi():
    from paged_kv_cache_464_b200 import build
    build.build()
    from paged_kv_cache_464_b200 import capi
    return capi


def declared_functions(headers=HEADERS):
    names = set()
    for h in headers:
        text = re.sub(r"/\*.*?\*/", "", open(h).read(), flags=re.S)
        names |= set(re.findall(r"\b(pa_[a-z0-9_]+)\s*\(", text))
    return sorted(names)


def test_header_declares_the_three_calls():
    names = declared_functions()
    for n in ("pa_reshape_and_cache", "pa_decode", "pa_copy_blocks"):
        assert n in names


def test_library_exports_every_declared_symbol(capi):
    out = subprocess.run(["nm", "-D", "--defined-only", capi.library_path()], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\sT\s(\w+)$", out, flags=re.M))
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, missing
    from paged_kv_cache_464_b200 import block_manager
    assert sorted(capi.EXPORTED + block_manager.EXPORTED) == declared_functions()


def test_header_compiles_as_c():
    src = "".join(f'#include "{h}"\n' for h in HEADERS) + "int main(void){ return (int)PA_OK + (int)PA_BM_OK; }\n"
    r = subprocess.run(["gcc", "-x", "c", "-std=c99", "-Wall", "-Werror", "-fsyntax-only", "-"], input=src,
                       text=True, capture_output=True)
    assert r.returncode == 0, r.stderr


def test_status_strings(capi):
    for code in range(7):
        assert capi.raw.pa_status_string(code).decode().startswith("PA_")


def test_partition_and_workspace_sizes(capi):
    # explicit partition sizes must be multiples of the block size
    assert capi.decode_partition_size(8, 64, 8, 128, 32768, 512) == 512
    assert capi.decode_partition_size(8, 64, 8, 128, 32768, 500) == -1
    assert capi.decode_partition_size(8, 64, 8, 128, -1, 0) == -1
    # automatic choice: one partition when short, split when long
    p = capi.decode_partition_size(4, 4, 4, 64, 100, 0)
    assert p >= 100 and p % 16 == 0
    assert capi.decode_workspace_bytes(4, 4, 4, 64, 100, 0) == 0
    p = capi.decode_partition_size(8, 64, 8, 128, 32768, 0)
    npart = -(-32768 // p)
    ws = capi.decode_workspace_bytes(8, 64, 8, 128, 32768, 0)
    assert ws >= 8 * 64 * npart * (128 + 2) * 4
    # long-context workload at partition 512: 8*64*64 rows of (128 + 2) floats
    assert capi.decode_workspace_bytes(8, 64, 8, 128, 32768, 512) >= 8 * 64 * 64 * 130 * 4


def _decode(capi, **kw):
    args = dict(out=16, q=16, k=16, v=16, bt=16, mbs=4, cl=16, S=2, Hq=4, maxL=64, scale=0.125, P=0,
                ws=None, wsb=0, NB=8, bs=16, Hkv=4, D=64, dt=0)
    args.update(kw)
    a = args
    return capi.raw.pa_decode(a["out"], a["q"], a["k"], a["v"], a["bt"], a["mbs"], a["cl"], a["S"], a["Hq"],
                              a["maxL"], a["scale"], a["P"], a["ws"], a["wsb"], a["NB"], a["bs"], a["Hkv"],
                              a["D"], a["dt"], None)


def test_decode_host_validation(capi):
    PA_ERR_NULL, PA_ERR_DTYPE, PA_ERR_SHAPE, PA_ERR_WORKSPACE, PA_ERR_ALIGN = 1, 2, 3, 4, 6
    assert _decode(capi, dt=7) == PA_ERR_DTYPE
    assert _decode(capi, bs=32) == PA_ERR_SHAPE                 # block size must be 16
    assert _decode(capi, D=128) == PA_ERR_SHAPE                 # fp32 row must be 256 B
    assert _decode(capi, dt=2, D=64) == PA_ERR_SHAPE            # bf16 needs D=128
    assert _decode(capi, Hq=6) == PA_ERR_SHAPE                  # Hq % Hkv
    assert _decode(capi, Hq=64) == PA_ERR_SHAPE                 # group 16 not built
    assert _decode(capi, P=24) == PA_ERR_SHAPE                  # partition not a multiple of 16
    assert _decode(capi, S=-1) == PA_ERR_SHAPE
    assert _decode(capi, NB=0) == PA_ERR_SHAPE
    assert _decode(capi, scale=float("nan")) == PA_ERR_SHAPE
    assert _decode(capi, q=None) == PA_ERR_NULL
    assert _decode(capi, out=8) == PA_ERR_ALIGN
    assert _decode(capi, maxL=4096, P=512) == PA_ERR_WORKSPACE  # split needs a workspace
    assert _decode(capi, maxL=4096, P=512, ws=256, wsb=10) == PA_ERR_WORKSPACE
    assert _decode(capi, S=0) == 0                              # nothing to do
    assert _decode(capi, dt=3, D=128) == PA_ERR_DTYPE           # 1-byte caches go through pa_decode_fp8


def test_cache_ops_host_validation(capi):
    r = capi.raw
    # (key, value, k_cache, v_cache, slots, T, NB, bs, Hkv, D, dtype, stream)
    assert r.pa_reshape_and_cache(16, 16, 16, 16, 16, 0, 8, 16, 4, 64, 0, None) == 0
    assert r.pa_reshape_and_cache(16, 16, 16, 16, 16, -1, 8, 16, 4, 64, 0, None) == 3
    assert r.pa_reshape_and_cache(None, 16, 16, 16, 16, 4, 8, 16, 4, 64, 0, None) == 1
    assert r.pa_reshape_and_cache(16, 16, 24, 16, 16, 4, 8, 16, 4, 64, 0, None) == 6
    assert r.pa_reshape_and_cache(16, 16, 16, 16, 16, 4, 8, 16, 4, 64, 7, None) == 2
    assert r.pa_reshape_and_cache(16, 16, 16, 16, 16, 4, 8, 16, 4, 64, 3, None) == 3     # 1-byte rows must be 128 B
    # (k_cache, v_cache, mapping, P, NB, bs, Hkv, D, dtype, stream)
    assert r.pa_copy_blocks(16, 16, 16, 0, 8, 16, 4, 64, 0, None) == 0
    assert r.pa_copy_blocks(16, 16, None, 2, 8, 16, 4, 64, 0, None) == 1
    assert r.pa_copy_blocks(16, 16, 16, -2, 8, 16, 4, 64, 0, None) == 3
    assert r.pa_copy_blocks(16, 16, 16, 2, 8, 16, 4, 96, 1, None) == 3


def test_fp8_host_validation(capi):
    r = capi.raw
    # pa_reshape_and_cache_fp8(key, value, kc, vc, slots, T, NB, bs, Hkv, D, src_dtype, k_scale, v_scale, stream)
    assert r.pa_reshape_and_cache_fp8(16, 16, 16, 16, 16, 0, 8, 16, 4, 128, 2, 0.1, 0.1, None) == 0
    assert r.pa_reshape_and_cache_fp8(16, 16, 16, 16, 16, 4, 8, 16, 4, 128, 0, 0.1, 0.1, None) == 2   # f32 source
    assert r.pa_reshape_and_cache_fp8(16, 16, 16, 16, 16, 4, 8, 16, 4, 64, 2, 0.1, 0.1, None) == 3    # D=64
    assert r.pa_reshape_and_cache_fp8(16, 16, 16, 16, 16, 4, 8, 16, 4, 128, 2, 0.0, 0.1, None) == 3   # scale 0
    assert r.pa_reshape_and_cache_fp8(16, 16, 8, 16, 16, 4, 8, 16, 4, 128, 2, 0.1, 0.1, None) == 6    # alignment
    # pa_decode_fp8(out, q, kc, vc, ks, vs, bt, mbs, cl, S, Hq, maxL, scale, P, ws, wsb, NB, bs, Hkv, D, q_dtype, s)
    dec = lambda **k: r.pa_decode_fp8(k.get("out", 16), 16, 16, 16, k.get("ks", 0.1), 0.1, 16, 4, 16, 2, 8, 64,
                                      0.088, 0, None, 0, 8, 16, 2, k.get("D", 128), k.get("qd", 2), None)
    assert dec(qd=0) == 2            # q must be fp16 or bf16
    assert dec(D=64) == 3
    assert dec(ks=float("inf")) == 3
    assert dec(out=8) == 6


def test_prefill_host_validation(capi):
    r = capi.raw
    # pa_prefill(out, q, kc, vc, bt, mbs, cl, qsl, S, Hq, max_query_len, scale, NB, bs, Hkv, D, dtype, stream)
    def pf(**k):
        a = dict(out=16, q=16, bt=16, mbs=8, cl=16, qsl=16, S=2, Hq=32, mq=64, scale=0.088, bs=16, Hkv=8, D=128,
                 dt=2)
        a.update(k)
        return r.pa_prefill(a["out"], a["q"], 16, 16, a["bt"], a["mbs"], a["cl"], a["qsl"], a["S"], a["Hq"],
                            a["mq"], a["scale"], 64, a["bs"], a["Hkv"], a["D"], a["dt"], None)
    assert pf(S=0) == 0 and pf(mq=0) == 0          # nothing to do
    assert pf(dt=0, D=64) == 2                     # fp32 caches: decode only
    assert pf(dt=7) == 2
    assert pf(D=64) == 3                           # head_dim 128 only
    assert pf(Hq=48) == 3                          # group 6
    assert pf(Hq=30) == 3                          # Hq % Hkv
    assert pf(mq=-1) == 3 and pf(S=-1) == 3 and pf(S=70000) == 3
    assert pf(scale=float("nan")) == 3
    assert pf(qsl=None) == 1 and pf(q=None) == 1
    assert pf(out=8) == 6 and pf(qsl=2) == 6


def test_copy_blocks_pair_cap(capi):
    r = capi.raw
    assert capi.MAX_COPY_PAIRS == 65536
    assert r.pa_copy_blocks(16, 16, 16, capi.MAX_COPY_PAIRS + 1, 8, 16, 4, 64, 0, None) == 3


def test_static_workspace_checks_follow_pa_decode(capi):
    """pa_decode_static_workspace runs every pa_decode check first, in its order;
    only then does an oversized scratch need return PA_ERR_WORKSPACE."""
    r = capi.raw

    def sw(**k):
        a = dict(out=16, q=16, S=4096, maxL=32768, P=16, dt=2, D=128, Hq=64)
        a.update(k)
        return r.pa_decode_static_workspace(a["out"], a["q"], 16, 16, 16, 2048, 16, a["S"], a["Hq"], a["maxL"],
                                            0.088, a["P"], 1 << 20, 16, 8, a["D"], a["dt"], None)
    assert sw() == 4                 # too large for the library's scratch
    assert sw(out=8) == 6            # misaligned out: pa_decode's PA_ERR_ALIGN comes first
    assert sw(q=None) == 1           # NULL q: PA_ERR_NULL comes first
    assert sw(dt=3) == 2             # 1-byte caches: PA_ERR_DTYPE, as pa_decode
    assert sw(D=64) == 3             # bf16 rows must be 256 bytes
    assert sw(P=24) == 3             # partition not a multiple of 16
    assert sw(S=0) == 0              # nothing to do


def test_stall_hook_arguments(capi):
    r = capi.raw
    assert r.pa_test_stall_next_launch(2, 0) == 3      # unknown kernel
    assert r.pa_test_stall_next_launch(0, -2) == 3     # bad CTA index
    assert r.pa_test_stall_next_launch(0, -1) == 0     # disarm
    assert r.pa_test_stall_next_launch(1, -1) == 0


def test_stream_read_host_validation(capi):
    r = capi.raw
    assert r.pa_stream_read(16, 0, 16, None) == 0       # nothing to read
    assert r.pa_stream_read(16, 24, 16, None) == 3      # not a multiple of 16 bytes
    assert r.pa_stream_read(None, 32, 16, None) == 1
    assert r.pa_stream_read(8, 32, 16, None) == 6       # buffer not 16-byte aligned
    assert r.pa_stream_read(16, 32, 12, None) == 6      # sink not 8-byte aligned
