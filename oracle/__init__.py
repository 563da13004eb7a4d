"""CPU oracle for paged decode attention (test infrastructure only).

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg
may import this package.  The product path never does: it has no fallback to
this code.  The arithmetic lives in ``pa_oracle.c`` (fp64, plain loops); this
file only compiles it with gcc and marshals arguments through ctypes.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np
import torch

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "pa_oracle.c")
LIB = os.path.join(HERE, "libpa_oracle.so")

DTYPE_CODE = {torch.float32: 0, torch.float16: 1, torch.bfloat16: 2}
STATUS = {0: "ok", 1: "bad arguments", 2: "block id out of range", 3: "slot out of range",
          4: "copy pair conflict", 5: "bad context length", 6: "out of memory"}


class OracleError(RuntimeError):
    def __init__(self, code: int):
        super().__init__(f"oracle: {STATUS.get(code, code)}")
        self.code = code


def compile_library(src: str = SRC, out: str = LIB, extra_flags=()) -> str:
    """Compile the oracle with gcc (-O2, no fast-math: no reassociation)."""
    cmd = ["gcc", "-O2", "-std=c99", "-fopenmp", "-fPIC", "-shared", "-Wall", "-Wextra",
           *extra_flags, src, "-o", out, "-lm"]
    subprocess.run(cmd, check=True)
    return out


def build(force: bool = False) -> str:
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        compile_library()
    return LIB


def _ptr(t) -> ctypes.c_void_p:
    if isinstance(t, np.ndarray):
        return ctypes.c_void_p(t.ctypes.data)
    assert t.device.type == "cpu" and t.is_contiguous(), "oracle takes contiguous CPU tensors"
    return ctypes.c_void_p(t.data_ptr())


class Oracle:
    """ctypes view of one compiled oracle library."""

    def __init__(self, path: Optional[str] = None):
        self.path = path or build()
        lib = ctypes.CDLL(self.path)
        P, I, I64, D = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_double
        lib.oracle_paged_decode.restype = I
        lib.oracle_paged_decode.argtypes = [P, P, I, P, P, P, P, I, P, I, I, I, I, I, I, D, I]
        lib.oracle_reshape_and_cache.restype = I
        lib.oracle_reshape_and_cache.argtypes = [P, P, P, P, P, I, I, I, I, I, I]
        lib.oracle_copy_blocks.restype = I
        lib.oracle_copy_blocks.argtypes = [P, P, P, I, I, I, I, I, I]
        lib.oracle_slot_for_position.restype = I64
        lib.oracle_slot_for_position.argtypes = [P, I, I64, I]
        lib.oracle_widen.restype = None
        lib.oracle_widen.argtypes = [P, P, I64, I]
        U8 = ctypes.c_void_p
        lib.oracle_e4m3_decode.restype = None
        lib.oracle_e4m3_decode.argtypes = [P, U8, I64]
        lib.oracle_e4m3_quantize.restype = None
        lib.oracle_e4m3_quantize.argtypes = [U8, P, I64, I, ctypes.c_float]
        lib.oracle_reshape_and_cache_fp8.restype = I
        lib.oracle_reshape_and_cache_fp8.argtypes = [U8, U8, P, P, P, I, I, I, I, I, I, ctypes.c_float,
                                                     ctypes.c_float]
        lib.oracle_paged_decode_fp8.restype = I
        lib.oracle_paged_decode_fp8.argtypes = [P, P, I, U8, U8, D, D, P, I, P, I, I, I, I, I, I, D]
        lib.oracle_paged_prefill.restype = I
        lib.oracle_paged_prefill.argtypes = [P, P, P, P, P, I, P, P, I, I, I, I, I, I, D, I]
        lib.oracle_num_threads.restype = I
        lib.oracle_set_num_threads.argtypes = [I]
        self.lib = lib

    # -- decode ---------------------------------------------------------------
    def paged_decode(self, q, k_cache, v_cache, block_tables, context_lens, scale,
                     *, num_kv_heads=None, block_size=None, return_weights=False):
        """fp64 paged decode.  q [S,Hq,D]; caches [NB,bs,Hkv,D]; returns out [S,Hq,D] f64
        (and weights [S,Hq,maxL] f64 when ``return_weights``)."""
        assert q.dtype == k_cache.dtype == v_cache.dtype
        S, Hq, D = q.shape
        NB, bs, Hkv, D2 = k_cache.shape
        assert D2 == D and tuple(v_cache.shape) == tuple(k_cache.shape)
        bt = block_tables.to(torch.int32).contiguous()
        cl = context_lens.to(torch.int32).contiguous()
        MBS = bt.shape[1] if bt.dim() == 2 else 0
        out = np.zeros((S, Hq, D), dtype=np.float64)
        maxL = int(cl.max().item()) if S else 0
        w = np.zeros((S, Hq, max(maxL, 1)), dtype=np.float64) if return_weights else None
        rc = self.lib.oracle_paged_decode(
            _ptr(out), _ptr(w) if w is not None else None, max(maxL, 1),
            _ptr(q.contiguous()), _ptr(k_cache.contiguous()), _ptr(v_cache.contiguous()),
            _ptr(bt), MBS, _ptr(cl), S, Hq, Hkv, D, bs, NB, float(np.float32(scale)),
            DTYPE_CODE[q.dtype])
        if rc:
            raise OracleError(rc)
        return (out, w) if return_weights else out

    def decode_case(self, case, return_weights=False):
        """Decode a workload case after its step (post-step cache)."""
        return self.paged_decode(case.q, case.k_cache_post, case.v_cache_post, case.block_tables,
                                 case.context_lens, case.scale, return_weights=return_weights)

    # -- cache writes -----------------------------------------------------------
    def reshape_and_cache(self, k_cache, v_cache, key, value, slot_mapping):
        """In place on CPU tensors; returns the status code (0 = ok)."""
        NB, bs, Hkv, D = k_cache.shape
        T = key.shape[0]
        assert k_cache.is_contiguous() and v_cache.is_contiguous()
        sm = slot_mapping.to(torch.int64).contiguous()
        return self.lib.oracle_reshape_and_cache(
            _ptr(k_cache), _ptr(v_cache), _ptr(key.contiguous()), _ptr(value.contiguous()),
            _ptr(sm), T, Hkv, D, bs, NB, DTYPE_CODE[k_cache.dtype])

    def copy_blocks(self, k_cache, v_cache, block_mapping):
        """In place on CPU tensors; returns the status code (0 = ok)."""
        NB, bs, Hkv, D = k_cache.shape
        bm = block_mapping.to(torch.int64).contiguous()
        P = bm.shape[0] if bm.numel() else 0
        return self.lib.oracle_copy_blocks(_ptr(k_cache), _ptr(v_cache), _ptr(bm) if P else None,
                                           P, Hkv, D, bs, NB, DTYPE_CODE[k_cache.dtype])

    def slot_for_position(self, block_table_row, pos, block_size):
        row = block_table_row.to(torch.int32).contiguous()
        return int(self.lib.oracle_slot_for_position(_ptr(row), row.numel(), int(pos), block_size))

    def widen(self, t) -> np.ndarray:
        t = t.contiguous()
        out = np.empty(t.numel(), dtype=np.float64)
        self.lib.oracle_widen(_ptr(out), _ptr(t), t.numel(), DTYPE_CODE[t.dtype])
        return out.reshape(tuple(t.shape))

    def step(self, case):
        """Run one decode step of a case on the CPU: copy-on-write copies, the
        new token's write, then decode.  Returns (out, k_cache, v_cache)."""
        k = case.k_cache.clone()
        v = case.v_cache.clone()
        return self.step_inplace(case, k, v), k, v

    def step_inplace(self, case, k, v):
        """The same step on caches the caller owns (modified in place); returns out."""
        rc = self.copy_blocks(k, v, case.block_mapping)
        if rc:
            raise OracleError(rc)
        rc = self.reshape_and_cache(k, v, case.key, case.value, case.slot_mapping)
        if rc:
            raise OracleError(rc)
        return self.paged_decode(case.q, k, v, case.block_tables, case.context_lens, case.scale)

    # -- prefill -------------------------------------------------------------------------
    def paged_prefill(self, q, k_cache, v_cache, block_tables, context_lens, query_start_loc, scale):
        """q [T, Hq, D]; chunk of sequence b = rows query_start_loc[b]:query_start_loc[b+1],
        the last tokens of its context.  Returns out [T, Hq, D] f64."""
        T, Hq, D = q.shape
        NB, bs, Hkv, D2 = k_cache.shape
        assert D2 == D and q.dtype == k_cache.dtype == v_cache.dtype
        bt = block_tables.to(torch.int32).contiguous()
        cl = context_lens.to(torch.int32).contiguous()
        qsl = query_start_loc.to(torch.int32).contiguous()
        S = cl.numel()
        out = np.zeros((T, Hq, D), dtype=np.float64)
        rc = self.lib.oracle_paged_prefill(_ptr(out), _ptr(q.contiguous()), _ptr(k_cache.contiguous()),
                                           _ptr(v_cache.contiguous()), _ptr(bt), bt.shape[1], _ptr(cl), _ptr(qsl), S,
                                           Hq, Hkv, D, bs, NB, float(np.float32(scale)), DTYPE_CODE[q.dtype])
        if rc:
            raise OracleError(rc)
        return out

    # -- FP8 (E4M3) caches ------------------------------------------------------------
    def e4m3_decode(self, codes: torch.Tensor) -> np.ndarray:
        c = codes.contiguous().view(torch.uint8)
        out = np.empty(c.numel(), dtype=np.float64)
        self.lib.oracle_e4m3_decode(_ptr(out), _ptr(c), c.numel())
        return out.reshape(tuple(codes.shape))

    def e4m3_quantize(self, x: torch.Tensor, scale: float) -> torch.Tensor:
        x = x.contiguous()
        out = torch.empty(x.shape, dtype=torch.uint8)
        self.lib.oracle_e4m3_quantize(_ptr(out), _ptr(x), x.numel(), DTYPE_CODE[x.dtype], float(scale))
        return out

    def reshape_and_cache_fp8(self, k_cache, v_cache, key, value, slot_mapping, k_scale, v_scale):
        """k_cache / v_cache: uint8 [NB, bs, Hkv, D], in place; returns the status code."""
        NB, bs, Hkv, D = k_cache.shape
        assert k_cache.dtype == torch.uint8 and k_cache.is_contiguous() and v_cache.is_contiguous()
        sm = slot_mapping.to(torch.int64).contiguous()
        return self.lib.oracle_reshape_and_cache_fp8(
            _ptr(k_cache), _ptr(v_cache), _ptr(key.contiguous()), _ptr(value.contiguous()), _ptr(sm),
            key.shape[0], Hkv, D, bs, NB, DTYPE_CODE[key.dtype], float(k_scale), float(v_scale))

    def paged_decode_fp8(self, q, k_cache, v_cache, k_scale, v_scale, block_tables, context_lens, scale):
        S, Hq, D = q.shape
        NB, bs, Hkv, D2 = k_cache.shape
        assert D2 == D and k_cache.dtype == torch.uint8
        bt = block_tables.to(torch.int32).contiguous()
        cl = context_lens.to(torch.int32).contiguous()
        out = np.zeros((S, Hq, D), dtype=np.float64)
        rc = self.lib.oracle_paged_decode_fp8(
            _ptr(out), _ptr(q.contiguous()), DTYPE_CODE[q.dtype], _ptr(k_cache.contiguous()),
            _ptr(v_cache.contiguous()), float(np.float32(k_scale)), float(np.float32(v_scale)), _ptr(bt),
            bt.shape[1], _ptr(cl), S, Hq, Hkv, D, bs, NB, float(np.float32(scale)))
        if rc:
            raise OracleError(rc)
        return out

    @property
    def num_threads(self) -> int:
        return self.lib.oracle_num_threads()

    def set_num_threads(self, n: int) -> None:
        self.lib.oracle_set_num_threads(n)


_default: Optional[Oracle] = None


def get() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle()
    return _default
