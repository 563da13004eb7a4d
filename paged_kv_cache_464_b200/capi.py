"""ctypes binding of libpa_b200.so (include/pa.h).  Argument marshalling only.

Every step of the path runs in the library's CUDA kernels; PyTorch supplies
device memory and the current stream.  Loading fails loudly when the library
has not been built -- there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libpa_b200.so")
if not os.path.exists(_LIB_PATH):
    raise ImportError(f"libpa_b200.so is not built ({_LIB_PATH}); run "
                      "`python -m paged_kv_cache_464_b200.build`")

_lib = ctypes.CDLL(_LIB_PATH)
_P, _I, _I64, _F, _SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t

_lib.pa_reshape_and_cache.restype = _I
_lib.pa_reshape_and_cache.argtypes = [_P, _P, _P, _P, _P, _I, _I64, _I, _I, _I, _I, _P]
_lib.pa_decode_partition_size.restype = _I
_lib.pa_decode_partition_size.argtypes = [_I, _I, _I, _I, _I, _I]
_lib.pa_decode_workspace_bytes.restype = _SZ
_lib.pa_decode_workspace_bytes.argtypes = [_I, _I, _I, _I, _I, _I]
_lib.pa_decode.restype = _I
_lib.pa_decode.argtypes = [_P, _P, _P, _P, _P, _I, _P, _I, _I, _I, _F, _I, _P, _SZ, _I64, _I, _I, _I, _I, _P]
_lib.pa_decode_append.restype = _I
_lib.pa_decode_append.argtypes = [_P, _P, _P, _P, _P, _P, _P, _I, _P, _I, _I, _I, _F, _I, _P, _SZ, _I64, _I, _I, _I,
                                  _I, _P]
_lib.pa_decode_static_workspace.restype = _I
_lib.pa_decode_static_workspace.argtypes = [_P, _P, _P, _P, _P, _I, _P, _I, _I, _I, _F, _I, _I64, _I, _I, _I, _I,
                                            _P]
_lib.pa_reshape_and_cache_fp8.restype = _I
_lib.pa_reshape_and_cache_fp8.argtypes = [_P, _P, _P, _P, _P, _I, _I64, _I, _I, _I, _I, _F, _F, _P]
_lib.pa_decode_fp8.restype = _I
_lib.pa_decode_fp8.argtypes = [_P, _P, _P, _P, _F, _F, _P, _I, _P, _I, _I, _I, _F, _I, _P, _SZ, _I64, _I, _I, _I, _I,
                               _P]
_lib.pa_prefill.restype = _I
_lib.pa_prefill.argtypes = [_P, _P, _P, _P, _P, _I, _P, _P, _I, _I, _I, _F, _I64, _I, _I, _I, _I, _P]
_lib.pa_copy_blocks.restype = _I
_lib.pa_copy_blocks.argtypes = [_P, _P, _P, _I, _I64, _I, _I, _I, _I, _P]
_lib.pa_stream_read.restype = _I
_lib.pa_stream_read.argtypes = [_P, _SZ, _P, _P]
_lib.pa_test_stall_next_launch.restype = _I
_lib.pa_test_stall_next_launch.argtypes = [_I, _I64]
_lib.pa_get_device_error.restype = _I
_lib.pa_get_device_error.argtypes = [_P, ctypes.POINTER(_I64), _I]
_lib.pa_status_string.restype = ctypes.c_char_p
_lib.pa_status_string.argtypes = [_I]

EXPORTED = ["pa_reshape_and_cache", "pa_decode_partition_size", "pa_decode_workspace_bytes", "pa_decode",
            "pa_decode_append", "pa_decode_static_workspace", "pa_reshape_and_cache_fp8", "pa_decode_fp8", "pa_prefill",
            "pa_copy_blocks", "pa_stream_read", "pa_test_stall_next_launch", "pa_get_device_error", "pa_status_string"]
MAX_COPY_PAIRS = 65536       # PA_MAX_COPY_PAIRS in include/pa.h
STATIC_WORKSPACE_BYTES = 64 << 20   # PA_STATIC_WORKSPACE_BYTES in include/pa.h

DTYPE_CODE = {torch.float32: 0, torch.float16: 1, torch.bfloat16: 2}
FP8 = 3                      # PA_FP8_E4M3: 1-byte caches held as torch.uint8 or torch.float8_e4m3fn
FP8_TORCH = (torch.uint8, torch.float8_e4m3fn)
DEVICE_ERRORS = {0: "ok", 1: "block id out of range", 2: "slot out of range", 3: "copy pair conflict",
                 4: "bad context length", 5: "wait timeout"}


class PaError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {_lib.pa_status_string(status).decode()}")
        self.status = status


def library_path() -> str:
    return _LIB_PATH


def _check(status: int, where: str) -> None:
    if status != 0:
        raise PaError(status, where)


def _stream(stream: Optional[torch.cuda.Stream]) -> ctypes.c_void_p:
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _dev(t: torch.Tensor, name: str) -> int:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def _cache_args(k_cache: torch.Tensor, v_cache: torch.Tensor):
    if k_cache.dim() != 4 or k_cache.shape != v_cache.shape or k_cache.dtype != v_cache.dtype:
        raise ValueError("k_cache and v_cache must both be [num_blocks, block_size, num_kv_heads, head_dim]")
    if k_cache.dtype not in DTYPE_CODE and k_cache.dtype not in FP8_TORCH:
        raise ValueError(f"unsupported cache dtype {k_cache.dtype}")
    nb, bs, hkv, d = k_cache.shape
    return nb, bs, hkv, d, (FP8 if k_cache.dtype in FP8_TORCH else DTYPE_CODE[k_cache.dtype])


def reshape_and_cache(key: torch.Tensor, value: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                      slot_mapping: torch.Tensor, stream: Optional[torch.cuda.Stream] = None) -> None:
    """Write key/value rows [T, Hkv, D] into the caches at ``slot_mapping`` [T] (int64)."""
    nb, bs, hkv, d, dt = _cache_args(k_cache, v_cache)
    if key.dtype != k_cache.dtype or value.dtype != k_cache.dtype or slot_mapping.dtype != torch.int64:
        raise ValueError("key/value must have the cache dtype and slot_mapping must be int64")
    T = key.shape[0]
    if tuple(key.shape) != (T, hkv, d) or tuple(value.shape) != (T, hkv, d) or slot_mapping.numel() != T:
        raise ValueError("key/value must be [T, num_kv_heads, head_dim] with T slots")
    _check(_lib.pa_reshape_and_cache(_dev(key, "key"), _dev(value, "value"), _dev(k_cache, "k_cache"),
                                     _dev(v_cache, "v_cache"), _dev(slot_mapping, "slot_mapping") if T else None,
                                     T, nb, bs, hkv, d, dt, _stream(stream)), "pa_reshape_and_cache")


def decode_partition_size(num_seqs: int, num_heads: int, num_kv_heads: int, head_dim: int,
                          max_context_len: int, partition_size: int = 0) -> int:
    return int(_lib.pa_decode_partition_size(num_seqs, num_heads, num_kv_heads, head_dim, max_context_len,
                                             partition_size))


def decode_workspace_bytes(num_seqs: int, num_heads: int, num_kv_heads: int, head_dim: int,
                           max_context_len: int, partition_size: int = 0) -> int:
    return int(_lib.pa_decode_workspace_bytes(num_seqs, num_heads, num_kv_heads, head_dim, max_context_len,
                                              partition_size))


def decode(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, block_tables: torch.Tensor,
           context_lens: torch.Tensor, scale: float, out: Optional[torch.Tensor] = None, *,
           max_context_len: Optional[int] = None, partition_size: int = 0,
           workspace: Optional[torch.Tensor] = None,
           stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """Paged decode attention.  q [S, Hq, D]; block_tables [S, MBS] int32; context_lens [S] int32.

    ``max_context_len`` should be passed by callers that know it (reading it
    from ``context_lens`` costs a device-to-host sync).  ``workspace`` is
    allocated here when needed and not given.
    """
    nb, bs, hkv, d, dt = _cache_args(k_cache, v_cache)
    S, hq, dq = q.shape
    if dq != d or q.dtype != k_cache.dtype:
        raise ValueError("q must be [S, num_heads, head_dim] with the cache dtype")
    if block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32:
        raise ValueError("block_tables and context_lens must be int32")
    if block_tables.dim() != 2 or block_tables.shape[0] != S or context_lens.numel() != S:
        raise ValueError("block_tables must be [S, max_blocks_per_seq] and context_lens [S]")
    if out is None:
        out = torch.empty_like(q)
    elif out.shape != q.shape or out.dtype != q.dtype:
        raise ValueError("out must match q")
    if max_context_len is None:
        max_context_len = int(context_lens.max().item()) if S else 0
    need = decode_workspace_bytes(S, hq, hkv, d, max_context_len, partition_size)
    if need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_ptr = _dev(workspace, "workspace") if workspace is not None else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(_lib.pa_decode(_dev(out, "out"), _dev(q, "q"), _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"),
                          _dev(block_tables, "block_tables"), block_tables.shape[1],
                          _dev(context_lens, "context_lens"), S, hq, max_context_len, float(scale),
                          partition_size, ws_ptr, ws_bytes, nb, bs, hkv, d, dt, _stream(stream)), "pa_decode")
    return out


def decode_append(q: torch.Tensor, key: torch.Tensor, value: torch.Tensor, k_cache: torch.Tensor,
                  v_cache: torch.Tensor, block_tables: torch.Tensor, context_lens: torch.Tensor, scale: float,
                  out: Optional[torch.Tensor] = None, *, max_context_len: Optional[int] = None,
                  partition_size: int = 0, workspace: Optional[torch.Tensor] = None,
                  stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """Write each sequence's new token (key/value [S, Hkv, D]) at position
    context_len - 1 through its block table, then decode -- one launch."""
    nb, bs, hkv, d, dt = _cache_args(k_cache, v_cache)
    S, hq, dq = q.shape
    if dq != d or q.dtype != k_cache.dtype or key.dtype != k_cache.dtype or value.dtype != k_cache.dtype:
        raise ValueError("q, key and value must have the cache dtype and head_dim")
    if tuple(key.shape) != (S, hkv, d) or tuple(value.shape) != (S, hkv, d):
        raise ValueError("key/value must be [S, num_kv_heads, head_dim]")
    if block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32:
        raise ValueError("block_tables and context_lens must be int32")
    if block_tables.dim() != 2 or block_tables.shape[0] != S or context_lens.numel() != S:
        raise ValueError("block_tables must be [S, max_blocks_per_seq] and context_lens [S]")
    if out is None:
        out = torch.empty_like(q)
    elif out.shape != q.shape or out.dtype != q.dtype:
        raise ValueError("out must match q")
    if max_context_len is None:
        max_context_len = int(context_lens.max().item()) if S else 0
    need = decode_workspace_bytes(S, hq, hkv, d, max_context_len, partition_size)
    if need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_ptr = _dev(workspace, "workspace") if workspace is not None else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(_lib.pa_decode_append(_dev(out, "out"), _dev(q, "q"), _dev(key, "key"), _dev(value, "value"),
                                 _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"),
                                 _dev(block_tables, "block_tables"), block_tables.shape[1],
                                 _dev(context_lens, "context_lens"), S, hq, max_context_len, float(scale),
                                 partition_size, ws_ptr, ws_bytes, nb, bs, hkv, d, dt, _stream(stream)),
           "pa_decode_append")
    return out


def decode_static_workspace(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                            block_tables: torch.Tensor, context_lens: torch.Tensor, scale: float,
                            out: Optional[torch.Tensor] = None, *, max_context_len: int,
                            partition_size: int = 0, stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """``decode`` for callers that cannot allocate device memory: the split-K
    scratch is the library's own fixed array (STATIC_WORKSPACE_BYTES per GPU),
    so the library allocates nothing.  ``out`` must be given by such callers
    (it is allocated here only as a convenience when omitted).  Calls that
    overlap on the GPU share the array and race.  Every call that needs scratch
    looks up the array's address on the current device (the first lookup may
    load the library's device code there, so make the first call on each
    device before any stream capture)."""
    nb, bs, hkv, d, dt = _cache_args(k_cache, v_cache)
    S, hq, dq = q.shape
    if dq != d or q.dtype != k_cache.dtype:
        raise ValueError("q must be [S, num_heads, head_dim] with the cache dtype")
    if block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32:
        raise ValueError("block_tables and context_lens must be int32")
    if block_tables.dim() != 2 or block_tables.shape[0] != S or context_lens.numel() != S:
        raise ValueError("block_tables must be [S, max_blocks_per_seq] and context_lens [S]")
    if out is None:
        out = torch.empty_like(q)
    elif out.shape != q.shape or out.dtype != q.dtype:
        raise ValueError("out must match q")
    _check(_lib.pa_decode_static_workspace(
        _dev(out, "out"), _dev(q, "q"), _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"),
        _dev(block_tables, "block_tables"), block_tables.shape[1], _dev(context_lens, "context_lens"), S, hq,
        max_context_len, float(scale), partition_size, nb, bs, hkv, d, dt, _stream(stream)),
        "pa_decode_static_workspace")
    return out


def reshape_and_cache_fp8(key: torch.Tensor, value: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                          slot_mapping: torch.Tensor, k_scale: float, v_scale: float,
                          stream: Optional[torch.cuda.Stream] = None) -> None:
    """Quantise key/value rows [T, Hkv, 128] (fp16/bf16) into 1-byte E4M3 caches at their slots."""
    nb, bs, hkv, d, dt = _cache_args(k_cache, v_cache)
    if dt != FP8 or key.dtype not in (torch.float16, torch.bfloat16) or value.dtype != key.dtype:
        raise ValueError("1-byte caches and fp16/bf16 key/value expected")
    T = key.shape[0]
    if tuple(key.shape) != (T, hkv, d) or tuple(value.shape) != (T, hkv, d) or slot_mapping.numel() != T:
        raise ValueError("key/value must be [T, num_kv_heads, head_dim] with T slots")
    if slot_mapping.dtype != torch.int64:
        raise ValueError("slot_mapping must be int64")
    _check(_lib.pa_reshape_and_cache_fp8(_dev(key, "key"), _dev(value, "value"), _dev(k_cache, "k_cache"),
                                         _dev(v_cache, "v_cache"),
                                         _dev(slot_mapping, "slot_mapping") if T else None, T, nb, bs, hkv, d,
                                         DTYPE_CODE[key.dtype], float(k_scale), float(v_scale), _stream(stream)),
           "pa_reshape_and_cache_fp8")


def decode_fp8(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, k_scale: float, v_scale: float,
               block_tables: torch.Tensor, context_lens: torch.Tensor, scale: float,
               out: Optional[torch.Tensor] = None, *, max_context_len: Optional[int] = None,
               partition_size: int = 0, workspace: Optional[torch.Tensor] = None,
               stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """Paged decode over 1-byte E4M3 caches; q/out fp16 or bf16."""
    nb, bs, hkv, d, dt = _cache_args(k_cache, v_cache)
    S, hq, dq = q.shape
    if dt != FP8 or q.dtype not in (torch.float16, torch.bfloat16) or dq != d:
        raise ValueError("1-byte caches and fp16/bf16 q [S, Hq, head_dim] expected")
    if block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32:
        raise ValueError("block_tables and context_lens must be int32")
    if block_tables.dim() != 2 or block_tables.shape[0] != S or context_lens.numel() != S:
        raise ValueError("block_tables must be [S, max_blocks_per_seq] and context_lens [S]")
    if out is None:
        out = torch.empty_like(q)
    elif out.shape != q.shape or out.dtype != q.dtype:
        raise ValueError("out must match q")
    if max_context_len is None:
        max_context_len = int(context_lens.max().item()) if S else 0
    need = decode_workspace_bytes(S, hq, hkv, d, max_context_len, partition_size)
    if need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_ptr = _dev(workspace, "workspace") if workspace is not None else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(_lib.pa_decode_fp8(_dev(out, "out"), _dev(q, "q"), _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"),
                              float(k_scale), float(v_scale), _dev(block_tables, "block_tables"),
                              block_tables.shape[1], _dev(context_lens, "context_lens"), S, hq, max_context_len,
                              float(scale), partition_size, ws_ptr, ws_bytes, nb, bs, hkv, d, DTYPE_CODE[q.dtype],
                              _stream(stream)), "pa_decode_fp8")
    return out


def prefill(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, block_tables: torch.Tensor,
            context_lens: torch.Tensor, query_start_loc: torch.Tensor, scale: float,
            out: Optional[torch.Tensor] = None, *, max_query_len: Optional[int] = None,
            stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """Paged chunked-prefill attention.  q [T, Hq, 128]; sequence b's chunk is rows
    query_start_loc[b]:query_start_loc[b+1] (int32 [S+1]), the last tokens of its
    context_lens[b] cached tokens.  ``max_query_len`` (the longest chunk) should be
    passed by callers that know it; reading it here costs a device-to-host sync."""
    nb, bs, hkv, d, dt = _cache_args(k_cache, v_cache)
    T, hq, dq = q.shape
    if dq != d or q.dtype != k_cache.dtype:
        raise ValueError("q must be [T, num_heads, head_dim] with the cache dtype")
    if block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32 or query_start_loc.dtype != torch.int32:
        raise ValueError("block_tables, context_lens and query_start_loc must be int32")
    S = context_lens.numel()
    if block_tables.dim() != 2 or block_tables.shape[0] != S or query_start_loc.numel() != S + 1:
        raise ValueError("block_tables must be [S, MBS] and query_start_loc [S + 1]")
    if max_query_len is None:
        qsl = query_start_loc.cpu()
        max_query_len = int((qsl[1:] - qsl[:-1]).max()) if S else 0
    if out is None:
        out = torch.empty_like(q)
    elif out.shape != q.shape or out.dtype != q.dtype:
        raise ValueError("out must match q")
    _check(_lib.pa_prefill(_dev(out, "out"), _dev(q, "q"), _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"),
                           _dev(block_tables, "block_tables"), block_tables.shape[1],
                           _dev(context_lens, "context_lens"), _dev(query_start_loc, "query_start_loc"), S, hq,
                           int(max_query_len), float(scale), nb, bs, hkv, d, dt, _stream(stream)), "pa_prefill")
    return out


def copy_blocks(k_cache: torch.Tensor, v_cache: torch.Tensor, block_mapping: torch.Tensor,
                stream: Optional[torch.cuda.Stream] = None) -> None:
    """Copy whole blocks (src, dst) = block_mapping[i] ([P, 2] int64) in both caches."""
    nb, bs, hkv, d, dt = _cache_args(k_cache, v_cache)
    if block_mapping.dtype != torch.int64 or (block_mapping.numel() and block_mapping.shape[-1] != 2):
        raise ValueError("block_mapping must be [P, 2] int64")
    P = block_mapping.numel() // 2
    _check(_lib.pa_copy_blocks(_dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"),
                               _dev(block_mapping, "block_mapping") if P else None, P, nb, bs, hkv, d, dt,
                               _stream(stream)), "pa_copy_blocks")


def stream_read(buf: torch.Tensor, sink: torch.Tensor, stream: Optional[torch.cuda.Stream] = None) -> None:
    """Read every byte of ``buf`` once (a plain streaming read, for measuring the
    read-only bandwidth); XORs its 8-byte words into ``sink`` (one int64 on the device)."""
    if sink.dtype != torch.int64 or sink.numel() != 1:
        raise ValueError("sink must be one int64")
    _check(_lib.pa_stream_read(_dev(buf, "buf"), buf.numel() * buf.element_size(), _dev(sink, "sink"),
                               _stream(stream)), "pa_stream_read")


def test_stall_next_launch(kernel: str, cta: int) -> None:
    """Test hook: the next launch of ``kernel`` ("decode" or "prefill") leaves
    one copy of CTA ``cta`` unissued, so that CTA's bounded wait runs out
    (PA_DEV_WAIT_TIMEOUT, detail = cta) within about a millisecond; ``cta=-1``
    disarms."""
    _check(_lib.pa_test_stall_next_launch({"decode": 0, "prefill": 1}[kernel], int(cta)),
           "pa_test_stall_next_launch")


def get_device_error(clear: bool = True, stream: Optional[torch.cuda.Stream] = None):
    """(kind, detail) of the first problem a kernel recorded on the current device."""
    detail = _I64(0)
    code = _lib.pa_get_device_error(_stream(stream), ctypes.byref(detail), 1 if clear else 0)
    if code < 0:
        raise PaError(5, "pa_get_device_error")
    return code, int(detail.value)


# -- raw entry points for callers that manage pointers themselves -----------------
raw = _lib
