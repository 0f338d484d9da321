"""Paged MLA decode attention for B200 (sm_100a): Python binding of the C ABI.

Every call here only marshals arguments (torch tensors -> device pointers,
current CUDA stream) and forwards them to ``libmla_decode.so``; all arithmetic
runs in the library's CUDA kernels.  The names and arguments mirror
``include/mla_decode.h``.  There is no fallback: if the library is missing or a
call fails, an exception is raised.

Typical use::

    parts = mla_get_num_sm_parts(s_q * h_q)
    meta, num_splits = mla_get_metadata(cache_seqlens, s_q * h_q, parts)
    ws = alloc_workspace(batch, s_q * h_q, parts)
    out, lse = mla_decode_fwd(q, kcache, block_table, cache_seqlens, 576 ** -0.5, False,
                              meta, num_splits, ws)

A cache of dtype ``torch.uint8`` or ``torch.float8_e5m2`` holds e5m2 values (one byte each); the
call then passes the base dtype of q with ``KV_FP8_E5M2`` (include/mla_decode.h), and partition
counts come from ``mla_get_num_sm_parts(rows, kv_fp8=True)``.
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

__all__ = [
    "MlaError",
    "lib",
    "library_path",
    "mla_version",
    "mla_get_num_sm_parts",
    "KV_FP8_E5M2",
    "mla_get_workspace_size",
    "alloc_workspace",
    "mla_get_metadata",
    "mla_decode_fwd",
    "mla_splitkv_fwd",
    "mla_combine_fwd",
    "mla_append_kv",
    "mla_decode_fwd_append",
    "mla_read_device_status",
    "mla_set_kernel_variant",
    "mla_get_kernel_variant",
    "KERNEL_VARIANTS",
    "HEAD_DIM_K",
    "HEAD_DIM_V",
    "PAGE_SIZE",
    "META_INTS",
]

HEAD_DIM_K = 576
HEAD_DIM_V = 512
PAGE_SIZE = 64
META_INTS = 8
_DTYPES = {torch.bfloat16: 0, torch.float16: 1}
KV_FP8_E5M2 = 0x100  # OR-ed into the dtype code: the cache holds e5m2 bytes
_FP8_CACHE = (torch.uint8, torch.float8_e5m2)
# split-KV kernel variants (include/mla_decode.h, MLA_KERNEL_*)
KERNEL_VARIANTS = {"auto": 0, "few-rows-one-cta": 1, "few-rows-pair": 2, "row-tile-pair": 3}

library_path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmla_decode.so")


class MlaError(RuntimeError):
    pass


def _load() -> ctypes.CDLL:
    if not os.path.exists(library_path):
        raise ImportError(
            f"{library_path} is not built; run `python -m mla_decode_attention_16_b200.build` "
            "(needs nvcc with sm_100a support)")
    L = ctypes.CDLL(library_path)
    c_int, c_i64, c_sz, c_f, vp = ctypes.c_int, ctypes.c_int64, ctypes.c_size_t, ctypes.c_float, ctypes.c_void_p
    L.mla_status_string.restype = ctypes.c_char_p
    L.mla_status_string.argtypes = [c_int]
    L.mla_last_cuda_error.restype = c_int
    L.mla_version.restype = c_int
    L.mla_get_num_sm_parts.argtypes = [c_int, c_int, ctypes.POINTER(c_int)]
    L.mla_get_num_sm_parts_dtype.argtypes = [c_int, c_int, c_int, ctypes.POINTER(c_int)]
    L.mla_get_workspace_size.argtypes = [c_int, c_int, c_int, ctypes.POINTER(c_sz)]
    L.mla_get_metadata.argtypes = [vp, c_int, c_int, c_int, vp, vp, vp]
    fwd = [vp, vp, c_i64, vp, c_i64, vp, c_int, c_int, c_int, c_int, c_f, c_int, vp, vp, c_int, vp, c_sz, vp, vp, vp]
    L.mla_decode_fwd.argtypes = fwd
    L.mla_splitkv_fwd.argtypes = fwd
    L.mla_combine_fwd.argtypes = [vp, c_int, c_int, c_int, c_int, vp, c_int, vp, c_sz, vp, vp, vp]
    L.mla_read_device_status.argtypes = [vp, vp, ctypes.POINTER(ctypes.c_int32)]
    L.mla_append_kv.argtypes = [vp, vp, c_i64, vp, c_i64, vp, c_int, c_int, c_int, vp, c_sz, vp]
    L.mla_decode_fwd_append.argtypes = [vp, vp, vp, c_i64, vp, c_i64, vp, c_int, c_int, c_int, c_int, c_f, c_int,
                                        vp, vp, c_int, vp, c_sz, vp, vp, vp]
    L.mla_set_kernel_variant.argtypes = [c_int]
    L.mla_get_kernel_variant.argtypes = [c_int]
    L.mla_get_kernel_variant.restype = c_int
    for name in ("mla_set_kernel_variant", "mla_get_num_sm_parts", "mla_get_num_sm_parts_dtype", "mla_get_workspace_size", "mla_get_metadata", "mla_decode_fwd",
                 "mla_splitkv_fwd", "mla_combine_fwd", "mla_read_device_status", "mla_append_kv",
                 "mla_decode_fwd_append"):
        getattr(L, name).restype = c_int
    return L


lib = _load()


def _check(rc: int, what: str) -> None:
    if rc != 0:
        extra = ""
        if rc == 4:
            extra = f" (cudaError {lib.mla_last_cuda_error()})"
        raise MlaError(f"{what}: {lib.mla_status_string(rc).decode()}{extra}")


def _stream(stream, device) -> int:
    if stream is None:
        return torch.cuda.current_stream(device).cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def mla_version() -> int:
    return lib.mla_version()


def mla_get_num_sm_parts(rows: int, device: Optional[int] = None, kv_fp8: bool = False) -> int:
    """Scheduler partitions for s_q * h_q = rows (kv_fp8: for an e5m2 cache)."""
    dev = torch.cuda.current_device() if device is None else int(device)
    out = ctypes.c_int(0)
    if kv_fp8:
        _check(lib.mla_get_num_sm_parts_dtype(dev, int(rows), KV_FP8_E5M2, ctypes.byref(out)),
               "mla_get_num_sm_parts_dtype")
    else:
        _check(lib.mla_get_num_sm_parts(dev, int(rows), ctypes.byref(out)), "mla_get_num_sm_parts")
    return out.value


def _cache_code(kcache: torch.Tensor, base: torch.dtype) -> int:
    """dtype code of a call whose 16-bit tensors are `base` and whose cache is kcache."""
    return _DTYPES[base] | (KV_FP8_E5M2 if kcache.dtype in _FP8_CACHE else 0)


def mla_get_workspace_size(batch: int, rows: int, num_sm_parts: int) -> int:
    out = ctypes.c_size_t(0)
    _check(lib.mla_get_workspace_size(int(batch), int(rows), int(num_sm_parts), ctypes.byref(out)),
           "mla_get_workspace_size")
    return out.value


def alloc_workspace(batch: int, rows: int, num_sm_parts: int, device=None) -> torch.Tensor:
    """Zeroed device workspace of the size the library asks for."""
    n = mla_get_workspace_size(batch, rows, num_sm_parts)
    return torch.zeros(n, dtype=torch.uint8, device=device if device is not None else "cuda")


def _need(t: torch.Tensor, name: str, dtype=None, dim=None) -> None:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise MlaError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise MlaError(f"{name} must be {dtype}, got {t.dtype}")
    if dim is not None and t.dim() != dim:
        raise MlaError(f"{name} must have {dim} dims, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise MlaError(f"{name} must be contiguous")


def mla_get_metadata(cache_seqlens: torch.Tensor, rows: int, num_sm_parts: Optional[int] = None,
                     tile_sched_metadata: Optional[torch.Tensor] = None, num_splits: Optional[torch.Tensor] = None,
                     stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Tile-scheduler metadata: ([num_sm_parts, 8] int32, [batch + 1] int32)."""
    _need(cache_seqlens, "cache_seqlens", torch.int32, 1)
    dev = cache_seqlens.device
    if num_sm_parts is None:
        num_sm_parts = mla_get_num_sm_parts(rows, dev.index)
    b = cache_seqlens.shape[0]
    if tile_sched_metadata is None:
        tile_sched_metadata = torch.empty(num_sm_parts, META_INTS, dtype=torch.int32, device=dev)
    if num_splits is None:
        num_splits = torch.empty(b + 1, dtype=torch.int32, device=dev)
    _need(tile_sched_metadata, "tile_sched_metadata", torch.int32)
    _need(num_splits, "num_splits", torch.int32, 1)
    if tile_sched_metadata.numel() < num_sm_parts * META_INTS or num_splits.numel() < b + 1:
        raise MlaError("metadata buffers too small")
    _check(lib.mla_get_metadata(_ptr(cache_seqlens), b, int(rows), int(num_sm_parts), _ptr(tile_sched_metadata),
                                _ptr(num_splits), _stream(stream, dev)), "mla_get_metadata")
    return tile_sched_metadata, num_splits


def _fwd_args(q, kcache, block_table, cache_seqlens, softmax_scale, causal, tile_sched_metadata, num_splits,
              workspace, out, lse, stream):
    _need(q, "q", dim=4)
    if q.dtype not in _DTYPES:
        raise MlaError(f"q must be bf16 or fp16, got {q.dtype}")
    b, s_q, h_q, dk = q.shape
    if dk != HEAD_DIM_K:
        raise MlaError(f"q last dim must be {HEAD_DIM_K}")
    _need(kcache, "kcache", None if kcache.dtype in _FP8_CACHE else q.dtype, 4)
    if tuple(kcache.shape[1:]) != (PAGE_SIZE, 1, HEAD_DIM_K):
        raise MlaError(f"kcache must be [pages, {PAGE_SIZE}, 1, {HEAD_DIM_K}], got {tuple(kcache.shape)}")
    _need(block_table, "block_table", torch.int32, 2)
    _need(cache_seqlens, "cache_seqlens", torch.int32, 1)
    _need(tile_sched_metadata, "tile_sched_metadata", torch.int32)
    _need(num_splits, "num_splits", torch.int32, 1)
    if block_table.shape[0] != b or cache_seqlens.shape[0] != b or num_splits.shape[0] != b + 1:
        raise MlaError("batch sizes of q, block_table, cache_seqlens and num_splits disagree")
    parts = tile_sched_metadata.numel() // META_INTS
    rows = s_q * h_q
    if workspace is None:
        workspace = alloc_workspace(b, rows, parts, q.device)
    _need(workspace, "workspace", torch.uint8, 1)
    if out is None:
        out = torch.empty(b, s_q, h_q, HEAD_DIM_V, dtype=q.dtype, device=q.device)
    if lse is None:
        lse = torch.empty(b, h_q, s_q, dtype=torch.float32, device=q.device)
    _need(out, "out", q.dtype, 4)
    _need(lse, "lse", torch.float32, 3)
    if tuple(out.shape) != (b, s_q, h_q, HEAD_DIM_V) or tuple(lse.shape) != (b, h_q, s_q):
        raise MlaError("out / lse shapes do not match q")
    args = (_ptr(q), _ptr(kcache), kcache.shape[0], _ptr(block_table), block_table.stride(0), _ptr(cache_seqlens),
            b, s_q, h_q, _cache_code(kcache, q.dtype), float(softmax_scale), 1 if causal else 0, _ptr(tile_sched_metadata),
            _ptr(num_splits), parts, _ptr(workspace), workspace.numel(), _ptr(out), _ptr(lse),
            _stream(stream, q.device))
    return args, out, lse


def mla_decode_fwd(q, kcache, block_table, cache_seqlens, softmax_scale, causal, tile_sched_metadata, num_splits,
                   workspace=None, out=None, lse=None, stream=None):
    """out [b, s_q, h_q, 512] (q's dtype) and lse [b, h_q, s_q] fp32."""
    args, out, lse = _fwd_args(q, kcache, block_table, cache_seqlens, softmax_scale, causal, tile_sched_metadata,
                               num_splits, workspace, out, lse, stream)
    _check(lib.mla_decode_fwd(*args), "mla_decode_fwd")
    return out, lse


def mla_splitkv_fwd(q, kcache, block_table, cache_seqlens, softmax_scale, causal, tile_sched_metadata, num_splits,
                    workspace, out=None, lse=None, stream=None):
    """First stage only (split-KV kernel); see include/mla_decode.h."""
    args, out, lse = _fwd_args(q, kcache, block_table, cache_seqlens, softmax_scale, causal, tile_sched_metadata,
                               num_splits, workspace, out, lse, stream)
    _check(lib.mla_splitkv_fwd(*args), "mla_splitkv_fwd")
    return out, lse


def mla_combine_fwd(cache_seqlens, s_q, h_q, dtype, num_splits, num_sm_parts, workspace, out, lse, stream=None):
    """Second stage only (log-sum-exp combine); see include/mla_decode.h."""
    _need(cache_seqlens, "cache_seqlens", torch.int32, 1)
    _need(workspace, "workspace", torch.uint8, 1)
    b = cache_seqlens.shape[0]
    _check(lib.mla_combine_fwd(_ptr(cache_seqlens), b, int(s_q), int(h_q), _DTYPES[dtype], _ptr(num_splits),
                               int(num_sm_parts), _ptr(workspace), workspace.numel(), _ptr(out), _ptr(lse),
                               _stream(stream, cache_seqlens.device)), "mla_combine_fwd")
    return out, lse


def _check_kv_new(kv_new, kcache, block_table):
    _need(kv_new, "kv_new", None if kcache.dtype in _FP8_CACHE else kcache.dtype, 3)
    if kv_new.dtype not in _DTYPES:
        raise MlaError(f"kv_new must be bf16 or fp16, got {kv_new.dtype}")
    if kv_new.shape[0] != block_table.shape[0] or kv_new.shape[2] != HEAD_DIM_K:
        raise MlaError(f"kv_new must be [batch, s_q, {HEAD_DIM_K}], got {tuple(kv_new.shape)}")


def mla_append_kv(kv_new, kcache, block_table, cache_seqlens, workspace, stream=None):
    """Write kv_new [b, s_q, 576] into the cache at positions L_b - s_q + s (in place); see
    include/mla_decode.h.  Returns kcache."""
    _need(kcache, "kcache", dim=4)
    if kcache.dtype not in _DTYPES and kcache.dtype not in _FP8_CACHE:
        raise MlaError(f"kcache must be bf16, fp16 or e5m2 bytes, got {kcache.dtype}")
    _need(block_table, "block_table", torch.int32, 2)
    _need(cache_seqlens, "cache_seqlens", torch.int32, 1)
    _need(workspace, "workspace", torch.uint8, 1)
    _check_kv_new(kv_new, kcache, block_table)
    b, s_q, _ = kv_new.shape
    _check(lib.mla_append_kv(_ptr(kv_new), _ptr(kcache), kcache.shape[0], _ptr(block_table), block_table.stride(0),
                             _ptr(cache_seqlens), b, s_q, _cache_code(kcache, kv_new.dtype), _ptr(workspace),
                             workspace.numel(),
                             _stream(stream, kcache.device)), "mla_append_kv")
    return kcache


def mla_decode_fwd_append(q, kv_new, kcache, block_table, cache_seqlens, softmax_scale, causal,
                          tile_sched_metadata, num_splits, workspace=None, out=None, lse=None, stream=None):
    """The decode step fused with the append of kv_new [b, s_q, 576] (kcache is written first);
    returns out [b, s_q, h_q, 512] and lse [b, h_q, s_q]."""
    args, out, lse = _fwd_args(q, kcache, block_table, cache_seqlens, softmax_scale, causal, tile_sched_metadata,
                               num_splits, workspace, out, lse, stream)
    _check_kv_new(kv_new, kcache, block_table)
    if kv_new.shape[1] != q.shape[1]:
        raise MlaError("kv_new and q must have the same s_q")
    if kv_new.dtype != q.dtype:
        raise MlaError("kv_new and q must have the same dtype")
    _check(lib.mla_decode_fwd_append(args[0], _ptr(kv_new), *args[1:]), "mla_decode_fwd_append")
    return out, lse


def mla_set_kernel_variant(variant) -> None:
    """Process-wide split-KV kernel choice: a name of KERNEL_VARIANTS or its number.  Partition
    counts depend on it: query mla_get_num_sm_parts / mla_get_metadata again afterwards."""
    v = KERNEL_VARIANTS[variant] if isinstance(variant, str) else int(variant)
    _check(lib.mla_set_kernel_variant(v), "mla_set_kernel_variant")


def mla_get_kernel_variant(rows: int) -> Optional[str]:
    """Name of the variant a call with s_q * h_q = rows runs now (None if none can)."""
    v = lib.mla_get_kernel_variant(int(rows))
    return {n: k for k, n in KERNEL_VARIANTS.items()}.get(v)


def mla_read_device_status(workspace: torch.Tensor, stream=None) -> Tuple[int, int]:
    """(error bits, first offending page index) from the workspace header; synchronises."""
    flags = (ctypes.c_int32 * 2)()
    _check(lib.mla_read_device_status(_ptr(workspace), _stream(stream, workspace.device), flags),
           "mla_read_device_status")
    return int(flags[0]), int(flags[1])
