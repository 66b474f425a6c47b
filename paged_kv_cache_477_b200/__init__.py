"""paged_kv_cache_477_b200 -- attention over a block-paged KV cache on B200.

Thin ctypes binding of ``libpagedkv.so`` (include/pagedkv.h).  This module only
marshals arguments: it checks tensor dtypes/devices/shapes, passes raw device
pointers and the current CUDA stream, and turns status codes into exceptions.
Every step of the computation runs in the library's sm_100a kernels; there is
no CPU or PyTorch fallback, and calling anything without the built library
raises.

Calls (same names as the C ABI):
    kv_cache_write(key, value, k_cache, v_cache, slot_mapping)
    paged_attention(q, k_cache, v_cache, block_tables, context_lens, scale, ...)
    paged_attention_split(..., pages_per_split)
    paged_attention_prefill(q, query_start_loc, k_cache, v_cache, block_tables,
                            context_lens, scale, max_q_len, ...)
    kv_cache_write_rope(key, value, k_cache, v_cache, slot_mapping, positions, rope_base)
    kv_cache_write_int8(key, value, k_cache, v_cache, k_scale, v_scale, slot_mapping)
    paged_attention_int8(q, k_cache, v_cache, k_scale, v_scale, block_tables,
                         context_lens, scale, ...)
    paged_attention_window(q, k_cache, v_cache, block_tables, context_lens, scale, window, ...)
    paged_attention_prefill_window(q, query_start_loc, k_cache, v_cache, block_tables,
                                   context_lens, scale, max_q_len, window, ...)
    paged_attention_int8_window(q, k_cache, v_cache, k_scale, v_scale, block_tables,
                                context_lens, scale, window, ...)
    copy_blocks(k_cache, v_cache, pairs);  BlockAllocator(num_blocks)
    hbm_read_probe(buf, sink, chunk_bytes)      (measurement utility)
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpagedkv.so")

PKV_BF16 = 0
STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported configuration", 3: "CUDA error",
          4: "device wait timed out", 5: "index out of range on the device",
          6: "workspace missing or too small", 7: "not enough free blocks"}

_lib = None

_P = ctypes.c_void_p
_I32 = ctypes.c_int32
_I64 = ctypes.c_int64
_F32 = ctypes.c_float
_SZ = ctypes.c_size_t

EXPORTS = {
    "pkv_kv_cache_write": ([_P, _P, _I64, _I64, _P, _P, _P, _I32, _I32, _I32, _I32, _I32, _I32, _P], _I32),
    "pkv_paged_attention": ([_P, _P, _P, _P, _P, _I32, _P, _I32, _I32, _I32, _I32, _I32, _I32, _F32,
                             _I32, _P, _SZ, _I32, _P], _I32),
    "pkv_paged_attention_workspace_size": ([_I32, _I32, _I32, _I32, _I32, _I32, _I32], _SZ),
    "pkv_paged_attention_split": ([_P, _P, _P, _P, _P, _I32, _P, _I32, _I32, _I32, _I32, _I32, _I32,
                                   _F32, _I32, _I32, _P, _SZ, _I32, _P], _I32),
    "pkv_split_workspace_size": ([_I32, _I32, _I32, _I32], _SZ),
    "pkv_paged_attention_split_noalloc": ([_P, _P, _P, _P, _P, _I32, _P, _I32, _I32, _I32, _I32, _I32,
                                           _I32, _F32, _I32, _I32, _I32, _P], _I32),
    "pkv_kv_cache_write_rope": ([_P, _P, _I64, _I64, _P, _P, _P, _P, _I32, _I32, _I32, _I32, _I32,
                                 ctypes.c_double, _I32, _P], _I32),
    "pkv_kv_cache_write_int8": ([_P, _P, _I64, _I64, _P, _P, _P, _P, _P, _I32, _I32, _I32, _I32, _I32, _P], _I32),
    "pkv_paged_attention_int8": ([_P, _P, _P, _P, _P, _P, _P, _I32, _P, _I32, _I32, _I32, _I32, _I32, _I32, _F32,
                                  _I32, _P, _SZ, _P], _I32),
    "pkv_paged_attention_int8_window": ([_P, _P, _P, _P, _P, _P, _P, _I32, _P, _I32, _I32, _I32, _I32, _I32, _I32,
                                         _F32, _I32, _P, _SZ, _P], _I32),
    "pkv_paged_attention_window": ([_P, _P, _P, _P, _P, _I32, _P, _I32, _I32, _I32, _I32, _I32, _I32, _F32,
                                    _I32, _P, _SZ, _I32, _P], _I32),
    "pkv_paged_attention_window_workspace_size": ([_I32, _I32, _I32, _I32, _I32, _I32, _I32], _SZ),
    "pkv_paged_attention_prefill": ([_P, _P, _P, _P, _P, _P, _I32, _P, _I32, _I32, _I32, _I32, _I32,
                                     _I32, _I32, _I32, _F32, _I32, _P], _I32),
    "pkv_paged_attention_prefill_window": ([_P, _P, _P, _P, _P, _P, _I32, _P, _I32, _I32, _I32, _I32, _I32,
                                            _I32, _I32, _I32, _F32, _I32, _I32, _P], _I32),
    "pkv_block_allocator_create": ([_I32, ctypes.POINTER(_P)], _I32),
    "pkv_block_allocator_destroy": ([_P], None),
    "pkv_block_allocator_alloc": ([_P, _I32, _P], _I32),
    "pkv_block_allocator_share": ([_P, _P, _I32], _I32),
    "pkv_block_allocator_release": ([_P, _P, _I32], _I32),
    "pkv_block_allocator_cow": ([_P, _I32, ctypes.POINTER(_I32), ctypes.POINTER(_I32)], _I32),
    "pkv_block_allocator_num_free": ([_P], _I32),
    "pkv_block_allocator_refcount": ([_P, _I32], _I32),
    "pkv_copy_blocks": ([_P, _P, _SZ, _P, _I32, _I32, _P], _I32),
    "pkv_hbm_read_probe": ([_P, _SZ, _I32, _P, _I32, _P], _I32),
    "pkv_get_device_error": ([_P, ctypes.POINTER(_I32)], _I32),
    "pkv_last_launch_count": ([], _I32),
    "pkv_status_string": ([_I32], ctypes.c_char_p),
    "pkv_selftest_wait_timeout": ([ctypes.c_uint32, _P], _I32),
}


class PagedKVError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {STATUS.get(status, status)} (status {status})")
        self.status = status


def load_library(path: Optional[str] = None) -> ctypes.CDLL:
    """Load libpagedkv.so (raises if it has not been built)."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise RuntimeError(f"{p} is missing: build it with `python -m paged_kv_cache_477_b200.build` "
                           "(nvcc, sm_100a); there is no fallback path")
    lib = ctypes.CDLL(p)
    for name, (args, res) in EXPORTS.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    if path is None:
        _lib = lib
    return lib


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _check(rc: int, what: str):
    if rc != 0:
        raise PagedKVError(rc, what)


def _dev(t: torch.Tensor, name: str, dtype=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    return t


def _contig(t: torch.Tensor, name: str):
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def _cache_dims(k_cache, v_cache):
    _dev(k_cache, "k_cache", torch.bfloat16)
    _dev(v_cache, "v_cache", torch.bfloat16)
    _contig(k_cache, "k_cache")
    _contig(v_cache, "v_cache")
    if k_cache.dim() != 4 or k_cache.shape != v_cache.shape:
        raise ValueError("k_cache/v_cache must both be [num_blocks, num_kv_heads, block_size, head_dim]")
    return k_cache.shape


def kv_cache_write(key, value, k_cache, v_cache, slot_mapping, stream=None) -> None:
    """Scatter key/value [T, Hkv, D] into k_cache/v_cache at slot_mapping [T] (int64)."""
    NB, Hkv, bs, D = _cache_dims(k_cache, v_cache)
    _dev(key, "key", torch.bfloat16)
    _dev(value, "value", torch.bfloat16)
    _dev(slot_mapping, "slot_mapping", torch.int64)
    _contig(slot_mapping, "slot_mapping")
    T = key.shape[0]
    for t, nm in ((key, "key"), (value, "value")):
        if t.dim() != 3 or t.shape[1] != Hkv or t.shape[2] != D or t.stride(2) != 1 or t.stride(1) != D:
            raise ValueError(f"{nm} must be [T, Hkv, D] with contiguous heads")
    if value.shape[0] != T or slot_mapping.numel() != T:
        raise ValueError("key, value and slot_mapping disagree on T")
    rc = load_library().pkv_kv_cache_write(key.data_ptr(), value.data_ptr(), key.stride(0),
                                           value.stride(0), k_cache.data_ptr(), v_cache.data_ptr(),
                                           slot_mapping.data_ptr(), T, Hkv, D, NB, bs, PKV_BF16,
                                           _stream(stream))
    _check(rc, "kv_cache_write")


def _decode_common(q, k_cache, v_cache, block_tables, context_lens, out):
    NB, Hkv, bs, D = _cache_dims(k_cache, v_cache)
    _contig(_dev(q, "q", torch.bfloat16), "q")
    _contig(_dev(block_tables, "block_tables", torch.int32), "block_tables")
    _contig(_dev(context_lens, "context_lens", torch.int32), "context_lens")
    if q.dim() != 3 or q.shape[2] != D:
        raise ValueError("q must be [B, Hq, D]")
    B, Hq, _ = q.shape
    if block_tables.dim() != 2 or block_tables.shape[0] != B or context_lens.numel() != B:
        raise ValueError("block_tables must be [B, MB] and context_lens [B]")
    if out is None:
        out = torch.empty_like(q)
    else:
        _contig(_dev(out, "out", torch.bfloat16), "out")
        if out.shape != q.shape:
            raise ValueError("out must have q's shape")
    return NB, Hkv, bs, D, B, Hq, block_tables.shape[1], out


def kv_cache_write_rope(key, value, k_cache, v_cache, slot_mapping, positions, rope_base: float,
                        stream=None) -> None:
    """Cache write with K rotated by RoPE at ``positions`` [T] (int64) on the way in."""
    for t, name in ((key, "key"), (value, "value")):
        _dev(t, name, torch.bfloat16)
        if t.dim() != 3 or t.stride(2) != 1 or t.stride(1) != t.shape[2]:
            raise ValueError(f"{name} must be [T, Hkv, D] with contiguous (head, dim)")
    NB, Hkv, bs, D = _cache_dims(k_cache, v_cache)
    _contig(_dev(slot_mapping, "slot_mapping", torch.int64), "slot_mapping")
    _contig(_dev(positions, "positions", torch.int64), "positions")
    T = key.shape[0]
    if key.shape[1:] != (Hkv, D) or value.shape != key.shape or slot_mapping.numel() != T \
            or positions.numel() != T:
        raise ValueError("shape mismatch between key/value, caches, slot_mapping and positions")
    rc = load_library().pkv_kv_cache_write_rope(
        key.data_ptr(), value.data_ptr(), key.stride(0), value.stride(0), k_cache.data_ptr(), v_cache.data_ptr(),
        slot_mapping.data_ptr(), positions.data_ptr(), T, Hkv, D, NB, bs, float(rope_base), PKV_BF16,
        _stream(stream))
    _check(rc, "kv_cache_write_rope")


def kv_cache_write_int8(key, value, k_cache, v_cache, k_scale, v_scale, slot_mapping, stream=None) -> None:
    """Quantise key/value [T, Hkv, D] (bf16, rows may be strided) into the int8
    cache k_cache/v_cache [NB, Hkv, bs, D] and its fp32 row scales [NB, Hkv, bs]."""
    for t, name in ((key, "key"), (value, "value")):
        _dev(t, name, torch.bfloat16)
        if t.dim() != 3 or t.stride(2) != 1 or t.stride(1) != t.shape[2]:
            raise ValueError(f"{name} must be [T, Hkv, D] with contiguous (head, dim)")
    for t, name in ((k_cache, "k_cache"), (v_cache, "v_cache")):
        _contig(_dev(t, name, torch.int8), name)
    for t, name in ((k_scale, "k_scale"), (v_scale, "v_scale")):
        _contig(_dev(t, name, torch.float32), name)
    _contig(_dev(slot_mapping, "slot_mapping", torch.int64), "slot_mapping")
    T, Hkv, D = key.shape
    NB, Hkv2, bs, D2 = k_cache.shape
    if (Hkv2, D2) != (Hkv, D) or value.shape != key.shape or v_cache.shape != k_cache.shape \
            or k_scale.shape != (NB, Hkv, bs) or v_scale.shape != k_scale.shape or slot_mapping.numel() != T:
        raise ValueError("shape mismatch between key/value, caches, scales and slot_mapping")
    rc = load_library().pkv_kv_cache_write_int8(
        key.data_ptr(), value.data_ptr(), key.stride(0), value.stride(0), k_cache.data_ptr(),
        v_cache.data_ptr(), k_scale.data_ptr(), v_scale.data_ptr(), slot_mapping.data_ptr(), T, Hkv, D, NB, bs,
        _stream(stream))
    _check(rc, "kv_cache_write_int8")


def _int8_common(q, k_cache, v_cache, k_scale, v_scale, block_tables, context_lens, out):
    for t, name in ((k_cache, "k_cache"), (v_cache, "v_cache")):
        _contig(_dev(t, name, torch.int8), name)
    for t, name in ((k_scale, "k_scale"), (v_scale, "v_scale")):
        _contig(_dev(t, name, torch.float32), name)
    _contig(_dev(q, "q", torch.bfloat16), "q")
    _contig(_dev(block_tables, "block_tables", torch.int32), "block_tables")
    _contig(_dev(context_lens, "context_lens", torch.int32), "context_lens")
    NB, Hkv, bs, D = k_cache.shape
    B, Hq, Dq = q.shape
    MB = block_tables.shape[1]
    if Dq != D or v_cache.shape != k_cache.shape or k_scale.shape != (NB, Hkv, bs) or \
            v_scale.shape != k_scale.shape or block_tables.shape[0] != B or context_lens.numel() != B:
        raise ValueError("shape mismatch between q, caches, scales, block_tables and context_lens")
    if out is None:
        out = torch.empty_like(q)
    else:
        _contig(_dev(out, "out", torch.bfloat16), "out")
    return NB, Hkv, bs, D, B, Hq, MB, out


def paged_attention_int8(q, k_cache, v_cache, k_scale, v_scale, block_tables, context_lens, scale: float,
                         out=None, max_context_len: int = 0, workspace: Optional[torch.Tensor] = None,
                         stream=None) -> torch.Tensor:
    """Decode over the int8 cache.  q [B, Hq, D] bf16 -> out [B, Hq, D] bf16."""
    NB, Hkv, bs, D, B, Hq, MB, out = _int8_common(q, k_cache, v_cache, k_scale, v_scale, block_tables,
                                                  context_lens, out)
    lib = load_library()
    need = int(lib.pkv_paged_attention_workspace_size(B, Hq, Hkv, D, MB, bs, max_context_len))
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_ptr = workspace.data_ptr() if workspace is not None else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    rc = lib.pkv_paged_attention_int8(out.data_ptr(), q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(),
                                      k_scale.data_ptr(), v_scale.data_ptr(), block_tables.data_ptr(), MB,
                                      context_lens.data_ptr(), B, Hq, Hkv, D, NB, bs, float(scale),
                                      int(max_context_len), ws_ptr, ws_bytes, _stream(stream))
    _check(rc, "paged_attention_int8")
    return out


def paged_attention_int8_window(q, k_cache, v_cache, k_scale, v_scale, block_tables, context_lens, scale: float,
                                window: int, out=None, workspace: Optional[torch.Tensor] = None,
                                stream=None) -> torch.Tensor:
    """Decode over the int8 cache under a sliding window of `window` keys."""
    NB, Hkv, bs, D, B, Hq, MB, out = _int8_common(q, k_cache, v_cache, k_scale, v_scale, block_tables,
                                                  context_lens, out)
    lib = load_library()
    need = int(lib.pkv_paged_attention_window_workspace_size(B, Hq, Hkv, D, MB, bs, int(window)))
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_ptr = workspace.data_ptr() if workspace is not None else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    rc = lib.pkv_paged_attention_int8_window(out.data_ptr(), q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(),
                                             k_scale.data_ptr(), v_scale.data_ptr(), block_tables.data_ptr(), MB,
                                             context_lens.data_ptr(), B, Hq, Hkv, D, NB, bs, float(scale),
                                             int(window), ws_ptr, ws_bytes, _stream(stream))
    _check(rc, "paged_attention_int8_window")
    return out


def paged_attention_window(q, k_cache, v_cache, block_tables, context_lens, scale: float, window: int,
                           out=None, workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Decode where each query sees only its last ``window`` keys.  q [B, Hq, D] bf16."""
    NB, Hkv, bs, D, B, Hq, MB, out = _decode_common(q, k_cache, v_cache, block_tables, context_lens, out)
    lib = load_library()
    need = int(lib.pkv_paged_attention_window_workspace_size(B, Hq, Hkv, D, MB, bs, int(window)))
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_ptr = workspace.data_ptr() if workspace is not None else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    rc = lib.pkv_paged_attention_window(out.data_ptr(), q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(),
                                        block_tables.data_ptr(), MB, context_lens.data_ptr(), B, Hq, Hkv, D, NB,
                                        bs, float(scale), int(window), ws_ptr, ws_bytes, PKV_BF16, _stream(stream))
    _check(rc, "paged_attention_window")
    return out


def window_workspace_size(B, Hq, Hkv, D, MB, bs, window) -> int:
    return int(load_library().pkv_paged_attention_window_workspace_size(B, Hq, Hkv, D, MB, bs, int(window)))


def workspace_size(B, Hq, Hkv, D, MB, bs=16, max_context_len: int = 0) -> int:
    return int(load_library().pkv_paged_attention_workspace_size(B, Hq, Hkv, D, MB, bs, max_context_len))


def split_workspace_size(B, Hq, D, num_splits) -> int:
    return int(load_library().pkv_split_workspace_size(B, Hq, D, num_splits))


def paged_attention(q, k_cache, v_cache, block_tables, context_lens, scale: float, out=None,
                    max_context_len: int = 0, workspace: Optional[torch.Tensor] = None,
                    stream=None) -> torch.Tensor:
    """Decode attention.  q [B, Hq, D] bf16 -> out [B, Hq, D] bf16.

    ``max_context_len`` is a host-side upper bound on context_lens (0: MB*bs).
    ``workspace`` (uint8 CUDA tensor) enables the split-KV path; when None, one
    of the right size is taken from PyTorch's allocator."""
    NB, Hkv, bs, D, B, Hq, MB, out = _decode_common(q, k_cache, v_cache, block_tables, context_lens, out)
    lib = load_library()
    need = int(lib.pkv_paged_attention_workspace_size(B, Hq, Hkv, D, MB, bs, max_context_len))
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_ptr = workspace.data_ptr() if workspace is not None else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    rc = lib.pkv_paged_attention(out.data_ptr(), q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(),
                                 block_tables.data_ptr(), MB, context_lens.data_ptr(), B, Hq, Hkv, D,
                                 NB, bs, float(scale), int(max_context_len), ws_ptr, ws_bytes, PKV_BF16,
                                 _stream(stream))
    _check(rc, "paged_attention")
    return out


def paged_attention_split(q, k_cache, v_cache, block_tables, context_lens, scale: float,
                          pages_per_split: int, out=None, max_context_len: int = 0,
                          workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Split-KV decode with an explicit split size (pages per CTA)."""
    NB, Hkv, bs, D, B, Hq, MB, out = _decode_common(q, k_cache, v_cache, block_tables, context_lens, out)
    lib = load_library()
    max_ctx = max_context_len if max_context_len > 0 else MB * bs
    max_pages = max(1, -(-min(max_ctx, MB * bs) // 16))
    C = -(-max_pages // int(pages_per_split))
    need = int(lib.pkv_split_workspace_size(B, Hq, D, C))
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_ptr = workspace.data_ptr() if workspace is not None else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    rc = lib.pkv_paged_attention_split(out.data_ptr(), q.data_ptr(), k_cache.data_ptr(),
                                       v_cache.data_ptr(), block_tables.data_ptr(), MB,
                                       context_lens.data_ptr(), B, Hq, Hkv, D, NB, bs, float(scale),
                                       int(max_context_len), int(pages_per_split), ws_ptr, ws_bytes,
                                       PKV_BF16, _stream(stream))
    _check(rc, "paged_attention_split")
    return out


# Bytes of the library's static split-KV scratch (one array per GPU).
NOALLOC_SCRATCH_BYTES = 8 << 20


def paged_attention_split_noalloc(q, k_cache, v_cache, block_tables, context_lens, scale: float,
                                  pages_per_split: int, out=None, max_context_len: int = 0,
                                  stream=None) -> torch.Tensor:
    """Split-KV decode for callers that must not allocate device memory.

    Same result as paged_attention_split, but the split partials live in a
    static array inside the library (NOALLOC_SCRATCH_BYTES per GPU), so the
    call allocates nothing.  Pass ``out`` to keep this wrapper allocation-free
    as well.  Calls that overlap on the GPU share that array and race."""
    NB, Hkv, bs, D, B, Hq, MB, out = _decode_common(q, k_cache, v_cache, block_tables, context_lens, out)
    rc = load_library().pkv_paged_attention_split_noalloc(
        out.data_ptr(), q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), block_tables.data_ptr(), MB,
        context_lens.data_ptr(), B, Hq, Hkv, D, NB, bs, float(scale), int(max_context_len),
        int(pages_per_split), PKV_BF16, _stream(stream))
    _check(rc, "paged_attention_split_noalloc")
    return out


def paged_attention_prefill(q, query_start_loc, k_cache, v_cache, block_tables, context_lens,
                            scale: float, max_q_len: int, out=None, stream=None) -> torch.Tensor:
    """Causal chunked prefill.  q [sumQ, Hq, D] bf16 -> out [sumQ, Hq, D] bf16."""
    NB, Hkv, bs, D = _cache_dims(k_cache, v_cache)
    _contig(_dev(q, "q", torch.bfloat16), "q")
    _contig(_dev(query_start_loc, "query_start_loc", torch.int32), "query_start_loc")
    _contig(_dev(block_tables, "block_tables", torch.int32), "block_tables")
    _contig(_dev(context_lens, "context_lens", torch.int32), "context_lens")
    sumQ, Hq, Dq = q.shape
    B = context_lens.numel()
    if Dq != D or query_start_loc.numel() != B + 1 or block_tables.shape[0] != B:
        raise ValueError("shape mismatch between q, query_start_loc, block_tables, context_lens")
    if out is None:
        out = torch.empty_like(q)
    else:
        _contig(_dev(out, "out", torch.bfloat16), "out")
    rc = load_library().pkv_paged_attention_prefill(
        out.data_ptr(), q.data_ptr(), query_start_loc.data_ptr(), k_cache.data_ptr(),
        v_cache.data_ptr(), block_tables.data_ptr(), block_tables.shape[1], context_lens.data_ptr(),
        B, sumQ, int(max_q_len), Hq, Hkv, D, NB, bs, float(scale), PKV_BF16, _stream(stream))
    _check(rc, "paged_attention_prefill")
    return out


def paged_attention_prefill_window(q, query_start_loc, k_cache, v_cache, block_tables, context_lens,
                                   scale: float, max_q_len: int, window: int, out=None, stream=None) -> torch.Tensor:
    """Causal chunked prefill where a query at position p sees keys p - window < j <= p."""
    NB, Hkv, bs, D = _cache_dims(k_cache, v_cache)
    _contig(_dev(q, "q", torch.bfloat16), "q")
    _contig(_dev(query_start_loc, "query_start_loc", torch.int32), "query_start_loc")
    _contig(_dev(block_tables, "block_tables", torch.int32), "block_tables")
    _contig(_dev(context_lens, "context_lens", torch.int32), "context_lens")
    sumQ, Hq, Dq = q.shape
    B = context_lens.numel()
    if Dq != D or query_start_loc.numel() != B + 1 or block_tables.shape[0] != B:
        raise ValueError("shape mismatch between q, query_start_loc, block_tables, context_lens")
    if out is None:
        out = torch.empty_like(q)
    else:
        _contig(_dev(out, "out", torch.bfloat16), "out")
    rc = load_library().pkv_paged_attention_prefill_window(
        out.data_ptr(), q.data_ptr(), query_start_loc.data_ptr(), k_cache.data_ptr(),
        v_cache.data_ptr(), block_tables.data_ptr(), block_tables.shape[1], context_lens.data_ptr(),
        B, sumQ, int(max_q_len), Hq, Hkv, D, NB, bs, float(scale), int(window), PKV_BF16, _stream(stream))
    _check(rc, "paged_attention_prefill_window")
    return out


class BlockAllocator:
    """Host bookkeeping of physical cache blocks with reference counts (the
    library's pkv_block_allocator_*; no device memory, no CUDA calls)."""

    def __init__(self, num_blocks: int):
        self._lib = load_library()
        h = _P()
        _check(self._lib.pkv_block_allocator_create(int(num_blocks), ctypes.byref(h)), "block_allocator_create")
        self._h = h

    def close(self):
        if self._h:
            self._lib.pkv_block_allocator_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    @staticmethod
    def _ids(ids):
        arr = (_I32 * len(ids))(*[int(i) for i in ids])
        return arr, len(ids)

    def alloc(self, n: int) -> list:
        arr = (_I32 * max(1, n))()
        _check(self._lib.pkv_block_allocator_alloc(self._h, int(n), arr), "block_allocator_alloc")
        return list(arr[:n])

    def share(self, ids) -> None:
        arr, n = self._ids(ids)
        _check(self._lib.pkv_block_allocator_share(self._h, arr, n), "block_allocator_share")

    def release(self, ids) -> None:
        arr, n = self._ids(ids)
        _check(self._lib.pkv_block_allocator_release(self._h, arr, n), "block_allocator_release")

    def cow(self, block: int):
        """(block to write into, whether the caller must copy the old block to it first)."""
        nid, must = _I32(0), _I32(0)
        _check(self._lib.pkv_block_allocator_cow(self._h, int(block), ctypes.byref(nid), ctypes.byref(must)),
               "block_allocator_cow")
        return int(nid.value), bool(must.value)

    def num_free(self) -> int:
        return int(self._lib.pkv_block_allocator_num_free(self._h))

    def refcount(self, block: int) -> int:
        return int(self._lib.pkv_block_allocator_refcount(self._h, int(block)))


def copy_blocks(k_cache: torch.Tensor, v_cache: torch.Tensor, pairs: torch.Tensor, stream=None) -> None:
    """Copy block pairs[i, 0] -> pairs[i, 1] in both pools, bit for bit.
    Pools [NB, ...] (any dtype, contiguous); pairs int32 [n, 2] on the device."""
    for t, name in ((k_cache, "k_cache"), (v_cache, "v_cache")):
        _contig(_dev(t, name), name)
    _contig(_dev(pairs, "pairs", torch.int32), "pairs")
    if k_cache.shape[0] != v_cache.shape[0] or k_cache[0].nbytes != v_cache[0].nbytes:
        raise ValueError("k_cache and v_cache must have the same number and size of blocks")
    if pairs.dim() != 2 or pairs.shape[1] != 2:
        raise ValueError("pairs must be [n, 2]")
    rc = load_library().pkv_copy_blocks(k_cache.data_ptr(), v_cache.data_ptr(), k_cache[0].nbytes,
                                        pairs.data_ptr(), pairs.shape[0], k_cache.shape[0], _stream(stream))
    _check(rc, "copy_blocks")


def hbm_read_probe(buf: torch.Tensor, sink: torch.Tensor, chunk_bytes: int = 32768, stream=None) -> None:
    """Read all of `buf` once in bulk copies of `chunk_bytes` (measurement
    utility); one uint32 per CTA into `sink`."""
    _contig(_dev(buf, "buf"), "buf")
    _contig(_dev(sink, "sink", torch.int32), "sink")
    rc = load_library().pkv_hbm_read_probe(buf.data_ptr(), buf.numel() * buf.element_size(), int(chunk_bytes),
                                           sink.data_ptr(), sink.numel(), _stream(stream))
    _check(rc, "hbm_read_probe")


def get_device_error(stream=None) -> int:
    """Synchronise the stream; return and clear the device error word (0 = none)."""
    v = _I32(0)
    _check(load_library().pkv_get_device_error(_stream(stream), ctypes.byref(v)), "get_device_error")
    return int(v.value)


def last_launch_count() -> int:
    return int(load_library().pkv_last_launch_count())


def selftest_wait_timeout(timeout_us: int = 2000, stream=None) -> None:
    _check(load_library().pkv_selftest_wait_timeout(int(timeout_us), _stream(stream)),
           "selftest_wait_timeout")
