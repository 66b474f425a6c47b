"""fp64 CPU oracle for paged-KV attention.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
baseline / reference leg of ``bench.py`` may import this package.  The CUDA
library (``paged_kv_cache_477_b200``) never imports it, and the two share no
code: both only see the same seeded inputs from
``paged_kv_cache_477_b200.workloads``.

Two independent formulations live here:

* ``pagedkv_oracle.c`` -- plain C, fp64, one query row at a time: gather keys
  through the block table, two-pass softmax, weighted sum of V.  Wrapped by
  :class:`Oracle` through ctypes.
* :mod:`oracle.brute` -- NumPy full-matrix form (dense gather, ``Q @ K^T``,
  additive -inf mask, softmax, ``@ V``) for tiny inputs.

Arrays cross the boundary as NumPy arrays: bf16 tensors as their uint16 bit
patterns, indices as int32/int64, results as float64.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import tempfile

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pagedkv_oracle.c")
LIB_PATH = os.path.join(_HERE, "libpagedkv_oracle.so")

_P = ctypes.c_void_p
_I32 = ctypes.c_int32
_I64 = ctypes.c_int64
_F32 = ctypes.c_float


def build(out_path: str | None = None, mutant: int = 0, force: bool = False) -> str:
    """Compile the C oracle with gcc (OpenMP, -O2, no fast-math)."""
    out_path = out_path or LIB_PATH
    if not force and mutant == 0 and os.path.exists(out_path) and (
        os.path.getmtime(out_path) >= os.path.getmtime(_SRC)
    ):
        return out_path
    cmd = [
        "gcc", "-O2", "-std=c11", "-fopenmp", "-shared", "-fPIC",
        f"-DPKV_ORACLE_MUTANT={int(mutant)}", _SRC, "-lm", "-o", out_path,
    ]
    subprocess.run(cmd, check=True)
    return out_path


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data


class OracleError(RuntimeError):
    pass


class Oracle:
    """ctypes front of the C oracle.  ``mutant`` > 0 loads a build with one
    deliberately planted mistake (used only to show that the pins catch it)."""

    def __init__(self, mutant: int = 0, path: str | None = None):
        if mutant:
            path = path or os.path.join(tempfile.mkdtemp(prefix="pkv_mut"), f"liboracle_m{mutant}.so")
            build(path, mutant=mutant, force=True)
        else:
            path = build(path)
        self.path = path
        lib = ctypes.CDLL(path)
        lib.ref_num_threads.restype = ctypes.c_int
        lib.ref_set_num_threads.argtypes = [ctypes.c_int]
        lib.ref_set_num_threads.restype = None
        lib.ref_mutant_id.restype = ctypes.c_int
        lib.ref_kv_cache_write.argtypes = [_P, _P, _I64, _I64, _P, _P, _P, _I32, _I32, _I32, _I32, _I32]
        lib.ref_paged_attention.argtypes = [_P, _P, _P, _P, _P, _I32, _P, _I32, _I32, _I32, _I32, _I32, _I32, _F32]
        lib.ref_contiguous_attention.argtypes = [_P, _P, _P, _P, _P, _I32, _I32, _I32, _I32, _I32, _F32]
        lib.ref_paged_attention_prefill.argtypes = [_P, _P, _P, _P, _P, _P, _I32, _P, _I32, _I32, _I32, _I32, _I32, _I32, _F32]
        lib.ref_decode_partials.argtypes = [_P, _P, _P, _P, _P, _P, _I32, _P, _I32, _I32, _I32, _I32, _I32, _I32, _F32, _I32, _I32]
        lib.ref_lse_merge.argtypes = [_P, _P, _P, _I64, _I32, _I32]
        lib.ref_kv_cache_write_int8.argtypes = [_P, _P, _I64, _I64, _P, _P, _P, _P, _P, _I32, _I32, _I32,
                                                _I32, _I32]
        lib.ref_paged_attention_int8.argtypes = [_P, _P, _P, _P, _P, _P, _P, _I32, _P, _I32, _I32, _I32, _I32,
                                                 _I32, _I32, _F32]
        lib.ref_paged_attention_int8_window.argtypes = [_P, _P, _P, _P, _P, _P, _P, _I32, _P, _I32, _I32, _I32,
                                                        _I32, _I32, _I32, _F32, _I32]
        lib.ref_paged_attention_window.argtypes = [_P, _P, _P, _P, _P, _I32, _P, _I32, _I32, _I32, _I32, _I32,
                                                   _I32, _F32, _I32]
        lib.ref_paged_attention_prefill_window.argtypes = [_P, _P, _P, _P, _P, _P, _I32, _P, _I32, _I32, _I32,
                                                           _I32, _I32, _I32, _F32, _I32]
        lib.ref_rope_rows.argtypes = [_P, _P, _I64, _P, _I64, _I32, _I32, ctypes.c_double]
        lib.ref_kv_cache_write_rope.argtypes = [_P, _P, _I64, _I64, _P, _P, _P, _P, _I32, _I32, _I32, _I32, _I32,
                                                ctypes.c_double]
        lib.ref_rope_rows.restype = ctypes.c_int
        lib.ref_kv_cache_write_rope.restype = ctypes.c_int
        for f in ("ref_kv_cache_write", "ref_paged_attention", "ref_contiguous_attention",
                  "ref_paged_attention_prefill", "ref_decode_partials", "ref_lse_merge",
                  "ref_kv_cache_write_int8", "ref_paged_attention_int8", "ref_paged_attention_window",
                  "ref_paged_attention_prefill_window"):
            getattr(lib, f).restype = ctypes.c_int
        self.lib = lib
        self.mutant = lib.ref_mutant_id()

    def num_threads(self) -> int:
        return int(self.lib.ref_num_threads())

    def set_num_threads(self, n: int) -> None:
        self.lib.ref_set_num_threads(int(n))

    @staticmethod
    def _check(rc: int, what: str, allow_bounds: bool = False) -> int:
        if rc == 0 or (allow_bounds and rc == 5):
            return rc
        raise OracleError(f"{what}: oracle status {rc}")

    # -- cache write ---------------------------------------------------------
    def kv_cache_write(self, key, value, k_cache, v_cache, slot_mapping, allow_bounds=False) -> int:
        """Scatter key/value [T, Hkv, D] (uint16 bits) into k_cache/v_cache
        [NB, Hkv, bs, D] in place.  Returns the status (5 = a slot outside the pool)."""
        T, Hkv, D = key.shape
        NB, Hkv2, bs, D2 = k_cache.shape
        assert Hkv == Hkv2 and D == D2 and value.shape == key.shape and v_cache.shape == k_cache.shape
        slot_mapping = np.ascontiguousarray(slot_mapping, dtype=np.int64)
        key = np.ascontiguousarray(key)
        value = np.ascontiguousarray(value)
        rc = self.lib.ref_kv_cache_write(_ptr(key), _ptr(value), Hkv * D, Hkv * D, _ptr(k_cache),
                                         _ptr(v_cache), _ptr(slot_mapping), T, Hkv, D, NB, bs)
        return self._check(rc, "kv_cache_write", allow_bounds)

    def kv_cache_write_int8(self, key, value, k_cache, v_cache, k_scale, v_scale, slot_mapping,
                            allow_bounds=False) -> int:
        """Quantise key/value [T, Hkv, D] (uint16 bf16 bits) into the int8 pools
        k_cache/v_cache [NB, Hkv, bs, D] and their fp32 scales [NB, Hkv, bs], in place."""
        T, Hkv, D = key.shape
        NB, Hkv2, bs, D2 = k_cache.shape
        assert Hkv == Hkv2 and D == D2 and value.shape == key.shape and v_cache.shape == k_cache.shape
        assert k_cache.dtype == np.int8 and k_scale.dtype == np.float32 and k_scale.shape == (NB, Hkv, bs)
        slot_mapping = np.ascontiguousarray(slot_mapping, dtype=np.int64)
        key = np.ascontiguousarray(key)
        value = np.ascontiguousarray(value)
        rc = self.lib.ref_kv_cache_write_int8(_ptr(key), _ptr(value), Hkv * D, Hkv * D, _ptr(k_cache),
                                              _ptr(v_cache), _ptr(k_scale), _ptr(v_scale), _ptr(slot_mapping),
                                              T, Hkv, D, NB, bs)
        return self._check(rc, "kv_cache_write_int8", allow_bounds)

    def paged_attention_int8(self, q, k_cache, v_cache, k_scale, v_scale, block_tables, context_lens, scale,
                             allow_bounds=False, window: int = 0) -> np.ndarray:
        """Decode over the int8 pools: attention over the values code * scale
        (window > 0: only the query's last `window` keys)."""
        B, Hq, D = q.shape
        NB, Hkv, bs, _ = k_cache.shape
        assert k_cache.dtype == np.int8 and k_scale.dtype == np.float32
        block_tables = np.ascontiguousarray(block_tables, dtype=np.int32)
        context_lens = np.ascontiguousarray(context_lens, dtype=np.int32)
        MB = block_tables.shape[1] if block_tables.ndim == 2 else 0
        out = np.zeros((B, Hq, D), dtype=np.float64)
        args = (_ptr(out), _ptr(np.ascontiguousarray(q)), _ptr(k_cache), _ptr(v_cache), _ptr(k_scale),
                _ptr(v_scale), _ptr(block_tables), MB, _ptr(context_lens), B, Hq, Hkv, D, NB, bs, float(scale))
        if window:
            rc = self.lib.ref_paged_attention_int8_window(*args, int(window))
        else:
            rc = self.lib.ref_paged_attention_int8(*args)
        self._check(rc, "paged_attention_int8", allow_bounds)
        return out

    # -- rotary position embedding ------------------------------------------
    def rope_rows(self, x, positions, base) -> np.ndarray:
        """fp64 rotated rows of x [T, H, D] (uint16 bf16 bits) at positions [T]."""
        T, H, D = x.shape
        x = np.ascontiguousarray(x)
        positions = np.ascontiguousarray(positions, dtype=np.int64)
        out = np.zeros((T, H, D), dtype=np.float64)
        rc = self.lib.ref_rope_rows(_ptr(out), _ptr(x), H * D, _ptr(positions), T, H, D, float(base))
        self._check(rc, "rope_rows")
        return out

    def kv_cache_write_rope(self, key, value, k_cache, v_cache, slot_mapping, positions, base,
                            allow_bounds=False) -> int:
        """Cache write with K rotated at its position (bf16 of the fp64 rotation); V copied."""
        T, Hkv, D = key.shape
        NB, Hkv2, bs, D2 = k_cache.shape
        assert Hkv == Hkv2 and D == D2 and value.shape == key.shape and v_cache.shape == k_cache.shape
        slot_mapping = np.ascontiguousarray(slot_mapping, dtype=np.int64)
        positions = np.ascontiguousarray(positions, dtype=np.int64)
        key = np.ascontiguousarray(key)
        value = np.ascontiguousarray(value)
        rc = self.lib.ref_kv_cache_write_rope(_ptr(key), _ptr(value), Hkv * D, Hkv * D, _ptr(k_cache),
                                              _ptr(v_cache), _ptr(slot_mapping), _ptr(positions), T, Hkv, D, NB,
                                              bs, float(base))
        return self._check(rc, "kv_cache_write_rope", allow_bounds)

    # -- sliding window -------------------------------------------------------
    def paged_attention_window(self, q, k_cache, v_cache, block_tables, context_lens, scale, window,
                               allow_bounds=False) -> np.ndarray:
        """Decode where the query (position L_b - 1) sees only its last ``window`` keys."""
        B, Hq, D = q.shape
        NB, Hkv, bs, _ = k_cache.shape
        block_tables = np.ascontiguousarray(block_tables, dtype=np.int32)
        context_lens = np.ascontiguousarray(context_lens, dtype=np.int32)
        MB = block_tables.shape[1] if block_tables.ndim == 2 else 0
        out = np.zeros((B, Hq, D), dtype=np.float64)
        rc = self.lib.ref_paged_attention_window(_ptr(out), _ptr(np.ascontiguousarray(q)), _ptr(k_cache),
                                                 _ptr(v_cache), _ptr(block_tables), MB, _ptr(context_lens),
                                                 B, Hq, Hkv, D, NB, bs, float(scale), int(window))
        self._check(rc, "paged_attention_window", allow_bounds)
        return out

    def paged_attention_prefill_window(self, q, query_start_loc, k_cache, v_cache, block_tables, context_lens,
                                       scale, window, allow_bounds=False) -> np.ndarray:
        sumQ, Hq, D = q.shape
        NB, Hkv, bs, _ = k_cache.shape
        B = len(context_lens)
        block_tables = np.ascontiguousarray(block_tables, dtype=np.int32)
        qsl = np.ascontiguousarray(query_start_loc, dtype=np.int32)
        context_lens = np.ascontiguousarray(context_lens, dtype=np.int32)
        MB = block_tables.shape[1] if block_tables.ndim == 2 else 0
        out = np.zeros((sumQ, Hq, D), dtype=np.float64)
        rc = self.lib.ref_paged_attention_prefill_window(_ptr(out), _ptr(np.ascontiguousarray(q)), _ptr(qsl),
                                                         _ptr(k_cache), _ptr(v_cache), _ptr(block_tables), MB,
                                                         _ptr(context_lens), B, Hq, Hkv, D, NB, bs, float(scale),
                                                         int(window))
        self._check(rc, "paged_attention_prefill_window", allow_bounds)
        return out

    # -- decode ----------------------------------------------------------------
    def paged_attention(self, q, k_cache, v_cache, block_tables, context_lens, scale,
                        allow_bounds=False) -> np.ndarray:
        B, Hq, D = q.shape
        NB, Hkv, bs, _ = k_cache.shape
        block_tables = np.ascontiguousarray(block_tables, dtype=np.int32)
        context_lens = np.ascontiguousarray(context_lens, dtype=np.int32)
        MB = block_tables.shape[1] if block_tables.ndim == 2 else 0
        out = np.zeros((B, Hq, D), dtype=np.float64)
        rc = self.lib.ref_paged_attention(_ptr(out), _ptr(np.ascontiguousarray(q)), _ptr(k_cache),
                                          _ptr(v_cache), _ptr(block_tables), MB, _ptr(context_lens),
                                          B, Hq, Hkv, D, NB, bs, float(scale))
        self._check(rc, "paged_attention", allow_bounds)
        return out

    def contiguous_attention(self, q, k, v, context_lens, scale) -> np.ndarray:
        B, Hq, D = q.shape
        B2, Lmax, Hkv, D2 = k.shape
        assert B == B2 and D == D2 and v.shape == k.shape
        context_lens = np.ascontiguousarray(context_lens, dtype=np.int32)
        out = np.zeros((B, Hq, D), dtype=np.float64)
        rc = self.lib.ref_contiguous_attention(_ptr(out), _ptr(np.ascontiguousarray(q)),
                                               _ptr(np.ascontiguousarray(k)), _ptr(np.ascontiguousarray(v)),
                                               _ptr(context_lens), B, Lmax, Hq, Hkv, D, float(scale))
        self._check(rc, "contiguous_attention")
        return out

    # -- prefill ---------------------------------------------------------------
    def paged_attention_prefill(self, q, query_start_loc, k_cache, v_cache, block_tables,
                                context_lens, scale, allow_bounds=False) -> np.ndarray:
        sumQ, Hq, D = q.shape
        NB, Hkv, bs, _ = k_cache.shape
        block_tables = np.ascontiguousarray(block_tables, dtype=np.int32)
        context_lens = np.ascontiguousarray(context_lens, dtype=np.int32)
        qsl = np.ascontiguousarray(query_start_loc, dtype=np.int32)
        B = context_lens.shape[0]
        assert qsl.shape[0] == B + 1 and qsl[-1] == sumQ
        MB = block_tables.shape[1]
        out = np.zeros((sumQ, Hq, D), dtype=np.float64)
        rc = self.lib.ref_paged_attention_prefill(_ptr(out), _ptr(np.ascontiguousarray(q)), _ptr(qsl),
                                                  _ptr(k_cache), _ptr(v_cache), _ptr(block_tables), MB,
                                                  _ptr(context_lens), B, Hq, Hkv, D, NB, bs, float(scale))
        self._check(rc, "paged_attention_prefill", allow_bounds)
        return out

    # -- split-KV algebra ------------------------------------------------------
    def decode_partials(self, q, k_cache, v_cache, block_tables, context_lens, scale,
                        split_tokens: int, num_splits: int):
        B, Hq, D = q.shape
        NB, Hkv, bs, _ = k_cache.shape
        block_tables = np.ascontiguousarray(block_tables, dtype=np.int32)
        context_lens = np.ascontiguousarray(context_lens, dtype=np.int32)
        MB = block_tables.shape[1]
        o = np.zeros((B, Hq, num_splits, D), dtype=np.float64)
        lse = np.zeros((B, Hq, num_splits), dtype=np.float64)
        rc = self.lib.ref_decode_partials(_ptr(o), _ptr(lse), _ptr(np.ascontiguousarray(q)), _ptr(k_cache),
                                          _ptr(v_cache), _ptr(block_tables), MB, _ptr(context_lens),
                                          B, Hq, Hkv, D, NB, bs, float(scale), int(split_tokens),
                                          int(num_splits))
        self._check(rc, "decode_partials")
        return o, lse

    def lse_merge(self, o_part, lse) -> np.ndarray:
        *lead, C, D = o_part.shape
        rows = int(np.prod(lead)) if lead else 1
        o_part = np.ascontiguousarray(o_part, dtype=np.float64)
        lse = np.ascontiguousarray(lse, dtype=np.float64)
        out = np.zeros((*lead, D), dtype=np.float64)
        rc = self.lib.ref_lse_merge(_ptr(out), _ptr(o_part), _ptr(lse), rows, C, D)
        self._check(rc, "lse_merge")
        return out


_DEFAULT: Oracle | None = None


def get() -> Oracle:
    """The default (unmutated) oracle, built on first use."""
    global _DEFAULT
    if _DEFAULT is None:
        _DEFAULT = Oracle()
    return _DEFAULT


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns (uint16) to float64."""
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
