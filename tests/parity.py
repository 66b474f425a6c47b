"""Helpers for GPU-vs-oracle parity tests.

The oracle's inputs always come from the seeded generator
(paged_kv_cache_477_b200.workloads) -- never from a CUDA kernel's output.
Where a CUDA kernel writes the cache before attention, the oracle applies its
own cache write to the generator's pre-write cache.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from paged_kv_cache_477_b200.workloads import PagedCase, bf16_bits

# Attention tolerance: |gpu - ref| <= ATOL + RTOL * |ref| (bf16 I/O, fp32 accumulate).
ATOL = 5e-3
RTOL = 1e-2


def assert_close(gpu_bf16: torch.Tensor, ref: np.ndarray, what: str = ""):
    got = gpu_bf16.detach().float().cpu().numpy().astype(np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    err = np.abs(got - ref)
    bound = ATOL + RTOL * np.abs(ref)
    bad = err > bound
    if bad.any():
        idx = np.unravel_index(np.argmax(err - bound), err.shape)
        raise AssertionError(f"{what}: {int(bad.sum())} of {err.size} outside tolerance; worst at {idx}: "
                             f"gpu={got[idx]!r} ref={ref[idx]!r} |d|={err[idx]:.3e}; max|d|={err.max():.3e}")
    return float(err.max())


class HostCase:
    """uint16/int views of a case for the oracle (pre-write cache)."""

    def __init__(self, case: PagedCase):
        self.case = case
        self.q = bf16_bits(case.q)
        self.int8 = case.kv_dtype == "int8"
        if self.int8:
            self.k = case.k_cache.cpu().numpy().copy()
            self.v = case.v_cache.cpu().numpy().copy()
            self.ks = case.k_scale.cpu().numpy().copy()
            self.vs = case.v_scale.cpu().numpy().copy()
        else:
            self.k = bf16_bits(case.k_cache).copy()
            self.v = bf16_bits(case.v_cache).copy()
        self.bt = case.block_tables.cpu().numpy().astype(np.int32)
        self.lens = case.context_lens.cpu().numpy().astype(np.int32)
        self.qsl = case.query_start_loc.cpu().numpy().astype(np.int32) if case.query_start_loc is not None else None
        self.written = False

    def apply_write(self):
        c = self.case
        if c.new_key is not None and not self.written:
            slots = c.slot_mapping.cpu().numpy().astype(np.int64)
            if self.int8:
                oracle.get().kv_cache_write_int8(bf16_bits(c.new_key), bf16_bits(c.new_value), self.k, self.v,
                                                 self.ks, self.vs, slots)
            else:
                oracle.get().kv_cache_write(bf16_bits(c.new_key), bf16_bits(c.new_value), self.k, self.v, slots)
        self.written = True
        return self

    def decode_ref(self, rows=None):
        rows = np.arange(self.case.B) if rows is None else np.asarray(rows)
        if self.int8:
            return oracle.get().paged_attention_int8(np.ascontiguousarray(self.q[rows]), self.k, self.v, self.ks,
                                                     self.vs, np.ascontiguousarray(self.bt[rows]),
                                                     np.ascontiguousarray(self.lens[rows]), self.case.scale)
        return oracle.get().paged_attention(np.ascontiguousarray(self.q[rows]), self.k, self.v,
                                            np.ascontiguousarray(self.bt[rows]),
                                            np.ascontiguousarray(self.lens[rows]), self.case.scale)

    def decode_window_ref(self, window, rows=None):
        rows = np.arange(self.case.B) if rows is None else np.asarray(rows)
        return oracle.get().paged_attention_window(np.ascontiguousarray(self.q[rows]), self.k, self.v,
                                                   np.ascontiguousarray(self.bt[rows]),
                                                   np.ascontiguousarray(self.lens[rows]), self.case.scale, window)

    def prefill_ref(self, seqs=None, window=0):
        """Reference for whole sequences ``seqs`` (sliding ``window`` if > 0);
        returns (ref, token_index)."""
        c = self.case
        seqs = list(range(c.B)) if seqs is None else list(seqs)
        qsl = self.qsl
        tok = np.concatenate([np.arange(qsl[b], qsl[b + 1]) for b in seqs]).astype(np.int64)
        sub_qsl = np.concatenate([[0], np.cumsum([qsl[b + 1] - qsl[b] for b in seqs])]).astype(np.int32)
        if window:
            ref = oracle.get().paged_attention_prefill_window(np.ascontiguousarray(self.q[tok]), sub_qsl, self.k,
                                                              self.v, np.ascontiguousarray(self.bt[seqs]),
                                                              np.ascontiguousarray(self.lens[seqs]), c.scale, window)
        else:
            ref = oracle.get().paged_attention_prefill(np.ascontiguousarray(self.q[tok]), sub_qsl, self.k, self.v,
                                                       np.ascontiguousarray(self.bt[seqs]),
                                                       np.ascontiguousarray(self.lens[seqs]), c.scale)
        return ref, tok
