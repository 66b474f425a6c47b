"""NumPy full-matrix brute force for tiny paged-attention inputs.

TEST INFRASTRUCTURE (see ``oracle/__init__.py``).  A second formulation,
written independently of the C oracle: build each sequence's dense K and V by
fancy-indexing the pool through its block table, repeat the kv heads to the
query heads, form the whole score matrix ``S = scale * Q K^T`` with an additive
``-inf`` causal mask, take a row softmax, multiply by V.  float64 throughout.

It follows the same pages as the C oracle: the logical-to-physical page map
("从零构建CUDA推理引擎：Tiny-Infer项目的技术深度解析", section
"分页KV缓存：借鉴操作系统的内存管理") and plain softmax attention, which
FlashAttention reorganises but does not change ("5 Fun Projects for LLM
Inference Engineering", section 2).
"""
from __future__ import annotations

import numpy as np

from . import bf16_bits_to_f64


def dense_kv(cache_bits: np.ndarray, block_table_row: np.ndarray, n: int) -> np.ndarray:
    """[n, Hkv, D] float64 view of one sequence's first n keys (or values)."""
    NB, Hkv, bs, D = cache_bits.shape
    npages = -(-n // bs)
    pages = block_table_row[:npages]
    g = bf16_bits_to_f64(cache_bits[pages])           # [npages, Hkv, bs, D]
    g = np.transpose(g, (0, 2, 1, 3)).reshape(npages * bs, Hkv, D)
    return g[:n]


def _softmax_rows(S: np.ndarray) -> np.ndarray:
    m = S.max(axis=-1, keepdims=True)
    P = np.exp(S - m)
    return P / P.sum(axis=-1, keepdims=True)


def attention_chunk(q_bits, k_bits, v_bits, block_table_row, L, scale):
    """q_bits [Q, Hq, D]: the last Q positions of a sequence with L keys.
    Returns [Q, Hq, D] float64."""
    Q, Hq, D = q_bits.shape
    Hkv = k_bits.shape[1]
    if L == 0 or Q == 0:
        return np.zeros((Q, Hq, D))
    K = dense_kv(k_bits, block_table_row, L)           # [L, Hkv, D]
    V = dense_kv(v_bits, block_table_row, L)
    rep = Hq // Hkv
    K = np.repeat(K, rep, axis=1).transpose(1, 0, 2)   # [Hq, L, D]
    V = np.repeat(V, rep, axis=1).transpose(1, 0, 2)
    qf = bf16_bits_to_f64(q_bits).transpose(1, 0, 2)   # [Hq, Q, D]
    # scale crosses the ABI as an fp32 value; widen that exact value
    S = np.float64(np.float32(scale)) * (qf @ K.transpose(0, 2, 1))  # [Hq, Q, L]
    pos = (L - Q) + np.arange(Q)[:, None]              # absolute query positions
    mask = np.where(np.arange(L)[None, :] <= pos, 0.0, -np.inf)
    P = _softmax_rows(S + mask[None])
    return (P @ V).transpose(1, 0, 2)                  # [Q, Hq, D]


def paged_attention(q_bits, k_bits, v_bits, block_tables, context_lens, scale):
    B, Hq, D = q_bits.shape
    out = np.zeros((B, Hq, D))
    for b in range(B):
        out[b] = attention_chunk(q_bits[b:b + 1], k_bits, v_bits, block_tables[b],
                                 int(context_lens[b]), scale)[0]
    return out


def paged_attention_prefill(q_bits, query_start_loc, k_bits, v_bits, block_tables,
                            context_lens, scale):
    sumQ, Hq, D = q_bits.shape
    out = np.zeros((sumQ, Hq, D))
    for b in range(len(context_lens)):
        s, e = int(query_start_loc[b]), int(query_start_loc[b + 1])
        out[s:e] = attention_chunk(q_bits[s:e], k_bits, v_bits, block_tables[b],
                                   int(context_lens[b]), scale)
    return out
