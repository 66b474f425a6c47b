"""Seeded synthetic inputs for paged-KV attention.

This module is the one thing the CUDA path and the fp64 oracle share: it draws
random tensors, context lengths, block tables and slot mappings, and holds none
of the attention arithmetic.  Every tensor is reproducible from its seed.

Recipe (one case):

1. ``pages_b = ceil(L_b / bs)``; the pool has ``NB >= sum_b pages_b`` blocks.
2. ``perm = randperm(NB)`` from a CPU generator seeded with ``seed``;
   sequence ``b`` takes the next ``pages_b`` entries of ``perm`` in batch
   order, so physical blocks are shuffled across the pool.  Unused block-table
   entries hold ``-1``.
3. On the target device, with a generator seeded ``seed + 1``: ``q``,
   ``k_cache``, ``v_cache`` and then the new rows to write are drawn as
   float32 N(0, 1) and rounded to bf16 (round-to-nearest-even).
4. Canaries: every pool slot that is not a valid key -- unused blocks, the
   tail of each sequence's last page, and the slots the write step is about to
   fill -- holds bf16 NaN, so an over-read or a missed write shows up as NaN.
5. ``scale = 1 / sqrt(D)`` computed in float32.
6. ``kv_dtype="int8"``: the pool holds int8 codes drawn uniformly from
   [-127, 127] and one fp32 scale per row drawn log-uniformly from
   [0.008, 0.03] (so values code * scale are of order 1); canary rows get a
   NaN scale.  No quantisation happens here: the new rows of the write step
   are bf16 N(0, 1) as above, and the write step quantises them.

The five named workloads reproduce the attention shapes of the pages' models
(Llama-3.2-1B and Llama-3-8B) as stand-ins: the pages measure on no dataset.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional, Sequence

import numpy as np
import torch

BF16_NAN_BITS = 0x7FC0


@dataclass
class PagedCase:
    name: str
    kind: str                      # "decode" or "prefill"
    B: int
    Hq: int
    Hkv: int
    D: int
    bs: int
    NB: int
    MB: int
    scale: float
    seed: int
    q: torch.Tensor                # decode [B, Hq, D]; prefill [sumQ, Hq, D]
    k_cache: torch.Tensor          # [NB, Hkv, bs, D] bf16
    v_cache: torch.Tensor
    block_tables: torch.Tensor     # [B, MB] int32, -1 padded
    context_lens: torch.Tensor     # [B] int32, includes rows written by the write step
    new_key: Optional[torch.Tensor] = None    # [T, Hkv, D] bf16 (write step)
    new_value: Optional[torch.Tensor] = None
    slot_mapping: Optional[torch.Tensor] = None  # [T] int64
    query_start_loc: Optional[torch.Tensor] = None  # prefill [B+1] int32
    max_q_len: int = 1
    lens: list = field(default_factory=list)
    kv_dtype: str = "bf16"         # "int8": k_cache/v_cache hold int8 codes
    k_scale: Optional[torch.Tensor] = None    # int8: [NB, Hkv, bs] fp32 row scales
    v_scale: Optional[torch.Tensor] = None

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    def kv_bytes_read(self) -> int:
        """K and V bytes a decode pass must read: sum_b L_b * Hkv * D * 2 B * 2
        (int8: sum_b L_b * Hkv * (D + 4) * 2, codes plus the row scale)."""
        if self.kv_dtype == "int8":
            return int(sum(self.lens)) * self.Hkv * (self.D + 4) * 2
        return int(sum(self.lens)) * self.Hkv * self.D * 2 * 2


def default_scale(D: int) -> float:
    return float(np.float32(1.0) / np.sqrt(np.float32(D)))


def make_case(*, name: str = "custom", kind: str = "decode", B: int, Hq: int, Hkv: int,
              D: int, bs: int = 16, lens: Sequence[int], seed: int, device="cpu",
              pool_blocks: Optional[int] = None, MB: Optional[int] = None,
              write_tokens: int = 0, q_len: Optional[Sequence[int]] = None,
              canaries: bool = True, scale: Optional[float] = None, kv_dtype: str = "bf16") -> PagedCase:
    """Build one seeded case.

    kind="decode": one query per sequence; the last ``write_tokens`` positions
    of each sequence are written by the write step (their slots start as NaN).
    kind="prefill": sequence b has a query chunk of ``q_len[b]`` new tokens,
    which are the last ``q_len[b]`` positions of its ``lens[b]`` keys; their
    K/V rows are the write step's rows.
    """
    lens = [int(x) for x in lens]
    assert len(lens) == B
    g = torch.Generator().manual_seed(int(seed))
    pages = [-(-L // bs) for L in lens]
    used = sum(pages)
    NB = int(pool_blocks) if pool_blocks is not None else used
    assert NB >= used, "pool smaller than the sequences need"
    MB = int(MB) if MB is not None else max(1, max(pages) if pages else 1)
    assert MB >= max(pages + [0])
    perm = torch.randperm(NB, generator=g) if NB > 0 else torch.zeros(0, dtype=torch.int64)
    bt = torch.full((B, MB), -1, dtype=torch.int32)
    off = 0
    for b in range(B):
        bt[b, :pages[b]] = perm[off:off + pages[b]].to(torch.int32)
        off += pages[b]

    if kind == "prefill":
        assert q_len is not None
        qlens = [int(x) for x in q_len]
        assert all(0 <= qlens[b] <= lens[b] for b in range(B))
        write_pos = [list(range(lens[b] - qlens[b], lens[b])) for b in range(B)]
        nq = sum(qlens)
    else:
        qlens = [1] * B
        assert all(write_tokens <= L for L in lens)
        write_pos = [list(range(L - write_tokens, L)) for L in lens]
        nq = B

    gd = torch.Generator(device=device).manual_seed(int(seed) + 1)

    def randn_bf16(*shape):
        out = torch.empty(*shape, dtype=torch.bfloat16, device=device)
        flat = out.view(-1)
        n = flat.numel()
        chunk = 1 << 26
        for s in range(0, n, chunk):
            e = min(n, s + chunk)
            flat[s:e] = torch.randn(e - s, generator=gd, device=device, dtype=torch.float32).to(torch.bfloat16)
        return out

    q = randn_bf16(nq, Hq, D)
    k_scale = v_scale = None
    if kv_dtype == "int8":
        assert kind == "decode", "the int8 cache is read by decode only"
        k_cache = torch.randint(-127, 128, (NB, Hkv, bs, D), generator=gd, device=device, dtype=torch.int8)
        v_cache = torch.randint(-127, 128, (NB, Hkv, bs, D), generator=gd, device=device, dtype=torch.int8)
        lo, hi = math.log(0.008), math.log(0.03)
        k_scale = torch.exp(lo + (hi - lo) * torch.rand(NB, Hkv, bs, generator=gd, device=device))
        v_scale = torch.exp(lo + (hi - lo) * torch.rand(NB, Hkv, bs, generator=gd, device=device))
    else:
        assert kv_dtype == "bf16"
        k_cache = randn_bf16(NB, Hkv, bs, D)
        v_cache = randn_bf16(NB, Hkv, bs, D)
    T = sum(len(w) for w in write_pos)
    new_key = new_value = slot_mapping = None
    if T > 0:
        new_key = randn_bf16(T, Hkv, D)
        new_value = randn_bf16(T, Hkv, D)
        slots = []
        for b in range(B):
            for pos in write_pos[b]:
                slots.append(int(bt[b, pos // bs]) * bs + pos % bs)
        slot_mapping = torch.tensor(slots, dtype=torch.int64)

    if canaries and NB > 0:
        valid = torch.zeros(NB, bs, dtype=torch.bool)
        for b in range(B):
            L_old = lens[b] - len(write_pos[b])
            for p in range(pages[b]):
                lo, hi = p * bs, min((p + 1) * bs, L_old)
                if hi > lo:
                    valid[int(bt[b, p]), : hi - lo] = True
        invalid = (~valid).to(device)                          # [NB, bs]
        if kv_dtype == "int8":
            nanf = torch.tensor(float("nan"), dtype=torch.float32, device=device)
            k_scale = torch.where(invalid[:, None, :], nanf, k_scale)
            v_scale = torch.where(invalid[:, None, :], nanf, v_scale)
        else:
            nanv = torch.tensor(float("nan"), dtype=torch.bfloat16, device=device)
            mask = invalid[:, None, :, None]
            k_cache = torch.where(mask, nanv, k_cache)
            v_cache = torch.where(mask, nanv, v_cache)

    qsl = None
    if kind == "prefill":
        qsl = torch.tensor(np.concatenate([[0], np.cumsum(qlens)]), dtype=torch.int32)

    return PagedCase(
        name=name, kind=kind, B=B, Hq=Hq, Hkv=Hkv, D=D, bs=bs, NB=NB, MB=MB,
        scale=float(scale) if scale is not None else default_scale(D), seed=int(seed),
        q=q, k_cache=k_cache.contiguous(), v_cache=v_cache.contiguous(),
        block_tables=bt.to(device), context_lens=torch.tensor(lens, dtype=torch.int32).to(device),
        new_key=new_key, new_value=new_value,
        slot_mapping=slot_mapping.to(device) if slot_mapping is not None else None,
        query_start_loc=qsl.to(device) if qsl is not None else None,
        max_q_len=max(qlens) if qlens else 0, lens=lens, kv_dtype=kv_dtype,
        k_scale=k_scale.contiguous() if k_scale is not None else None,
        v_scale=v_scale.contiguous() if v_scale is not None else None,
    )


# --------------------------------------------------------------------------- #
# The named workloads (the five of the measurement plan, their INT8 and
# eight-heads-per-group variants).                                                    #
# --------------------------------------------------------------------------- #

def _lens_llama32_1b(seed: int):
    g = torch.Generator().manual_seed(seed)
    return torch.randint(512, 4097, (64,), generator=g).tolist()


def _lens_ragged(seed: int):
    g = torch.Generator().manual_seed(seed)
    u = torch.rand(12, generator=g, dtype=torch.float64)
    short = torch.round(torch.exp(math.log(128) + u * (math.log(8192) - math.log(128)))).long().tolist()
    lens = [32768] * 4 + short
    order = torch.randperm(16, generator=g).tolist()
    return [lens[i] for i in order]


WORKLOADS = {
    # name: (builder kwargs, one-line description)
    "tiny_decode": dict(
        kind="decode", B=2, Hq=4, Hkv=2, D=64, bs=16, lens=[37, 100], seed=1001, pool_blocks=16,
        desc="tiny paged decode: B=2, Hq=4/Hkv=2, D=64, bs=16, lens 37 and 100, 16-block pool"),
    "llama32_1b_decode": dict(
        kind="decode", B=64, Hq=32, Hkv=8, D=64, bs=16, lens=_lens_llama32_1b(1002), seed=1002,
        desc="Llama-3.2-1B-shaped decode: B=64, Hq=32/Hkv=8, D=64, bs=16, lens U[512,4096]"),
    "llama3_8b_decode": dict(
        kind="decode", B=128, Hq=32, Hkv=8, D=128, bs=16, lens=[4096] * 128, seed=1003,
        write_tokens=1,
        desc="Llama-3-8B-shaped decode: B=128, Hq=32/Hkv=8, D=128, bs=16, ctx 4096, "
             "one new token written per sequence before attention"),
    "llama3_8b_decode_int8": dict(
        kind="decode", B=128, Hq=32, Hkv=8, D=128, bs=16, lens=[4096] * 128, seed=1006,
        write_tokens=1, kv_dtype="int8",
        desc="Llama-3-8B-shaped decode over an INT8 cache (one fp32 scale per row): B=128, Hq=32/Hkv=8, "
             "D=128, bs=16, ctx 4096, one new token quantised into the cache per sequence before attention"),
    "ragged_long_decode": dict(
        kind="decode", B=16, Hq=32, Hkv=8, D=128, bs=16, lens=_lens_ragged(1004), seed=1004,
        desc="ragged long-context decode: B=16, Hq=32/Hkv=8, D=128, 4 x 32768 + 12 log-uniform "
             "[128, 8192]"),
    "gqa8_decode": dict(
        kind="decode", B=64, Hq=64, Hkv=8, D=128, bs=16, lens=[4096] * 64, seed=1007,
        desc="grouped-query decode with eight query heads per kv head: B=64, Hq=64/Hkv=8, D=128, bs=16, "
             "ctx 4096"),
    "chunked_prefill": dict(
        kind="prefill", B=4, Hq=32, Hkv=8, D=128, bs=16, lens=[4096] * 4, q_len=[512] * 4,
        seed=1005, pool_blocks=1024,
        desc="causal chunked prefill: B=4, Hq=32/Hkv=8, D=128, 512-token chunk after 3584 "
             "cached tokens, bs=16, 1024-block pool"),
}


def workload(name: str, device="cpu", **overrides) -> PagedCase:
    kw = dict(WORKLOADS[name])
    kw.pop("desc", None)
    kw.update(overrides)
    return make_case(name=name, device=device, **kw)


def describe(name: str) -> str:
    return WORKLOADS[name]["desc"]


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """uint16 bit patterns of a bf16 tensor (copied to host memory)."""
    assert t.dtype == torch.bfloat16
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)
