"""The bench's algorithmic byte and flop counts (the numerators of every
roofline fraction) against figures worked out by hand from the workload
definitions, and against counts taken from a generated case's own arrays."""
import types

import numpy as np
import torch

import bench
from paged_kv_cache_477_b200 import workloads as wl


def _spec_case(name, **kw):
    """A stand-in with the fields the counts read, built from the workload's
    definition without allocating its pools."""
    sp = dict(wl.WORKLOADS[name])
    sp.update(kw)
    c = types.SimpleNamespace(B=sp["B"], Hq=sp["Hq"], Hkv=sp["Hkv"], D=sp["D"], bs=sp["bs"], lens=list(sp["lens"]),
                              kv_dtype=sp.get("kv_dtype", "bf16"), new_key=None)
    c.kv_bytes_read = lambda: wl.PagedCase.kv_bytes_read(c)
    return c, sp


def test_llama3_8b_decode_bytes_by_hand():
    # K+V: 128 sequences x 4096 keys x 8 kv heads x 128 x 2 B x 2 = 2 GiB;
    # q and out 128 x 32 x 128 x 2 B each; 256 block-table entries per
    # sequence (4 B) and 128 lengths (4 B)
    c, _ = _spec_case("llama3_8b_decode")
    assert bench.decode_bytes(c) == 2_147_483_648 + 2 * 1_048_576 + 128 * 256 * 4 + 128 * 4 == 2_149_712_384


def test_llama3_8b_decode_int8_bytes_by_hand():
    # codes: half the bf16 bytes; scales: one fp32 per (token, kv head) for K and V
    c, _ = _spec_case("llama3_8b_decode_int8")
    kv = 1_073_741_824 + 128 * 4096 * 8 * 4 * 2
    assert kv == 1_107_296_256
    assert bench.decode_bytes(c) == kv + 2 * 1_048_576 + 128 * 256 * 4 + 128 * 4 == 1_109_524_992


def test_tiny_decode_kv_bytes_by_hand():
    # 37 + 100 keys x 2 kv heads x 64 x 2 B x 2
    c, _ = _spec_case("tiny_decode")
    assert c.kv_bytes_read() == 70_144


def test_cache_write_bytes_by_hand():
    # 128 rows x 8 kv heads x 128 x 2 B, read and written, for K and V; 8 B of slot each
    key = torch.empty(128, 8, 128, dtype=torch.bfloat16)
    c = types.SimpleNamespace(new_key=key, Hkv=8, D=128)
    assert bench.write_bytes(c) == 2 * (2 * 128 * 8 * 128 * 2) + 128 * 8 == 1_049_600


def test_chunked_prefill_flops_closed_form():
    # per (sequence, q head): 4 D sum_{i<512} (3584 + i + 1) keys seen; 4 sequences x 32 heads
    _, sp = _spec_case("chunked_prefill")
    B, Hq, D = sp["B"], sp["Hq"], sp["D"]
    Q = 512
    qsl = torch.tensor([b * Q for b in range(B + 1)], dtype=torch.int32)
    c = types.SimpleNamespace(B=B, Hq=Hq, D=D, lens=[4096] * B, query_start_loc=qsl)
    per = 4 * D * (Q * 3585 + Q * (Q - 1) // 2)
    assert bench.prefill_flops(c) == per * Hq * B == 128_865_796_096


def test_decode_bytes_match_a_generated_case():
    """On a generated case the counts follow from its arrays: keys from the
    lengths, block-table entries from the pages actually used."""
    case = wl.make_case(B=5, Hq=8, Hkv=2, D=64, bs=16, lens=[1, 15, 16, 17, 300], seed=3)
    lens = case.context_lens.numpy()
    pages_used = int(sum(-(-int(L) // 16) for L in lens))
    kv = int(lens.sum()) * 2 * 64 * 2 * 2
    qo = 2 * case.q.numel() * case.q.element_size()
    assert bench.decode_bytes(case) == kv + qo + pages_used * 4 + 5 * 4
    assert case.kv_bytes_read() == kv
    assert int((case.block_tables.numpy() >= 0).sum()) == pages_used  # padding entries are -1
