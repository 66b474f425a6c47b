"""GPU parity of block copies (bit-exact against the oracle's copy) and of a
parallel-sampling run over shared prompt blocks: allocator, copy-on-write,
cache write and decode through the C ABI against the oracle doing the same
steps on the host."""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_477_b200 as pkv
from oracle.blocks import BlockPool, copy_blocks as ref_copy_blocks
from paged_kv_cache_477_b200.workloads import bf16_bits
from parity import assert_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _library():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from paged_kv_cache_477_b200 import build
    build.build()
    pkv.load_library()
    pkv.get_device_error()
    yield


def _pairs(NB, n, seed):
    """n (src, dst) pairs with distinct dsts, none of them a src."""
    perm = torch.randperm(NB, generator=torch.Generator().manual_seed(seed))
    dst = perm[:n]
    src = perm[n:][torch.randint(0, NB - n, (n,), generator=torch.Generator().manual_seed(seed + 1))]
    return torch.stack([src, dst], 1).to(torch.int32)


@pytest.mark.parametrize("NB,Hkv,bs,D,n", [(40, 8, 16, 128, 12), (9, 2, 16, 64, 4), (300, 1, 16, 128, 100),
                                          (5, 3, 4, 64, 1)])
def test_copy_blocks_bf16_bit_exact(NB, Hkv, bs, D, n):
    g = torch.Generator().manual_seed(NB + D)
    k = torch.randn(NB, Hkv, bs, D, generator=g).to(torch.bfloat16)
    v = torch.randn(NB, Hkv, bs, D, generator=g).to(torch.bfloat16)
    pairs = _pairs(NB, n, seed=NB)
    hk, hv = bf16_bits(k).copy(), bf16_bits(v).copy()
    assert ref_copy_blocks([hk, hv], pairs.numpy()) == 0
    kd, vd = k.cuda(), v.cuda()
    pkv.copy_blocks(kd, vd, pairs.cuda())
    assert pkv.last_launch_count() == 1
    assert np.array_equal(bf16_bits(kd), hk) and np.array_equal(bf16_bits(vd), hv)
    assert pkv.get_device_error() == 0


def test_copy_blocks_int8_codes_and_scales():
    NB, Hkv, bs, D = 33, 2, 16, 128
    g = torch.Generator().manual_seed(7)
    k = torch.randint(-127, 128, (NB, Hkv, bs, D), generator=g, dtype=torch.int8)
    v = torch.randint(-127, 128, (NB, Hkv, bs, D), generator=g, dtype=torch.int8)
    ks = torch.rand(NB, Hkv, bs, generator=g) * 0.03
    vs = torch.rand(NB, Hkv, bs, generator=g) * 0.03
    pairs = _pairs(NB, 10, seed=8)
    host = [t.numpy().copy() for t in (k, v, ks, vs)]
    ref_copy_blocks(host, pairs.numpy())
    dev = [t.cuda() for t in (k, v, ks, vs)]
    p = pairs.cuda()
    pkv.copy_blocks(dev[0], dev[1], p)
    pkv.copy_blocks(dev[2], dev[3], p)
    for d, h in zip(dev, host):
        assert np.array_equal(d.cpu().numpy().view(np.uint8), h.view(np.uint8))
    assert pkv.get_device_error() == 0


def test_copy_blocks_out_of_range_pair_is_reported_and_skipped():
    NB, Hkv, bs, D = 6, 1, 16, 64
    g = torch.Generator().manual_seed(9)
    k = torch.randn(NB, Hkv, bs, D, generator=g).to(torch.bfloat16)
    v = torch.randn(NB, Hkv, bs, D, generator=g).to(torch.bfloat16)
    pairs = torch.tensor([[0, 1], [2, NB], [-1, 3], [4, 5]], dtype=torch.int32)
    hk, hv = bf16_bits(k).copy(), bf16_bits(v).copy()
    assert ref_copy_blocks([hk, hv], pairs.numpy()) == 2
    kd, vd = k.cuda(), v.cuda()
    pkv.copy_blocks(kd, vd, pairs.cuda())
    assert pkv.get_device_error() == 5
    assert np.array_equal(bf16_bits(kd), hk) and np.array_equal(bf16_bits(vd), hv)


def test_copy_blocks_empty_launches_nothing():
    k = torch.zeros(4, 1, 16, 64, dtype=torch.bfloat16, device="cuda")
    pkv.copy_blocks(k, k.clone(), torch.zeros(0, 2, dtype=torch.int32, device="cuda"))
    assert pkv.last_launch_count() == 0


@pytest.mark.parametrize("prompt_len", [37, 48])
def test_parallel_sampling_over_shared_prompt_blocks(prompt_len):
    """Four samples fork from one prompt: the prompt's blocks are shared, each
    sample copies-on-write the block it writes its next token into, writes it
    and decodes.  Both sides take the same steps; the pools must match bit for
    bit and attention within tolerance."""
    Hq, Hkv, D, bs, NB, S = 8, 2, 128, 16, 16, 4
    g = torch.Generator().manual_seed(prompt_len)
    k0 = torch.randn(NB, Hkv, bs, D, generator=g).to(torch.bfloat16)   # stale contents
    v0 = torch.randn(NB, Hkv, bs, D, generator=g).to(torch.bfloat16)
    pk = torch.randn(prompt_len, Hkv, D, generator=g).to(torch.bfloat16)
    pv = torch.randn(prompt_len, Hkv, D, generator=g).to(torch.bfloat16)
    nk = torch.randn(S, Hkv, D, generator=g).to(torch.bfloat16)       # each sample's new token
    nv = torch.randn(S, Hkv, D, generator=g).to(torch.bfloat16)
    q = torch.randn(S, Hq, D, generator=g).to(torch.bfloat16)
    scale = D ** -0.5

    alloc, model = pkv.BlockAllocator(NB), BlockPool(NB)
    npages = -(-prompt_len // bs)
    prompt = alloc.alloc(npages)
    assert prompt == model.alloc(npages)
    alloc.share(prompt * (S - 1))
    assert model.share(prompt * (S - 1))
    slot_prompt = torch.tensor([prompt[t // bs] * bs + t % bs for t in range(prompt_len)], dtype=torch.int64)

    # each sample's next token goes to row prompt_len of its table
    tables, pairs, slots = [], [], []
    for s in range(S):
        table = list(prompt)
        page, row = divmod(prompt_len, bs)
        if page == len(table):                   # the prompt filled its last block: a fresh one
            b = alloc.alloc(1)[0]
            assert [b] == model.alloc(1)
            table.append(b)
        else:                                    # writing into a shared block
            b, must = alloc.cow(table[page])
            assert (b, must) == model.cow(table[page])
            if must:
                pairs.append((table[page], b))
            table[page] = b
        tables.append(table)
        slots.append(table[page] * bs + row)
    MB = max(len(t) for t in tables)
    bt = torch.tensor([t + [0] * (MB - len(t)) for t in tables], dtype=torch.int32)
    lens = torch.full((S,), prompt_len + 1, dtype=torch.int32)
    pairs_t = torch.tensor(pairs, dtype=torch.int32).reshape(-1, 2)
    slots_t = torch.tensor(slots, dtype=torch.int64)

    # host: the oracle's steps
    hk, hv = bf16_bits(k0).copy(), bf16_bits(v0).copy()
    orc = oracle.get()
    orc.kv_cache_write(bf16_bits(pk), bf16_bits(pv), hk, hv, slot_prompt.numpy())
    ref_copy_blocks([hk, hv], pairs_t.numpy())
    orc.kv_cache_write(bf16_bits(nk), bf16_bits(nv), hk, hv, slots_t.numpy())
    ref = orc.paged_attention(bf16_bits(q), hk, hv, bt.numpy(), lens.numpy(), scale)

    # device: the library's steps
    kd, vd = k0.cuda(), v0.cuda()
    pkv.kv_cache_write(pk.cuda(), pv.cuda(), kd, vd, slot_prompt.cuda())
    pkv.copy_blocks(kd, vd, pairs_t.cuda())
    pkv.kv_cache_write(nk.cuda(), nv.cuda(), kd, vd, slots_t.cuda())
    out = pkv.paged_attention(q.cuda(), kd, vd, bt.cuda(), lens.cuda(), scale)

    assert np.array_equal(bf16_bits(kd), hk) and np.array_equal(bf16_bits(vd), hv)
    assert_close(out, ref, f"parallel sampling prompt_len={prompt_len}")
    assert pkv.get_device_error() == 0
    if prompt_len % bs:
        assert len(pairs) == S - 1               # the last holder writes in place
    alloc.close()
