"""GPU parity of the INT8 KV cache (one fp32 scale per row) against the fp64 oracle.

Cache writes (codes and scales, over the whole pool) must match the oracle
bit for bit; attention over the int8 pool must satisfy
|gpu - ref| <= 5e-3 + 1e-2 |ref|, where ref is plain fp64 attention over the
values code * scale (the kernel holds q as a 15-bit fixed-point pair per head
for its integer tensor-core scores).  Every call goes through the C ABI.
"""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_477_b200 as pkv
from paged_kv_cache_477_b200 import workloads as wl
from paged_kv_cache_477_b200.workloads import bf16_bits
from parity import HostCase, assert_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _library():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from paged_kv_cache_477_b200 import build
    build.build()
    pkv.load_library()
    pkv.get_device_error()
    yield


def _pools(NB, Hkv, bs, D, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    k = torch.randint(-127, 128, (NB, Hkv, bs, D), generator=g, device="cuda", dtype=torch.int8)
    v = torch.randint(-127, 128, (NB, Hkv, bs, D), generator=g, device="cuda", dtype=torch.int8)
    ks = torch.full((NB, Hkv, bs), float("nan"), device="cuda")     # canaries
    vs = torch.full((NB, Hkv, bs), float("nan"), device="cuda")
    return k, v, ks, vs


def _same_bits(a: torch.Tensor, b: np.ndarray) -> bool:
    """Bitwise equality (NaN canaries compare equal to themselves)."""
    x = a.detach().cpu().numpy()
    return x.shape == b.shape and np.array_equal(x.view(np.uint8), b.view(np.uint8))


@pytest.mark.parametrize("T,Hkv,D,bs,NB", [(37, 2, 64, 16, 9), (128, 8, 128, 16, 64), (5, 3, 256, 4, 4),
                                         (300, 1, 128, 8, 50)])
def test_int8_cache_write_bit_exact(T, Hkv, D, bs, NB):
    g = torch.Generator(device="cuda").manual_seed(T + D)
    key = (torch.randn(T, Hkv, D, device="cuda", generator=g) * 3).to(torch.bfloat16)
    val = torch.randn(T, Hkv, D, device="cuda", generator=g).to(torch.bfloat16)
    key[1] = 0                                            # a zero row: codes 0, scale 0
    val[2, 0, :4] = torch.tensor([127.0, 2.5, -3.5, 0.5])  # exact ties with amax 127
    val[2, 0, 4:] = 0
    k, v, ks, vs = _pools(NB, Hkv, bs, D, seed=T)
    gc = torch.Generator().manual_seed(T)
    slots = torch.randperm(NB * bs, generator=gc)[:T].to(torch.int64)
    slots[::7] = -1                                       # padding tokens are skipped
    hk, hv, hks, hvs = (t.cpu().numpy().copy() for t in (k, v, ks, vs))
    oracle.get().kv_cache_write_int8(bf16_bits(key), bf16_bits(val), hk, hv, hks, hvs, slots.numpy())
    pkv.kv_cache_write_int8(key, val, k, v, ks, vs, slots.cuda())
    assert pkv.last_launch_count() == 1
    assert _same_bits(k, hk) and _same_bits(v, hv)
    assert _same_bits(ks, hks) and _same_bits(vs, hvs)
    assert pkv.get_device_error() == 0


def test_int8_cache_write_strided_rows():
    """key/value taken as column slices of a fused [T, 3*Hkv*D] projection."""
    T, Hkv, D, bs, NB = 20, 2, 128, 16, 4
    g = torch.Generator(device="cuda").manual_seed(3)
    qkv = torch.randn(T, 3 * Hkv * D, device="cuda", generator=g).to(torch.bfloat16)
    key = qkv[:, Hkv * D:2 * Hkv * D].view(T, Hkv, D)
    val = qkv[:, 2 * Hkv * D:].view(T, Hkv, D)
    k, v, ks, vs = _pools(NB, Hkv, bs, D, seed=4)
    slots = torch.arange(T, dtype=torch.int64, device="cuda") * 3 % (NB * bs)
    hk, hv, hks, hvs = (t.cpu().numpy().copy() for t in (k, v, ks, vs))
    oracle.get().kv_cache_write_int8(bf16_bits(key.contiguous()), bf16_bits(val.contiguous()), hk, hv, hks, hvs,
                                     slots.cpu().numpy())
    pkv.kv_cache_write_int8(key, val, k, v, ks, vs, slots)
    assert _same_bits(k, hk) and _same_bits(v, hv) and _same_bits(ks, hks) and _same_bits(vs, hvs)
    assert pkv.get_device_error() == 0


def test_int8_cache_write_out_of_range_slot_is_reported_and_skipped():
    NB, Hkv, bs, D = 2, 1, 16, 64
    k, v, ks, vs = _pools(NB, Hkv, bs, D, seed=5)
    key = torch.ones(2, Hkv, D, device="cuda", dtype=torch.bfloat16)
    before = k.clone()
    slots = torch.tensor([NB * bs, 5], dtype=torch.int64, device="cuda")
    pkv.kv_cache_write_int8(key, key, k, v, ks, vs, slots)
    assert pkv.get_device_error() == 5
    assert torch.equal(k[0, 0, 5], torch.full((D,), 127, dtype=torch.int8, device="cuda"))
    k[0, 0, 5] = before[0, 0, 5]
    assert torch.equal(k, before)                         # nothing else written


def _case(lens, Hq, Hkv, D, seed, write_tokens=0):
    pages = sum(-(-L // 16) for L in lens)
    return wl.make_case(B=len(lens), Hq=Hq, Hkv=Hkv, D=D, bs=16, lens=lens, seed=seed, device="cuda",
                        pool_blocks=pages + 3, write_tokens=write_tokens, kv_dtype="int8")


def _decode(case, **kw):
    return pkv.paged_attention_int8(case.q, case.k_cache, case.v_cache, case.k_scale, case.v_scale,
                                    case.block_tables, case.context_lens, case.scale, **kw)


EDGE_LENS = [0, 1, 15, 16, 17, 31, 32, 33, 100, 257, 600]


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (4, 2), (8, 2), (6, 2), (32, 8)])
def test_int8_decode_shapes_and_edges(D, Hq, Hkv):
    case = _case(EDGE_LENS, Hq, Hkv, D, seed=200 + D + Hq)
    out = _decode(case)
    assert_close(out, HostCase(case).decode_ref(), f"int8 D={D} G={Hq // Hkv}")
    assert torch.count_nonzero(out[0]) == 0              # empty context -> zero row
    assert pkv.get_device_error() == 0


@pytest.mark.parametrize("D", [64, 128])
def test_int8_decode_query_dynamic_range(D):
    """Query heads far from unit scale, one dominated by a single element, one
    all zero: the scores stay within tolerance of plain fp64 attention."""
    case = _case([5, 77, 300, 1000], 8, 2, D, seed=230 + D)
    q = case.q.float()
    q[:, 0] *= 1000.0
    q[:, 1] *= 1e-3
    q[:, 2, 0] = 100.0
    q[:, 3] = 0.0
    q[:, 4] *= 3e-20
    q[:, 5] *= 2e15
    case.q = q.to(torch.bfloat16)
    out = _decode(case)
    assert_close(out, HostCase(case).decode_ref(), f"int8 q range D={D}")
    assert pkv.get_device_error() == 0


@pytest.mark.parametrize("D", [64, 128])
def test_int8_decode_negative_scale(D):
    """A negative scale over the INT8 cache (the integer scores are scaled after
    the tensor-core product), plain and split, against the oracle."""
    lens = [5000, 3, 0, 17, 1200, 640]
    pages = sum(-(-L // 16) for L in lens)
    case = wl.make_case(B=len(lens), Hq=16, Hkv=4, D=D, bs=16, lens=lens, seed=215 + D, device="cuda",
                        pool_blocks=pages + 3, kv_dtype="int8", scale=-0.2)
    ref = HostCase(case).decode_ref()
    assert_close(_decode(case), ref, f"int8 negative scale D={D}")
    assert pkv.get_device_error() == 0


def test_int8_decode_long_contexts_split():
    """Contexts long enough for the automatic plan to split (partials + merge)."""
    case = _case([5000, 3, 0, 17, 1200, 4096, 640, 33] * 2, 32, 8, 128, seed=210)
    out = _decode(case)
    assert pkv.last_launch_count() == 2
    assert_close(out, HostCase(case).decode_ref(), "int8 split")
    assert pkv.get_device_error() == 0


def test_int8_write_then_decode_llama3_8b_shaped_full():
    """The bench's int8 step: quantise one new token per sequence into the
    cache, then decode; the written pool is bit-exact, every row in tolerance."""
    case = wl.workload("llama3_8b_decode_int8", device="cuda")
    host = HostCase(case)
    pkv.kv_cache_write_int8(case.new_key, case.new_value, case.k_cache, case.v_cache, case.k_scale,
                            case.v_scale, case.slot_mapping)
    out = _decode(case, max_context_len=4096)
    host.apply_write()
    assert _same_bits(case.k_cache, host.k) and _same_bits(case.v_cache, host.v)
    assert _same_bits(case.k_scale, host.ks) and _same_bits(case.v_scale, host.vs)
    assert_close(out, host.decode_ref(), "llama3_8b_decode_int8")
    assert pkv.get_device_error() == 0


def test_int8_decode_ragged_long_workload_full():
    """The ragged long-context batch over the int8 cache (4 x 32768 and 12 shorter
    contexts, split into the int8 kernel's longer splits and merged); every row
    of the 16 sequences against the int8 oracle."""
    case = wl.workload("ragged_long_decode", device="cuda", kv_dtype="int8")
    out = _decode(case, max_context_len=32768)
    assert pkv.last_launch_count() == 2                  # split partials + merge
    assert_close(out, HostCase(case).decode_ref(), "ragged_long_decode int8")
    assert pkv.get_device_error() == 0


def test_int8_decode_bad_block_id_is_reported():
    case = _case([40, 40], 4, 2, 64, seed=211)
    bt = case.block_tables.clone()
    bt[1, 1] = case.NB + 5                                # outside the pool
    pkv.paged_attention_int8(case.q, case.k_cache, case.v_cache, case.k_scale, case.v_scale, bt,
                             case.context_lens, case.scale)
    assert pkv.get_device_error() == 5


# --------------------------------------------------------------------------- #
# sliding window over the INT8 cache                                           #
# --------------------------------------------------------------------------- #

def _decode_window(case, window, **kw):
    return pkv.paged_attention_int8_window(case.q, case.k_cache, case.v_cache, case.k_scale, case.v_scale,
                                           case.block_tables, case.context_lens, case.scale, window, **kw)


def _window_ref(case, window):
    h = HostCase(case)
    return oracle.get().paged_attention_int8(h.q, h.k, h.v, h.ks, h.vs, h.bt, h.lens, case.scale, window=window)


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("window", [1, 15, 16, 17, 100, 1000])
def test_int8_decode_window_edges(D, window):
    case = _case(EDGE_LENS, 8, 2, D, seed=240 + D + window)
    out = _decode_window(case, window)
    assert_close(out, _window_ref(case, window), f"int8 window={window} D={D}")
    assert torch.count_nonzero(out[0]) == 0
    assert pkv.get_device_error() == 0


@pytest.mark.parametrize("window", [64, 500, 4096])
def test_int8_decode_window_long_contexts_split(window):
    """Long contexts: the window plan splits the pages a window touches."""
    case = _case([5000, 3, 0, 17, 1200, 4096, 640, 33] * 2, 32, 8, 128, seed=250 + window)
    out = _decode_window(case, window)
    assert_close(out, _window_ref(case, window), f"int8 window={window} split")
    assert pkv.get_device_error() == 0


def test_int8_decode_window_rejects_zero():
    case = _case([40], 4, 2, 64, seed=260)
    with pytest.raises(pkv.PagedKVError):
        _decode_window(case, 0)
