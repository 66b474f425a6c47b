"""GPU parity of the cache write and decode attention against the fp64 oracle.

Every call goes through the C ABI (via the ctypes binding).  Cache writes must
be bit-exact over the whole pool; attention must satisfy
|gpu - ref| <= 5e-3 + 1e-2 |ref| element by element.
"""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_477_b200 as pkv
from paged_kv_cache_477_b200 import workloads as wl
from paged_kv_cache_477_b200.workloads import bf16_bits
from oracle import bf16_bits_to_f64
from parity import HostCase, assert_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _library():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from paged_kv_cache_477_b200 import build
    build.build()
    pkv.load_library()
    pkv.get_device_error()  # start from a clean error word
    yield


def _no_device_error():
    assert pkv.get_device_error() == 0


# --------------------------------------------------------------------------- #
# kv_cache_write                                                               #
# --------------------------------------------------------------------------- #

@pytest.mark.parametrize("T,Hkv,D,bs,NB", [(37, 2, 64, 16, 9), (128, 8, 128, 16, 64), (5, 3, 8, 4, 4),
                                         (300, 1, 256, 8, 50)])
def test_kv_cache_write_bit_exact(T, Hkv, D, bs, NB):
    g = torch.Generator(device="cuda").manual_seed(T * 7 + D)
    k_cache = torch.randn(NB, Hkv, bs, D, device="cuda", generator=g).to(torch.bfloat16)
    v_cache = torch.randn(NB, Hkv, bs, D, device="cuda", generator=g).to(torch.bfloat16)
    key = torch.randn(T, Hkv, D, device="cuda", generator=g).to(torch.bfloat16)
    val = torch.randn(T, Hkv, D, device="cuda", generator=g).to(torch.bfloat16)
    gc = torch.Generator().manual_seed(T)
    slots = torch.randperm(NB * bs, generator=gc)[:T].to(torch.int64)
    slots[::7] = -1                                     # padding tokens are skipped
    k_host, v_host = bf16_bits(k_cache).copy(), bf16_bits(v_cache).copy()
    oracle.get().kv_cache_write(bf16_bits(key), bf16_bits(val), k_host, v_host, slots.numpy())
    pkv.kv_cache_write(key, val, k_cache, v_cache, slots.cuda())
    assert pkv.last_launch_count() == 1
    assert np.array_equal(bf16_bits(k_cache), k_host)
    assert np.array_equal(bf16_bits(v_cache), v_host)
    _no_device_error()


def test_kv_cache_write_strided_rows():
    """key/value taken as column slices of a fused [T, 3*Hkv*D] projection."""
    T, Hkv, D, bs, NB = 20, 2, 64, 16, 4
    g = torch.Generator(device="cuda").manual_seed(3)
    qkv = torch.randn(T, 3 * Hkv * D, device="cuda", generator=g).to(torch.bfloat16)
    key = qkv[:, Hkv * D:2 * Hkv * D].view(T, Hkv, D)
    val = qkv[:, 2 * Hkv * D:].view(T, Hkv, D)
    k_cache = torch.zeros(NB, Hkv, bs, D, device="cuda", dtype=torch.bfloat16)
    v_cache = torch.zeros_like(k_cache)
    slots = torch.arange(T, dtype=torch.int64, device="cuda") * 3 % (NB * bs)
    k_host, v_host = bf16_bits(k_cache).copy(), bf16_bits(v_cache).copy()
    oracle.get().kv_cache_write(bf16_bits(key.contiguous()), bf16_bits(val.contiguous()), k_host, v_host,
                                slots.cpu().numpy())
    pkv.kv_cache_write(key, val, k_cache, v_cache, slots)
    assert np.array_equal(bf16_bits(k_cache), k_host)
    assert np.array_equal(bf16_bits(v_cache), v_host)
    _no_device_error()


def test_kv_cache_write_out_of_range_slot_is_reported_and_skipped():
    NB, Hkv, bs, D = 2, 1, 16, 64
    k_cache = torch.zeros(NB, Hkv, bs, D, device="cuda", dtype=torch.bfloat16)
    v_cache = torch.zeros_like(k_cache)
    key = torch.ones(2, Hkv, D, device="cuda", dtype=torch.bfloat16)
    slots = torch.tensor([NB * bs, 5], dtype=torch.int64, device="cuda")
    pkv.kv_cache_write(key, key, k_cache, v_cache, slots)
    assert pkv.get_device_error() == 5
    assert float(k_cache.float().sum()) == D            # only slot 5 was written


def test_kv_cache_write_empty_is_noop():
    k_cache = torch.zeros(1, 1, 16, 64, device="cuda", dtype=torch.bfloat16)
    e = torch.empty(0, 1, 64, device="cuda", dtype=torch.bfloat16)
    pkv.kv_cache_write(e, e, k_cache, k_cache, torch.empty(0, dtype=torch.int64, device="cuda"))
    assert pkv.last_launch_count() == 0


# --------------------------------------------------------------------------- #
# decode                                                                       #
# --------------------------------------------------------------------------- #

def _decode_case(lens, Hq, Hkv, D, seed, write_tokens=0, pool_extra=3):
    pages = sum(-(-L // 16) for L in lens)
    return wl.make_case(B=len(lens), Hq=Hq, Hkv=Hkv, D=D, bs=16, lens=lens, seed=seed, device="cuda",
                        pool_blocks=pages + pool_extra, write_tokens=write_tokens)


def test_decode_tiny_workload():
    case = wl.workload("tiny_decode", device="cuda")
    host = HostCase(case)
    out = pkv.paged_attention(case.q, case.k_cache, case.v_cache, case.block_tables, case.context_lens,
                              case.scale)
    assert_close(out, host.decode_ref(), "tiny_decode")
    _no_device_error()


EDGE_LENS = [0, 1, 15, 16, 17, 31, 32, 33, 100, 257, 600]


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (4, 2), (8, 2), (16, 2), (6, 2), (32, 8), (16, 8), (24, 12), (8, 8),
                                    (3, 3), (6, 3), (12, 3), (4, 1)])
def test_decode_shapes_and_edges(D, Hq, Hkv):
    """Query heads per kv head from 1 to 8 (dividing 4 or not), odd and even kv-head
    counts, at both head sizes; ragged lengths from empty to several pages."""
    case = _decode_case(EDGE_LENS, Hq, Hkv, D, seed=100 + D + Hq)
    host = HostCase(case)
    ref = host.decode_ref()
    out = pkv.paged_attention(case.q, case.k_cache, case.v_cache, case.block_tables, case.context_lens,
                              case.scale)
    assert_close(out, ref, f"auto D={D} G={Hq // Hkv}")
    assert torch.count_nonzero(out[0]) == 0              # empty context -> zero row
    for pps in (1, 2, 3, 7):
        out_s = pkv.paged_attention_split(case.q, case.k_cache, case.v_cache, case.block_tables,
                                          case.context_lens, case.scale, pages_per_split=pps)
        assert_close(out_s, ref, f"split pps={pps} D={D} G={Hq // Hkv}")
    _no_device_error()


def test_decode_llama32_1b_workload_full():
    case = wl.workload("llama32_1b_decode", device="cuda")
    host = HostCase(case)
    out = pkv.paged_attention(case.q, case.k_cache, case.v_cache, case.block_tables, case.context_lens,
                              case.scale, max_context_len=4096)
    assert_close(out, host.decode_ref(), "llama32_1b_decode")
    _no_device_error()


def test_decode_llama3_8b_workload_with_write_full():
    """The bench's launch sequence: cache write of one token per sequence, then
    decode; every output row of the 128 sequences against the oracle."""
    case = wl.workload("llama3_8b_decode", device="cuda")
    host = HostCase(case)                       # pre-write pool, copied before any kernel runs
    pkv.kv_cache_write(case.new_key, case.new_value, case.k_cache, case.v_cache, case.slot_mapping)
    out = pkv.paged_attention(case.q, case.k_cache, case.v_cache, case.block_tables, case.context_lens,
                              case.scale, max_context_len=4096)
    host.apply_write()
    # the write is bit-exact over the whole pool
    assert np.array_equal(bf16_bits(case.k_cache), host.k)
    assert np.array_equal(bf16_bits(case.v_cache), host.v)
    assert_close(out, host.decode_ref(), "llama3_8b_decode")
    _no_device_error()


def test_decode_ragged_long_workload_full():
    """Split-KV partials and the merge over the ragged long-context batch;
    every row of the 16 sequences against the oracle."""
    case = wl.workload("ragged_long_decode", device="cuda")
    host = HostCase(case)
    out = pkv.paged_attention(case.q, case.k_cache, case.v_cache, case.block_tables, case.context_lens,
                              case.scale, max_context_len=32768)
    assert pkv.last_launch_count() == 2               # split-KV partials + merge
    assert_close(out, host.decode_ref(), "ragged_long_decode")
    _no_device_error()


def test_decode_gqa8_workload_full():
    """Eight query heads per kv head (64 q / 8 kv heads, D=128, ctx 4096): one
    CTA takes the whole group, so each page is read once; every row against
    the oracle."""
    case = wl.workload("gqa8_decode", device="cuda")
    out = pkv.paged_attention(case.q, case.k_cache, case.v_cache, case.block_tables, case.context_lens,
                              case.scale, max_context_len=4096)
    assert_close(out, HostCase(case).decode_ref(), "gqa8_decode")
    _no_device_error()


@pytest.mark.parametrize("D", [64, 128])
def test_decode_gqa8_split_and_window(D):
    """Eight heads per kv head through explicit splits and a sliding window,
    ragged lengths with empty and partial pages."""
    case = _decode_case([3000, 1, 0, 517, 2048, 33], 32, 4, D, seed=90 + D)
    ref = HostCase(case).decode_ref()
    for pps in (1, 7, 64):
        out = pkv.paged_attention_split(case.q, case.k_cache, case.v_cache, case.block_tables,
                                        case.context_lens, case.scale, pages_per_split=pps)
        assert_close(out, ref, f"gqa8 split pps={pps} D={D}")
    for window in (1, 100, 1000):
        out = pkv.paged_attention_window(case.q, case.k_cache, case.v_cache, case.block_tables,
                                         case.context_lens, case.scale, window)
        assert_close(out, HostCase(case).decode_window_ref(window), f"gqa8 window={window} D={D}")
    _no_device_error()


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("scale", [-0.125, -1.0])
def test_decode_negative_scale(D, scale):
    """A negative scale reverses the score order; one CTA per head group, explicit
    splits and a sliding window, against the oracle (pinned for negative scales)."""
    lens = [3000, 1, 0, 517, 2048, 33]
    pages = sum(-(-L // 16) for L in lens)
    case = wl.make_case(B=len(lens), Hq=16, Hkv=4, D=D, bs=16, lens=lens, seed=95 + D, device="cuda",
                        pool_blocks=pages + 3, scale=scale)
    host = HostCase(case)
    ref = host.decode_ref()
    out = pkv.paged_attention(case.q, case.k_cache, case.v_cache, case.block_tables, case.context_lens,
                              case.scale)
    assert_close(out, ref, f"negative scale {scale} D={D}")
    out = pkv.paged_attention_split(case.q, case.k_cache, case.v_cache, case.block_tables,
                                    case.context_lens, case.scale, pages_per_split=7)
    assert_close(out, ref, f"negative scale {scale} D={D} split")
    out = pkv.paged_attention_window(case.q, case.k_cache, case.v_cache, case.block_tables,
                                     case.context_lens, case.scale, 100)
    assert_close(out, host.decode_window_ref(100), f"negative scale {scale} D={D} window")
    _no_device_error()


def test_split_count_invariance():
    case = _decode_case([2000, 37, 900, 1], 8, 2, 128, seed=9)
    ref = HostCase(case).decode_ref()
    outs = []
    for pps in (1, 4, 16, 64, 1000):
        outs.append(pkv.paged_attention_split(case.q, case.k_cache, case.v_cache, case.block_tables,
                                              case.context_lens, case.scale, pages_per_split=pps))
        assert_close(outs[-1], ref, f"pps={pps}")
    for o in outs[1:]:
        d = (o.float() - outs[0].float()).abs().max().item()
        assert d <= 2 * (5e-3 + 1e-2 * outs[0].float().abs().max().item())


@pytest.mark.parametrize("Hq,Hkv,D", [(4, 2, 64), (16, 4, 128), (16, 8, 64)])
def test_decode_bad_block_id_is_reported(Hq, Hkv, D):
    case = _decode_case([40, 40], Hq, Hkv, D, seed=5)
    bt = case.block_tables.clone()
    bt[1, 1] = case.NB + 5                            # outside the pool
    pkv.paged_attention(case.q, case.k_cache, case.v_cache, bt, case.context_lens, case.scale)
    assert pkv.get_device_error() == 5


def test_decode_context_longer_than_table_is_reported():
    case = _decode_case([40], 4, 2, 64, seed=6)
    lens = torch.tensor([40 + 16 * 8], dtype=torch.int32, device="cuda")
    pkv.paged_attention(case.q, case.k_cache, case.v_cache, case.block_tables, lens, case.scale)
    assert pkv.get_device_error() == 5


def test_decode_context_longer_than_hint_is_reported():
    """max_context_len is a host-side hint the library never checks against the
    device lengths: the launch is sized from it, so a context longer than the
    hint (while the table holds it) must be reported, and the output stay finite."""
    lens = [6000, 700, 1600]
    case = _decode_case(lens, 32, 8, 128, seed=61)
    ref = HostCase(case).decode_ref()
    for hint in (1600, 3000):                   # the plan splits the hinted pages: 2 x 50, 2 x 94
        out = pkv.paged_attention(case.q, case.k_cache, case.v_cache, case.block_tables, case.context_lens,
                                  case.scale, max_context_len=hint)
        assert pkv.last_launch_count() == 2
        assert pkv.get_device_error() == 5, hint
        assert torch.isfinite(out.float()).all()
    # a hint too short to split leaves one CTA per head group over the whole
    # table: nothing is cut, and the result is exact
    out = pkv.paged_attention(case.q, case.k_cache, case.v_cache, case.block_tables, case.context_lens,
                              case.scale, max_context_len=100)
    assert pkv.last_launch_count() == 1
    assert_close(out, ref, "short hint, one split")
    _no_device_error()
    # with a true hint the split call is clean and matches the oracle
    out = pkv.paged_attention(case.q, case.k_cache, case.v_cache, case.block_tables, case.context_lens,
                              case.scale, max_context_len=6000)
    assert_close(out, ref, "true hint")
    _no_device_error()


def test_bounded_wait_gives_up_and_context_survives():
    pkv.selftest_wait_timeout(2000)                   # 2 ms limit on a barrier nobody completes
    assert pkv.get_device_error() == 4
    case = wl.workload("tiny_decode", device="cuda")
    out = pkv.paged_attention(case.q, case.k_cache, case.v_cache, case.block_tables, case.context_lens,
                              case.scale)
    assert_close(out, HostCase(case).decode_ref(), "after timeout")
    _no_device_error()


def test_decode_many_short_sequences():
    """B = 2100 short sequences (one CTA per head group, several waves),
    including empty and one-token contexts."""
    g = torch.Generator().manual_seed(77)
    lens = torch.randint(0, 40, (2100,), generator=g).tolist()
    for Hq, Hkv in ((8, 2), (16, 4)):
        case = _decode_case(lens, Hq, Hkv, 64, seed=77)
        ref = HostCase(case).decode_ref()
        out = pkv.paged_attention(case.q, case.k_cache, case.v_cache, case.block_tables, case.context_lens,
                                  case.scale)
        assert_close(out, ref, f"B=2100 Hq={Hq} Hkv={Hkv}")
        _no_device_error()


def test_decode_ragged_batch_auto_and_split_agree():
    """A ragged batch (empty, one-page and long contexts) through the automatic
    plan and an explicit split size, every row checked."""
    lens = [5000, 3, 0, 17, 1200, 4096, 640, 33] * 3
    case = _decode_case(lens, 32, 8, 128, seed=78)
    ref = HostCase(case).decode_ref()
    auto = pkv.paged_attention(case.q, case.k_cache, case.v_cache, case.block_tables, case.context_lens,
                               case.scale)
    assert_close(auto, ref, "auto")
    split = pkv.paged_attention_split(case.q, case.k_cache, case.v_cache, case.block_tables,
                                      case.context_lens, case.scale, pages_per_split=64)
    assert pkv.last_launch_count() == 2
    assert_close(split, ref, "split pps=64")
    _no_device_error()


# --------------------------------------------------------------------------- #
# sliding window                                                               #
# --------------------------------------------------------------------------- #

@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("window", [1, 15, 16, 17, 100, 1000])
def test_decode_window_edges(D, window):
    """Windows shorter and longer than the contexts, starting inside a page
    and on a page boundary; canaries in every slot outside the contexts."""
    case = _decode_case(EDGE_LENS, 8, 2, D, seed=300 + D + window)
    out = pkv.paged_attention_window(case.q, case.k_cache, case.v_cache, case.block_tables,
                                     case.context_lens, case.scale, window)
    assert_close(out, HostCase(case).decode_window_ref(window), f"window={window} D={D}")
    assert torch.count_nonzero(out[0]) == 0              # empty context -> zero row
    _no_device_error()


@pytest.mark.parametrize("window", [64, 500, 4096])
def test_decode_window_long_contexts_split(window):
    """Contexts far longer than the window: only the window's pages are read,
    split across CTAs when the window is long."""
    case = _decode_case([20000, 3, 5000, 777, 4096, 12345], 32, 8, 128, seed=310 + window)
    out = pkv.paged_attention_window(case.q, case.k_cache, case.v_cache, case.block_tables,
                                     case.context_lens, case.scale, window)
    if window == 4096:                                   # 257 window pages: split
        assert pkv.last_launch_count() == 2
    assert_close(out, HostCase(case).decode_window_ref(window), f"window={window}")
    _no_device_error()


def test_decode_window_rejects_zero():
    case = _decode_case([40], 4, 2, 64, seed=320)
    with pytest.raises(pkv.PagedKVError):
        pkv.paged_attention_window(case.q, case.k_cache, case.v_cache, case.block_tables,
                                   case.context_lens, case.scale, 0)


# --------------------------------------------------------------------------- #
# RoPE fused into the cache write                                              #
# --------------------------------------------------------------------------- #

@pytest.mark.parametrize("T,Hkv,D,bs,NB,base", [(37, 2, 64, 16, 9, 10000.0), (128, 8, 128, 16, 64, 500000.0),
                                               (6, 3, 256, 4, 4, 10000.0)])
def test_kv_cache_write_rope(T, Hkv, D, bs, NB, base):
    """Rotated K rows within half a bf16 step of the fp64 rotation (plus fp32
    slack on the pair); V rows and every untouched slot bit-exact."""
    g = torch.Generator(device="cuda").manual_seed(T * 3 + D)
    k_cache = torch.randn(NB, Hkv, bs, D, device="cuda", generator=g).to(torch.bfloat16)
    v_cache = torch.randn(NB, Hkv, bs, D, device="cuda", generator=g).to(torch.bfloat16)
    key = torch.randn(T, Hkv, D, device="cuda", generator=g).to(torch.bfloat16)
    val = torch.randn(T, Hkv, D, device="cuda", generator=g).to(torch.bfloat16)
    gc = torch.Generator().manual_seed(T)
    slots = torch.randperm(NB * bs, generator=gc)[:T].to(torch.int64)
    slots[::5] = -1
    pos = torch.randint(0, 131072, (T,), generator=gc, dtype=torch.int64)
    pos[0] = 0
    k_before, v_before = bf16_bits(k_cache).copy(), bf16_bits(v_cache).copy()
    pkv.kv_cache_write_rope(key, val, k_cache, v_cache, slots.cuda(), pos.cuda(), base)
    assert pkv.last_launch_count() == 1
    want = oracle.get().rope_rows(bf16_bits(key), pos.numpy(), base)       # fp64 [T, Hkv, D]
    kb, vb = bf16_bits(k_cache), bf16_bits(v_cache)
    x = np.abs(bf16_bits_to_f64(bf16_bits(key)))
    half = D // 2
    pair = x[..., :half] + x[..., half:]
    pair = np.concatenate([pair, pair], axis=-1)
    for t, sl in enumerate(slots.tolist()):
        if sl < 0:
            continue
        blk, off = sl // bs, sl % bs
        got = bf16_bits_to_f64(kb[blk, :, off])
        bound = np.abs(want[t]) * 2.0 ** -8 + pair[t] * 2.0 ** -20
        assert np.all(np.abs(got - want[t]) <= bound), (t, np.abs(got - want[t]).max())
        assert np.array_equal(vb[blk, :, off], bf16_bits(val)[t])
        k_before[blk, :, off] = kb[blk, :, off]
        v_before[blk, :, off] = vb[blk, :, off]
    assert np.array_equal(kb, k_before) and np.array_equal(vb, v_before)
    _no_device_error()


def test_rope_write_then_decode():
    """Decode over a cache whose newest rows were rotated on the way in,
    against the oracle's own rotated write (nothing taken from the GPU)."""
    case = wl.workload("llama3_8b_decode", device="cuda", B=16, lens=[4096] * 16)
    host = HostCase(case)
    pos = (case.context_lens.to(torch.int64) - 1)                       # the new token's position
    pkv.kv_cache_write_rope(case.new_key, case.new_value, case.k_cache, case.v_cache, case.slot_mapping, pos,
                            500000.0)
    out = pkv.paged_attention(case.q, case.k_cache, case.v_cache, case.block_tables, case.context_lens,
                              case.scale, max_context_len=4096)
    oracle.get().kv_cache_write_rope(bf16_bits(case.new_key), bf16_bits(case.new_value), host.k, host.v,
                                     case.slot_mapping.cpu().numpy(), pos.cpu().numpy(), 500000.0)
    host.written = True
    assert_close(out, host.decode_ref(), "rope write + decode")
    _no_device_error()
