"""GPU parity of the tcgen05 chunked causal prefill against the fp64 oracle.

The chunk's K/V rows are written by the library's cache write first, as a
caller would; the oracle applies its own cache write to the generator's
pre-write pool.  Attention outputs must satisfy |gpu - ref| <= 5e-3 + 1e-2 |ref|.
"""
import pytest
import torch

import paged_kv_cache_477_b200 as pkv
from paged_kv_cache_477_b200 import workloads as wl
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


def _run(case):
    host = HostCase(case)
    pkv.kv_cache_write(case.new_key, case.new_value, case.k_cache, case.v_cache, case.slot_mapping)
    out = pkv.paged_attention_prefill(case.q, case.query_start_loc, case.k_cache, case.v_cache,
                                      case.block_tables, case.context_lens, case.scale, case.max_q_len)
    assert pkv.last_launch_count() == 1
    host.apply_write()
    return out, host


def _prefill_case(lens, qlens, Hq, Hkv, seed, extra_blocks=2, D=128):
    pages = sum(-(-L // 16) for L in lens)
    return wl.make_case(kind="prefill", B=len(lens), Hq=Hq, Hkv=Hkv, D=D, bs=16, lens=lens, q_len=qlens,
                        seed=seed, device="cuda", pool_blocks=pages + extra_blocks)


@pytest.mark.parametrize("D", [128, 64])
@pytest.mark.parametrize("Hq,Hkv", [(8, 2), (32, 8), (4, 4), (16, 8), (16, 2)])
def test_prefill_small_full(Hq, Hkv, D):
    # ragged chunks, partial last pages (NaN canaries in the tails), a chunk that
    # is the whole context, single-token chunks, several Q tiles per sequence
    lens = [200, 77, 300, 1, 129, 45]
    qlens = [130, 77, 33, 1, 1, 45]
    case = _prefill_case(lens, qlens, Hq, Hkv, seed=500 + Hq + Hkv + D, D=D)
    out, host = _run(case)
    ref, tok = host.prefill_ref()
    assert_close(out[tok], ref, f"prefill Hq={Hq} Hkv={Hkv} D={D}")
    assert pkv.get_device_error() == 0


def test_prefill_llama32_1b_shaped_chunks():
    """Head size 64 at the Llama-3.2-1B shape (32 q / 8 kv heads): 512-token
    chunks after cached context, every row checked."""
    case = _prefill_case([1536, 700, 512], [512, 300, 512], 32, 8, seed=620, D=64)
    out, host = _run(case)
    ref, tok = host.prefill_ref()
    assert_close(out[tok], ref, "prefill D=64 Llama-3.2-1B shape")
    assert pkv.get_device_error() == 0


def test_prefill_empty_chunk_and_long_chunk():
    lens = [16, 700, 64]
    qlens = [0, 700, 2]          # a sequence with nothing new, a 700-token chunk, a short one
    case = _prefill_case(lens, qlens, 32, 8, seed=600)
    out, host = _run(case)
    ref, tok = host.prefill_ref()
    assert_close(out[tok], ref, "prefill empty/long chunk")
    assert pkv.get_device_error() == 0


def test_prefill_workload_full():
    """The bench's prefill workload (B=4, 512-token chunks after 3584 cached
    tokens, 32 q / 8 kv heads): every query row of every head against the
    oracle's chunked causal prefill."""
    case = wl.workload("chunked_prefill", device="cuda")
    out, host = _run(case)
    ref, tok = host.prefill_ref()
    assert len(tok) == case.q.shape[0] == 2048
    assert_close(out[tok], ref, "chunked_prefill")
    assert pkv.get_device_error() == 0


def test_prefill_matches_decode_on_last_row():
    """The last query of a chunk is a decode step over the whole context."""
    case = _prefill_case([513, 1000], [100, 513], 32, 8, seed=601)
    out, host = _run(case)
    qsl = host.qsl
    last = [int(qsl[1]) - 1, int(qsl[2]) - 1]
    q_dec = case.q[last].contiguous()
    dec = pkv.paged_attention(q_dec, case.k_cache, case.v_cache, case.block_tables, case.context_lens,
                              case.scale)
    d = (out[last].float() - dec.float()).abs().max().item()
    assert d <= 2e-2, d


def test_prefill_rejects_unsupported_shapes_and_bad_scales():
    case = _prefill_case([32], [16], 8, 2, seed=602)
    for scale, status in ((float("nan"), 1), (float("inf"), 1), (float("-inf"), 1)):
        with pytest.raises(pkv.PagedKVError) as e:
            pkv.paged_attention_prefill(case.q, case.query_start_loc, case.k_cache, case.v_cache,
                                        case.block_tables, case.context_lens, scale, case.max_q_len)
        assert e.value.status == status
        assert pkv.last_launch_count() == 0
    wide = _prefill_case([32], [16], 129, 1, seed=604)      # 129 query heads per kv head: more than a tile
    with pytest.raises(pkv.PagedKVError) as e:
        pkv.paged_attention_prefill(wide.q, wide.query_start_loc, wide.k_cache, wide.v_cache, wide.block_tables,
                                    wide.context_lens, wide.scale, wide.max_q_len)
    assert e.value.status == 2
    assert pkv.last_launch_count() == 0


@pytest.mark.parametrize("D", [128, 64])
@pytest.mark.parametrize("Hq,Hkv", [(12, 4), (6, 2), (10, 2), (7, 1), (24, 2)])
def test_prefill_group_sizes_not_dividing_128(Hq, Hkv, D):
    """Groups of 3, 5, 7 and 12 query heads: a tile holds floor(128 / G) whole
    positions and its last rows stay idle; chunks across several tiles,
    partial last pages."""
    lens = [300, 77, 129, 45]
    qlens = [130, 77, 1, 45]
    case = _prefill_case(lens, qlens, Hq, Hkv, seed=700 + Hq + D, D=D)
    out, host = _run(case)
    ref, tok = host.prefill_ref()
    assert_close(out[tok], ref, f"prefill G={Hq // Hkv} D={D}")
    assert pkv.get_device_error() == 0


@pytest.mark.parametrize("D", [128, 64])
@pytest.mark.parametrize("scale", [-0.125, -1.0])
def test_prefill_negative_scale(D, scale):
    """A negative scale reverses the score order (the row maximum of the scaled
    scores comes from the raw minimum); ragged chunks and partial pages."""
    lens = [300, 77, 129, 1000]
    qlens = [130, 77, 1, 257]
    pages = sum(-(-L // 16) for L in lens)
    case = wl.make_case(kind="prefill", B=4, Hq=16, Hkv=4, D=D, bs=16, lens=lens, q_len=qlens,
                        seed=605 + D, device="cuda", pool_blocks=pages + 2, scale=scale)
    out, host = _run(case)
    ref, tok = host.prefill_ref()
    assert_close(out[tok], ref, f"prefill scale={scale} D={D}")
    assert pkv.get_device_error() == 0


def test_prefill_zero_scale_gives_mean_of_visible_values():
    case = wl.make_case(kind="prefill", B=2, Hq=8, Hkv=2, D=128, bs=16, lens=[150, 40], q_len=[70, 40],
                        seed=603, device="cuda", scale=0.0)
    out, host = _run(case)
    ref, tok = host.prefill_ref()
    assert_close(out[tok], ref, "prefill scale=0")
    assert pkv.get_device_error() == 0


@pytest.mark.parametrize("D", [128, 64])
@pytest.mark.parametrize("window", [1, 17, 128, 129, 300, 5000])
def test_prefill_window(window, D):
    """Sliding window: tiles below every row's window skipped, edge tiles masked
    per row (windows shorter than a tile, tile-aligned, spanning tiles, wider
    than the context)."""
    lens = [700, 77, 1300, 45]
    qlens = [300, 77, 129, 1]
    case = _prefill_case(lens, qlens, 16, 4, seed=560 + window + D, D=D)
    host = HostCase(case)
    pkv.kv_cache_write(case.new_key, case.new_value, case.k_cache, case.v_cache, case.slot_mapping)
    out = pkv.paged_attention_prefill_window(case.q, case.query_start_loc, case.k_cache, case.v_cache,
                                             case.block_tables, case.context_lens, case.scale, case.max_q_len,
                                             window)
    assert pkv.last_launch_count() == 1
    host.apply_write()
    ref, tok = host.prefill_ref(window=window)
    assert_close(out[tok], ref, f"prefill window={window}")
    assert pkv.get_device_error() == 0
