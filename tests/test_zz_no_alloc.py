"""The allocation-free split-KV decode entry point (GPU).

pkv_paged_attention_split_noalloc serves callers that cannot allocate device
memory -- plugins whose enqueue hook forbids it, serving loops that cannot
afford the synchronisation a cudaMalloc may bring, processes whose device memory
another allocator has already reserved.  It keeps its split partials in a
static array inside the library instead of a caller workspace.  This file runs
last (its name sorts last) so a failure here comes after every other test.
"""
import ctypes

import pytest
import torch

import paged_kv_cache_477_b200 as pkv
from paged_kv_cache_477_b200 import workloads as wl
from parity import ATOL, RTOL, HostCase, assert_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _library():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from paged_kv_cache_477_b200 import build
    build.build()
    pkv.load_library()
    pkv.get_device_error()
    yield


def _within(a: torch.Tensor, ref: torch.Tensor):
    a, ref = a.float(), ref.float()
    assert torch.isfinite(a).all()
    assert ((a - ref).abs() <= ATOL + RTOL * ref.abs()).all(), float((a - ref).abs().max())


def test_noalloc_matches_oracle_and_workspace_entry_point_twice():
    """Two calls in a row share the static array; each result matches the fp64
    oracle and the entry point that takes a caller workspace."""
    case = wl.make_case(B=6, Hq=32, Hkv=8, D=128, bs=16, lens=[3000, 1, 517, 2048, 33, 1200], seed=77,
                        device="cuda")
    ref = HostCase(case).decode_ref()
    pps = 16
    ws_out = pkv.paged_attention_split(case.q, case.k_cache, case.v_cache, case.block_tables,
                                       case.context_lens, case.scale, pages_per_split=pps)
    torch.cuda.synchronize()
    for _ in range(2):
        out = torch.full_like(case.q, float("nan"))
        pkv.paged_attention_split_noalloc(case.q, case.k_cache, case.v_cache, case.block_tables,
                                          case.context_lens, case.scale, pages_per_split=pps, out=out)
        assert pkv.last_launch_count() == 2  # split partials + merge
        torch.cuda.synchronize()
        assert_close(out, ref, "no-alloc split decode")
        _within(out, ws_out)
    assert pkv.get_device_error() == 0


def test_noalloc_second_shape_after_first():
    """A different shape right after: the array keeps the last call's contents,
    which must not leak into this result."""
    case = wl.make_case(B=3, Hq=32, Hkv=8, D=64, bs=16, lens=[700, 4096, 64], seed=78, device="cuda")
    ref = HostCase(case).decode_ref()
    for _ in range(2):
        out = pkv.paged_attention_split_noalloc(case.q, case.k_cache, case.v_cache, case.block_tables,
                                                case.context_lens, case.scale, pages_per_split=8)
        torch.cuda.synchronize()
        assert_close(out, ref, "no-alloc split decode, D=64")
    assert pkv.get_device_error() == 0


def test_noalloc_rejects_requests_beyond_the_static_array():
    lib = pkv.load_library()
    B, Hq, D, pps, MB = 64, 32, 128, 1, 256          # 256 splits of partials: far over 8 MiB
    need = lib.pkv_split_workspace_size(B, Hq, D, MB // pps)
    assert need > pkv.NOALLOC_SCRATCH_BYTES
    dummy = torch.empty(16, dtype=torch.uint8, device="cuda")
    p = dummy.data_ptr()
    rc = lib.pkv_paged_attention_split_noalloc(p, p, p, p, p, MB, p, B, Hq, 8, D, 4, 16, 1.0, 0, pps, 0,
                                               torch.cuda.current_stream().cuda_stream)
    assert rc == 6                                   # PKV_ERR_WORKSPACE, nothing launched
    assert lib.pkv_last_launch_count() == 0
