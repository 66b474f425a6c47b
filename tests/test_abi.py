"""The C-ABI library builds, loads and exports every symbol its header declares;
host-side argument checks answer without touching a GPU (CPU only)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER_DIR = os.path.join(ROOT, "include")


def declared_symbols():
    names = set()
    for fn in os.listdir(HEADER_DIR):
        if fn.endswith(".h"):
            text = open(os.path.join(HEADER_DIR, fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(pkv_\w+)\s*\(", text))
    return sorted(names)


@pytest.fixture(scope="module")
def lib():
    from paged_kv_cache_477_b200 import build, load_library
    build.build()
    return load_library()


def test_header_declares_the_three_calls():
    names = declared_symbols()
    for n in ("pkv_kv_cache_write", "pkv_paged_attention", "pkv_paged_attention_prefill"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    missing = [n for n in declared_symbols() if not hasattr(lib, n)]
    assert not missing, f"declared but not exported: {missing}"


def test_binding_covers_every_symbol():
    from paged_kv_cache_477_b200 import EXPORTS
    assert sorted(EXPORTS) == declared_symbols()


def test_status_strings(lib):
    for code in range(8):
        assert lib.pkv_status_string(code)


def test_host_validation_needs_no_gpu(lib):
    P = None
    # unsupported dtype
    assert lib.pkv_kv_cache_write(P, P, 8, 8, P, P, P, 1, 1, 8, 1, 16, 1, P) == 2
    # D not a multiple of 8
    assert lib.pkv_kv_cache_write(P, P, 12, 12, P, P, P, 1, 1, 12, 1, 16, 0, P) == 2
    # null pointers with T > 0
    assert lib.pkv_kv_cache_write(P, P, 8, 8, P, P, P, 1, 1, 8, 1, 16, 0, P) == 1
    # T = 0 is a no-op
    assert lib.pkv_kv_cache_write(P, P, 8, 8, P, P, P, 0, 1, 8, 1, 16, 0, P) == 0
    # decode: head_dim 96 unsupported, Hq % Hkv != 0 invalid, block size 32 unsupported
    args = lambda B, Hq, Hkv, D, bs: (P, P, P, P, P, 4, P, B, Hq, Hkv, D, 4, bs, 1.0, 0, P, 0, 0, P)
    assert lib.pkv_paged_attention(*args(1, 4, 2, 96, 16)) == 2
    assert lib.pkv_paged_attention(*args(1, 3, 2, 64, 16)) == 1
    assert lib.pkv_paged_attention(*args(1, 4, 2, 64, 32)) == 2
    assert lib.pkv_paged_attention(*args(0, 4, 2, 64, 16)) == 0
    assert lib.pkv_paged_attention(*args(1, 4, 2, 64, 16)) == 1   # null pointers
    # explicit split size must be positive
    assert lib.pkv_paged_attention_split(P, P, P, P, P, 4, P, 1, 4, 2, 64, 4, 16, 1.0, 0, 0,
                                         P, 0, 0, P) == 1
    # workspace sizes are pure host arithmetic
    assert lib.pkv_split_workspace_size(2, 4, 64, 1) == 0
    assert lib.pkv_split_workspace_size(2, 4, 64, 3) == 2 * 4 * 3 * 64 * 4 + 256  # partials + lse
    # a pool with no blocks cannot back a non-empty block table
    assert lib.pkv_paged_attention(P, P, P, P, P, 4, P, 1, 4, 2, 64, 0, 16, 1.0, 0, P, 0, 0, P) == 1
    # the window entry points validate on the host and launch nothing (here: null pointers, window 0)
    assert lib.pkv_paged_attention_window(P, P, P, P, P, 4, P, 1, 4, 2, 64, 4, 16, 1.0, 0, P, 0, 0, P) == 1
    assert lib.pkv_paged_attention_int8_window(P, P, P, P, P, P, P, 4, P, 1, 4, 2, 64, 4, 16, 1.0, 0, P, 0,
                                               P) == 1
    # prefill: head sizes 64 and 128 only, block size 16 only
    pf = lambda D, bs: (P, P, P, P, P, P, 4, P, 1, 8, 8, 4, 2, D, 4, bs, 1.0, 0, P)
    assert lib.pkv_paged_attention_prefill(*pf(96, 16)) == 2
    assert lib.pkv_paged_attention_prefill(*pf(64, 32)) == 2
    assert lib.pkv_paged_attention_prefill(*pf(64, 16)) == 1      # null pointers


def test_product_path_fails_loudly_without_library(tmp_path):
    import paged_kv_cache_477_b200 as pkv
    with pytest.raises(RuntimeError):
        pkv.load_library(str(tmp_path / "missing.so"))
