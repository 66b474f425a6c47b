"""Shared cache blocks on the host: the reference model in ``oracle.blocks``
pinned by hand-worked scenarios and a holder ledger, then the library's C++
allocator (through the C ABI, no GPU) checked against the model step by step."""
import random
import threading

import numpy as np
import pytest

import paged_kv_cache_477_b200 as pkv
from oracle.blocks import BlockPool, copy_blocks


# --------------------------------------------------------------------------- model pins

def test_model_parallel_sampling_scenario_by_hand():
    """A 37-token prompt in 16-row blocks takes blocks 0, 1, 2 (the last holds 5
    rows).  Four samples fork from it: each shares the three blocks; before
    writing its next token each sample copies-on-write the partial block."""
    pool = BlockPool(8)
    prompt = pool.alloc(3)
    assert prompt == [0, 1, 2]
    assert pool.share(prompt * 3)                     # three more holders (4 samples)
    assert [pool.refcount(b) for b in range(8)] == [4, 4, 4, 0, 0, 0, 0, 0]
    # samples 0..2 get private copies of block 2; the last holder writes in place
    assert pool.cow(2) == (3, True)
    assert pool.cow(2) == (4, True)
    assert pool.cow(2) == (5, True)
    assert pool.cow(2) == (2, False)
    assert [pool.refcount(b) for b in range(8)] == [4, 4, 1, 1, 1, 1, 0, 0]
    assert pool.num_free() == 2
    # sample 1 finishes: its blocks 0, 1 and 4 lose one holder; 4 is free again
    assert pool.release([0, 1, 4])
    assert [pool.refcount(b) for b in range(8)] == [3, 3, 1, 1, 0, 1, 0, 0]
    assert pool.alloc(1) == [4]                       # the freed block is reused first
    pool.check()


def test_model_all_or_nothing():
    pool = BlockPool(4)
    a = pool.alloc(3)
    assert pool.alloc(2) is None and pool.num_free() == 1       # not enough: nothing taken
    assert not pool.share([a[0], 3])                            # 3 is free: nothing shared
    assert pool.refcount(a[0]) == 1
    assert not pool.release([a[1], a[1]])                       # one holder, two releases
    assert pool.refcount(a[1]) == 1
    assert not pool.release([a[2], 7]) and pool.refcount(a[2]) == 1
    assert pool.share([a[0]]) and pool.alloc(1) == [3]
    assert pool.cow(a[0]) is None                               # shared, but nothing free
    assert pool.refcount(a[0]) == 2
    assert pool.cow(3) == (3, False)
    assert pool.cow(-1) is None and pool.refcount(-1) == -1 and pool.refcount(4) == -1
    pool.check()


def _random_ops(seed, nb, steps):
    """A seeded run of sequences that allocate, fork, write (copy-on-write) and
    finish; yields (op, args) and keeps an independent ledger of holdings."""
    rng = random.Random(seed)
    seqs = []                       # each a list of block ids it holds
    for _ in range(steps):
        r = rng.random()
        if r < 0.3 or not seqs:
            yield "alloc", rng.randint(0, 4), seqs
        elif r < 0.5:
            yield "fork", rng.randrange(len(seqs)), seqs
        elif r < 0.75:
            yield "write", rng.randrange(len(seqs)), seqs
        elif r < 0.85:
            yield "bad", rng.choice([-3, nb, nb + 5]), seqs
        else:
            yield "finish", rng.randrange(len(seqs)), seqs


def _drive(pool, seed, nb, steps, other=None):
    """Apply the seeded run to ``pool`` (and ``other`` in lockstep, comparing)."""
    for op, arg, seqs in _random_ops(seed, nb, steps):
        if op == "alloc":
            got = pool.alloc(arg)
            if other is not None:
                want = other.alloc(arg)
                assert got == want
            if got is not None:
                seqs.append(list(got))
        elif op == "fork":
            ok = pool.share(seqs[arg])
            if other is not None:
                assert ok == other.share(seqs[arg])
            assert ok
            seqs.append(list(seqs[arg]))
        elif op == "write" and seqs[arg]:
            b = seqs[arg][-1]
            got = pool.cow(b)
            if other is not None:
                assert got == other.cow(b)
            if got is not None:
                seqs[arg][-1] = got[0]
                assert got[1] == (got[0] != b)
        elif op == "bad":
            assert not pool.share([arg]) and not pool.release([arg]) and pool.cow(arg) is None
            if other is not None:
                assert not other.share([arg]) and not other.release([arg]) and other.cow(arg) is None
        elif op == "finish":
            ok = pool.release(seqs[arg])
            if other is not None:
                assert ok == other.release(seqs[arg])
            assert ok
            seqs.pop(arg)
        # the ledger: every block's count is the number of its holders
        held = np.zeros(nb, dtype=np.int64)
        for s in seqs:
            for b in s:
                held[b] += 1
        assert [pool.refcount(b) for b in range(nb)] == held.tolist()
        assert pool.num_free() == int((held == 0).sum())
        if other is not None:
            assert other.num_free() == pool.num_free()


@pytest.mark.parametrize("seed", range(6))
def test_model_matches_holder_ledger(seed):
    pool = BlockPool(24)
    _drive(pool, seed, 24, 400)
    pool.check()


def test_model_copy_blocks_by_hand():
    k = np.arange(4 * 6, dtype=np.uint16).reshape(4, 2, 3)
    v = -np.arange(4 * 6, dtype=np.int64).reshape(4, 2, 3)
    k0, v0 = k.copy(), v.copy()
    assert copy_blocks([k, v], [[2, 0], [1, 3], [0, 9]]) == 1
    assert np.array_equal(k[0], k0[2]) and np.array_equal(v[0], v0[2])
    assert np.array_equal(k[3], k0[1]) and np.array_equal(v[3], v0[1])
    assert np.array_equal(k[1:3], k0[1:3]) and np.array_equal(v[1:3], v0[1:3])


# --------------------------------------------------------------------------- the library

def test_library_allocator_matches_model_scenario():
    a = pkv.BlockAllocator(8)
    prompt = a.alloc(3)
    assert prompt == [0, 1, 2]
    a.share(prompt * 3)
    assert [a.cow(2) for _ in range(4)] == [(3, True), (4, True), (5, True), (2, False)]
    a.release([0, 1, 4])
    assert [a.refcount(b) for b in range(8)] == [3, 3, 1, 1, 0, 1, 0, 0]
    assert a.alloc(1) == [4] and a.num_free() == 2
    a.close()


class _LibAsModel:
    """The library allocator with the model's return conventions (None or
    False where the library reports an error)."""

    def __init__(self, nb):
        self.a = pkv.BlockAllocator(nb)

    def _call(self, f, *args):
        try:
            out = f(*args)
            return True if out is None else out
        except pkv.PagedKVError:
            return None

    def alloc(self, n):
        return self._call(self.a.alloc, n)

    def share(self, ids):
        return self._call(self.a.share, ids) is not None

    def release(self, ids):
        return self._call(self.a.release, ids) is not None

    def cow(self, b):
        return self._call(self.a.cow, b)

    def num_free(self):
        return self.a.num_free()

    def refcount(self, b):
        return self.a.refcount(b)


@pytest.mark.parametrize("seed", range(6))
def test_library_allocator_matches_model_random(seed):
    lib = _LibAsModel(24)
    _drive(lib, seed, 24, 400, other=BlockPool(24))
    lib.a.close()


def test_library_allocator_errors():
    a = pkv.BlockAllocator(2)
    with pytest.raises(pkv.PagedKVError, match="not enough free blocks"):
        a.alloc(3)
    assert a.num_free() == 2
    ids = a.alloc(2)
    with pytest.raises(pkv.PagedKVError, match="not enough free blocks"):
        a.share([ids[0]]) or a.cow(ids[0])
    assert a.refcount(ids[0]) == 2
    with pytest.raises(pkv.PagedKVError):
        a.release([ids[1], ids[1]])
    assert a.refcount(ids[1]) == 1
    with pytest.raises(pkv.PagedKVError):
        a.share([5])
    assert a.refcount(5) == -1 and a.refcount(-1) == -1
    with pytest.raises(pkv.PagedKVError):
        pkv.BlockAllocator(-1)
    empty = pkv.BlockAllocator(0)
    assert empty.num_free() == 0 and empty.alloc(0) == []
    a.close()
    empty.close()


def test_library_allocator_threads():
    """Four host threads fork, copy-on-write and finish sequences on one
    allocator; at the end every block is free again and counts are 0."""
    nb = 64
    a = pkv.BlockAllocator(nb)
    errors = []

    def worker(seed):
        rng = random.Random(seed)
        try:
            for _ in range(300):
                try:
                    base = a.alloc(rng.randint(1, 3))
                except pkv.PagedKVError:
                    continue
                a.share(base)
                fork = list(base)
                try:
                    fork[-1], must = a.cow(fork[-1])
                    assert must
                except pkv.PagedKVError:
                    pass                                # nothing free: keeps sharing
                a.release(base)
                a.release(fork)
        except Exception as e:                          # noqa: BLE001 -- reported below
            errors.append(e)

    threads = [threading.Thread(target=worker, args=(s,)) for s in range(4)]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    assert not errors, errors
    assert a.num_free() == nb
    assert all(a.refcount(b) == 0 for b in range(nb))
    a.close()


def test_library_copy_blocks_rejects_bad_arguments_without_launching():
    """Argument checks that return before any device work (no GPU needed)."""
    lib = pkv.load_library()
    assert lib.pkv_copy_blocks(None, None, 0, None, 1, 4, None) == 1          # block_bytes 0
    assert lib.pkv_copy_blocks(None, None, 24, None, 1, 4, None) == 1         # not a multiple of 16
    assert lib.pkv_copy_blocks(None, None, 32, None, -1, 4, None) == 1        # n < 0
    assert lib.pkv_copy_blocks(None, None, 32, None, 0, 4, None) == 0         # nothing to copy
    assert lib.pkv_copy_blocks(None, None, 32, None, 2, 4, None) == 1         # null pools
