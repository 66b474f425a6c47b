"""Pins that tie the fp64 oracle to something other than itself.

Each pin is a function ``pin_xxx(orc)`` that raises ``AssertionError`` when the
oracle ``orc`` is wrong.  They are run twice: against the real oracle (all must
pass) and against builds with one planted mistake each (at least one must
fail), so a plausible slip -- a wrong head map, a swapped page/row index, a
dropped scale or normaliser, an off-by-one causal edge, the wrong cache layout,
a flipped merge sign -- cannot hide.

What pins what (the method: paged gather through a block table, Tiny-Infer page
section "分页KV缓存：借鉴操作系统的内存管理"; exact softmax attention,
"5 Fun Projects for LLM Inference Engineering" section 2):

* closed-form golden cases (tests/golden) -- hand-derived softmax values;
* brute force -- an independent NumPy full-matrix formulation;
* paged == contiguous -- a static cache written into shuffled pages by the
  oracle's own scatter gives bit-identical results;
* scatter/gather identity, skip of negative slots, rejection of slots outside
  the pool;
* single key -> its V row; identical keys -> mean of V; scale 0 -> mean of V;
* one-hot V exposes the probability row: it sums to 1 and matches exp/sum;
* causal: future keys do not matter; the last query of a chunk equals decode;
* GQA equals materialised MHA; G = 1 is plain MHA;
* split-KV partials merged by log-sum-exp equal the plain result;
* an empty context gives a zero row;
* a negative scale: a closed form (weights sigmoid(-2) and sigmoid(2)), the
  identity (-scale, -q) == (scale, q) bit for bit, and brute force;
* INT8 cache (one fp32 scale per token row, the reading of the Tiny-Infer
  page's section "推测性解码与INT8量化"): rows built as k * 2^-e decode to
  exactly k and 2^-e; ties round to even; every value is within scale/2 of
  its code; a zero row gives zero codes and scale; attention over the int8
  pool equals NumPy brute force over the dequantised values, and equals the
  pinned bf16 path bit for bit when the values are bf16-exact;
* sliding window W (a query at p sees keys p - W < j <= p; the reading of the
  inference-lab page's sliding-window cache): W >= L is full attention bit for
  bit, W = 1 returns the last key's V row, decode equals full attention over a
  contiguous cache holding only the last W keys, the last query of a prefill
  chunk equals windowed decode, and NumPy brute force with a banded mask agrees;
* RoPE written with K (the fused-ops page's fusion of RoPE into the step
  before; Llama's form, element i paired with i + D/2, angle pos*base^(-2i/D)):
  position 0 is the identity; a unit vector at D = 4 gives cos/sin of the
  expected angles in the expected slots (pairing, sign and both frequencies);
  pair norms are kept; dot products depend only on the position difference;
  the cache write stores bf16 of the fp64 rotation, copies V bit for bit and
  leaves every other slot alone.
"""
from __future__ import annotations

import json
import os

import numpy as np

from oracle import bf16_bits_to_f64
from oracle import brute

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "closed_form_cases.json")


# --------------------------------------------------------------------------- #
# small helpers (numpy only; bf16 values as uint16 bit patterns)               #
# --------------------------------------------------------------------------- #

def f32_to_bf16_bits(x) -> np.ndarray:
    """Round float values to bf16 (round to nearest even) and return the bits."""
    f = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    u = f.view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return rounded.astype(np.uint16)


def rand_bits(rng, shape, std=1.0):
    return f32_to_bf16_bits(rng.standard_normal(shape) * std)


def make_paged(rng, lens, Hkv, D, bs, extra_blocks=3):
    """Random paged pool for the given lengths; NaN in every unused slot."""
    pages = [-(-L // bs) for L in lens]
    NB = sum(pages) + extra_blocks
    perm = rng.permutation(NB)
    MB = max(pages + [1])
    bt = np.full((len(lens), MB), -1, dtype=np.int32)
    off = 0
    for b, p in enumerate(pages):
        bt[b, :p] = perm[off:off + p]
        off += p
    k = rand_bits(rng, (NB, Hkv, bs, D))
    v = rand_bits(rng, (NB, Hkv, bs, D))
    valid = np.zeros((NB, bs), dtype=bool)
    for b, L in enumerate(lens):
        for j in range(L):
            valid[bt[b, j // bs], j % bs] = True
    bad = np.broadcast_to((~valid)[:, None, :, None], k.shape)
    k[bad] = 0x7FC0
    v[bad] = 0x7FC0
    return k, v, bt, np.asarray(lens, dtype=np.int32)


def scatter_contiguous(orc, kc, vc, lens, bs, rng, extra_blocks=2):
    """Write a contiguous [B, Lmax, Hkv, D] cache into shuffled pages using the
    oracle's own cache write; returns (k_cache, v_cache, block_tables)."""
    B, Lmax, Hkv, D = kc.shape
    pages = [-(-int(L) // bs) for L in lens]
    NB = sum(pages) + extra_blocks
    perm = rng.permutation(NB)
    MB = max(pages + [1])
    bt = np.full((B, MB), -1, dtype=np.int32)
    off = 0
    for b, p in enumerate(pages):
        bt[b, :p] = perm[off:off + p]
        off += p
    k_cache = np.full((NB, Hkv, bs, D), 0x7FC0, dtype=np.uint16)
    v_cache = np.full((NB, Hkv, bs, D), 0x7FC0, dtype=np.uint16)
    for b in range(B):
        L = int(lens[b])
        if L == 0:
            continue
        slots = np.array([bt[b, j // bs] * bs + j % bs for j in range(L)], dtype=np.int64)
        orc.kv_cache_write(np.ascontiguousarray(kc[b, :L]), np.ascontiguousarray(vc[b, :L]),
                           k_cache, v_cache, slots)
    return k_cache, v_cache, bt


# --------------------------------------------------------------------------- #
# pins                                                                         #
# --------------------------------------------------------------------------- #

def pin_golden_closed_form(orc):
    cases = json.load(open(GOLDEN))["cases"]
    rng = np.random.default_rng(7)
    for c in cases:
        keys = np.asarray(c["keys"], dtype=np.float32)
        vals = np.asarray(c["values"], dtype=np.float32)
        q = np.asarray(c["q"], dtype=np.float32)
        L, D = keys.shape
        Q = q.shape[0]
        assert c["query_positions"] == list(range(L - Q, L))
        kb, vb = f32_to_bf16_bits(keys), f32_to_bf16_bits(vals)
        assert np.array_equal(bf16_bits_to_f64(kb), keys.astype(np.float64)), "inputs must be bf16-exact"
        bs = 2
        kc, vc, bt = scatter_contiguous(orc, kb[None, :, None, :], vb[None, :, None, :], [L], bs, rng)
        qb = f32_to_bf16_bits(q)[:, None, :]                      # [Q, 1, D]
        expected = np.asarray(c["expected"], dtype=np.float64)
        out = orc.paged_attention_prefill(qb, np.array([0, Q], np.int32), kc, vc, bt,
                                          np.array([L], np.int32), c["scale"])
        np.testing.assert_allclose(out[:, 0, :], expected, rtol=0, atol=1e-15, err_msg=c["name"])
        # the last query is a decode over all L keys
        dec = orc.paged_attention(qb[-1:], kc, vc, bt, np.array([L], np.int32), c["scale"])
        np.testing.assert_allclose(dec[0, 0], expected[-1], rtol=0, atol=1e-15, err_msg=c["name"])


def pin_brute_force_decode(orc):
    rng = np.random.default_rng(11)
    for (lens, Hq, Hkv, D, bs) in [([37, 100], 4, 2, 64, 16), ([1, 5, 16, 17, 33], 8, 2, 32, 4),
                                   ([70, 3], 6, 3, 16, 8), ([20], 4, 4, 8, 16)]:
        k, v, bt, cl = make_paged(rng, lens, Hkv, D, bs)
        q = rand_bits(rng, (len(lens), Hq, D))
        scale = float(np.float32(1.0) / np.sqrt(np.float32(D)))
        got = orc.paged_attention(q, k, v, bt, cl, scale)
        ref = brute.paged_attention(q, k, v, bt, cl, scale)
        np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


def pin_brute_force_prefill(orc):
    rng = np.random.default_rng(12)
    for (lens, qlens, Hq, Hkv, D, bs) in [([40, 19], [7, 19], 4, 2, 32, 16),
                                          ([9, 33, 1], [9, 5, 1], 6, 2, 16, 4)]:
        k, v, bt, cl = make_paged(rng, lens, Hkv, D, bs)
        qsl = np.concatenate([[0], np.cumsum(qlens)]).astype(np.int32)
        q = rand_bits(rng, (int(qsl[-1]), Hq, D))
        scale = 0.3
        got = orc.paged_attention_prefill(q, qsl, k, v, bt, cl, scale)
        ref = brute.paged_attention_prefill(q, qsl, k, v, bt, cl, scale)
        np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


def pin_paged_equals_contiguous(orc):
    rng = np.random.default_rng(13)
    B, Lmax, Hq, Hkv, D, bs = 3, 50, 4, 2, 16, 16
    lens = np.array([50, 17, 33], dtype=np.int32)
    kc = rand_bits(rng, (B, Lmax, Hkv, D))
    vc = rand_bits(rng, (B, Lmax, Hkv, D))
    q = rand_bits(rng, (B, Hq, D))
    k_cache, v_cache, bt = scatter_contiguous(orc, kc, vc, lens, bs, rng)
    paged = orc.paged_attention(q, k_cache, v_cache, bt, lens, 0.25)
    contig = orc.contiguous_attention(q, kc, vc, lens, 0.25)
    assert np.array_equal(paged, contig), "paged and contiguous layouts must agree bit for bit"


def pin_scatter_gather_identity(orc):
    rng = np.random.default_rng(14)
    NB, Hkv, bs, D, T = 6, 2, 4, 8, 9
    k_cache = rand_bits(rng, (NB, Hkv, bs, D))
    v_cache = rand_bits(rng, (NB, Hkv, bs, D))
    k0, v0 = k_cache.copy(), v_cache.copy()
    key = rand_bits(rng, (T, Hkv, D))
    val = rand_bits(rng, (T, Hkv, D))
    slots = rng.permutation(NB * bs)[:T].astype(np.int64)
    slots[3] = -1                                   # padding token: skipped
    rc = orc.kv_cache_write(key, val, k_cache, v_cache, slots)
    assert rc == 0
    touched = np.zeros((NB, bs), dtype=bool)
    for t, s in enumerate(slots):
        if s < 0:
            continue
        blk, off = divmod(int(s), bs)
        touched[blk, off] = True
        assert np.array_equal(k_cache[blk, :, off, :], key[t])
        assert np.array_equal(v_cache[blk, :, off, :], val[t])
    keep = np.broadcast_to((~touched)[:, None, :, None], k_cache.shape)
    assert np.array_equal(k_cache[keep], k0[keep]), "untouched slots changed"
    assert np.array_equal(v_cache[keep], v0[keep])
    # a slot outside the pool is reported and writes nothing
    k1, v1 = k_cache.copy(), v_cache.copy()
    rc = orc.kv_cache_write(key[:1], val[:1], k_cache, v_cache,
                            np.array([NB * bs], np.int64), allow_bounds=True)
    assert rc == 5 and np.array_equal(k_cache, k1) and np.array_equal(v_cache, v1)


def pin_single_key_returns_v(orc):
    rng = np.random.default_rng(15)
    k, v, bt, cl = make_paged(rng, [1, 1, 1], 2, 32, 16)
    q = rand_bits(rng, (3, 4, 32))
    out = orc.paged_attention(q, k, v, bt, cl, 0.7)
    for b in range(3):
        for h in range(4):
            vrow = bf16_bits_to_f64(v[bt[b, 0], h // 2, 0])
            assert np.array_equal(out[b, h], vrow)


def pin_identical_keys_mean_v(orc):
    rng = np.random.default_rng(16)
    L, Hkv, D, bs = 45, 1, 16, 16
    kc = np.repeat(rand_bits(rng, (1, 1, 1, D)), L, axis=1)
    vc = rand_bits(rng, (1, L, Hkv, D))
    q = rand_bits(rng, (1, 2, D))
    k_cache, v_cache, bt = scatter_contiguous(orc, kc, vc, [L], bs, rng)
    out = orc.paged_attention(q, k_cache, v_cache, bt, np.array([L], np.int32), 0.125)
    mean = bf16_bits_to_f64(vc[0, :, 0, :]).mean(axis=0)
    for h in range(2):
        np.testing.assert_allclose(out[0, h], mean, rtol=0, atol=1e-14)


def pin_scale_zero_mean_v(orc):
    rng = np.random.default_rng(17)
    k, v, bt, cl = make_paged(rng, [29], 2, 16, 8)
    q = rand_bits(rng, (1, 2, 16))
    out = orc.paged_attention(q, k, v, bt, cl, 0.0)
    V = brute.dense_kv(v, bt[0], 29)
    for h in range(2):
        np.testing.assert_allclose(out[0, h], V[:, h].mean(axis=0), rtol=0, atol=1e-14)


def pin_softmax_row_sums_to_one(orc):
    """With V row j = unit vector e_j the output row IS the probability row."""
    rng = np.random.default_rng(18)
    L, D, bs = 24, 32, 8
    kc = rand_bits(rng, (1, L, 1, D))
    eye = np.zeros((1, L, 1, D), dtype=np.float32)
    for j in range(L):
        eye[0, j, 0, j] = 1.0
    vc = f32_to_bf16_bits(eye)
    q = rand_bits(rng, (1, 1, D))
    k_cache, v_cache, bt = scatter_contiguous(orc, kc, vc, [L], bs, rng)
    scale = 0.2
    p = orc.paged_attention(q, k_cache, v_cache, bt, np.array([L], np.int32), scale)[0, 0, :L]
    assert abs(p.sum() - 1.0) < 1e-13
    s = np.float64(np.float32(scale)) * (bf16_bits_to_f64(kc[0, :, 0, :]) @ bf16_bits_to_f64(q[0, 0]))
    w = np.exp(s - s.max())
    np.testing.assert_allclose(p, w / w.sum(), rtol=1e-13, atol=1e-16)


def pin_causal_mask(orc):
    rng = np.random.default_rng(19)
    L, Q, Hq, Hkv, D, bs = 40, 12, 4, 2, 16, 8
    kc = rand_bits(rng, (1, L, Hkv, D))
    vc = rand_bits(rng, (1, L, Hkv, D))
    q = rand_bits(rng, (Q, Hq, D))
    qsl = np.array([0, Q], np.int32)
    cl = np.array([L], np.int32)
    k1, v1, bt = scatter_contiguous(orc, kc, vc, [L], bs, np.random.default_rng(5))
    base = orc.paged_attention_prefill(q, qsl, k1, v1, bt, cl, 0.25)
    # perturb keys/values after position p: queries at positions <= p unchanged
    p = L - Q + 4                                   # query index 4 sits at position p
    kc2, vc2 = kc.copy(), vc.copy()
    kc2[0, p + 1:] = rand_bits(rng, kc2[0, p + 1:].shape)
    vc2[0, p + 1:] = rand_bits(rng, vc2[0, p + 1:].shape)
    k2, v2, bt2 = scatter_contiguous(orc, kc2, vc2, [L], bs, np.random.default_rng(5))
    pert = orc.paged_attention_prefill(q, qsl, k2, v2, bt2, cl, 0.25)
    assert np.array_equal(base[:5], pert[:5]), "a query saw a future key"
    assert not np.array_equal(base[5:], pert[5:]), "later queries must see the change"
    # the chunk's last query equals decode over all L keys
    dec = orc.paged_attention(q[-1:], k1, v1, bt, cl, 0.25)
    assert np.array_equal(dec[0], base[-1])


def pin_gqa_equals_materialised_mha(orc):
    rng = np.random.default_rng(20)
    B, Lmax, Hq, Hkv, D, bs = 2, 30, 6, 2, 16, 8
    lens = np.array([30, 11], np.int32)
    kc = rand_bits(rng, (B, Lmax, Hkv, D))
    vc = rand_bits(rng, (B, Lmax, Hkv, D))
    q = rand_bits(rng, (B, Hq, D))
    G = Hq // Hkv
    kg, vg, btg = scatter_contiguous(orc, kc, vc, lens, bs, np.random.default_rng(1))
    gqa = orc.paged_attention(q, kg, vg, btg, lens, 0.3)
    # materialise: kv head h of the MHA cache is the GQA head h // G (consecutive groups)
    km, vm, btm = scatter_contiguous(orc, np.repeat(kc, G, axis=2), np.repeat(vc, G, axis=2), lens,
                                     bs, np.random.default_rng(1))
    mha = orc.paged_attention(q, km, vm, btm, lens, 0.3)
    assert np.array_equal(gqa, mha)
    # two query heads of one group with the same q give the same row
    q2 = q.copy()
    q2[:, 1] = q2[:, 0]
    o2 = orc.paged_attention(q2, kg, vg, btg, lens, 0.3)
    assert np.array_equal(o2[:, 0], o2[:, 1])


def pin_split_merge_equals_plain(orc):
    rng = np.random.default_rng(21)
    lens = [100, 1, 64, 0, 37]
    k, v, bt, cl = make_paged(rng, lens, 2, 16, 16)
    q = rand_bits(rng, (len(lens), 4, 16))
    plain = orc.paged_attention(q, k, v, bt, cl, 0.25)
    for S in (16, 32, 48, 100, 128):
        C = -(-max(lens) // S)
        o, lse = orc.decode_partials(q, k, v, bt, cl, 0.25, S, C)
        merged = orc.lse_merge(o, lse)
        np.testing.assert_allclose(merged, plain, rtol=0, atol=1e-12)
    # the merge itself: two halves with known weights
    o_part = np.array([[[1.0, 0.0], [0.0, 1.0]]])
    lse = np.array([[np.log(3.0), np.log(1.0)]])
    np.testing.assert_allclose(orc.lse_merge(o_part, lse), [[0.75, 0.25]], atol=1e-15)


def pin_empty_context_is_zero(orc):
    rng = np.random.default_rng(22)
    k, v, bt, cl = make_paged(rng, [0, 5], 1, 8, 4)
    q = rand_bits(rng, (2, 2, 8))
    out = orc.paged_attention(q, k, v, bt, cl, 1.0)
    assert np.array_equal(out[0], np.zeros((2, 8)))
    assert np.isfinite(out[1]).all()


# --------------------------------------------------------------------------- #
# INT8 cache                                                                   #
# --------------------------------------------------------------------------- #

def _int8_pool(NB, Hkv, bs, D):
    """Empty int8 pools with canaries: code 99 and a NaN scale in every slot."""
    k = np.full((NB, Hkv, bs, D), 99, dtype=np.int8)
    v = np.full((NB, Hkv, bs, D), 99, dtype=np.int8)
    ks = np.full((NB, Hkv, bs), np.nan, dtype=np.float32)
    vs = np.full((NB, Hkv, bs), np.nan, dtype=np.float32)
    return k, v, ks, vs


def pin_int8_exact_grid_rows(orc):
    """Values k * 2^-e with max |k| = 127 are bf16-exact; the row's scale is
    then exactly 2^-e and its codes exactly k."""
    rng = np.random.default_rng(31)
    T, Hkv, D, bs, NB = 6, 2, 32, 4, 3
    kk = rng.integers(-127, 128, size=(T, Hkv, D))
    kk[..., 0] = 127 * np.where(rng.random((T, Hkv)) < 0.5, 1, -1)   # amax = 127 * 2^-e
    e = rng.integers(0, 12, size=(T, Hkv, 1))
    x = (kk * np.ldexp(1.0, -e)).astype(np.float32)
    bits = f32_to_bf16_bits(x)
    assert np.array_equal(bf16_bits_to_f64(bits), x.astype(np.float64))
    k, v, ks, vs = _int8_pool(NB, Hkv, bs, D)
    slots = np.array([0, 5, 2, 11, 7, 3], dtype=np.int64)
    orc.kv_cache_write_int8(bits, bits, k, v, ks, vs, slots)
    for t, sl in enumerate(slots):
        blk, off = sl // bs, sl % bs
        assert np.array_equal(k[blk, :, off, :], kk[t].astype(np.int8))
        assert np.array_equal(v[blk, :, off, :], kk[t].astype(np.int8))
        assert np.array_equal(ks[blk, :, off], np.ldexp(1.0, -e[t, :, 0]).astype(np.float32))


def pin_int8_ties_round_to_even(orc):
    """amax = 127 makes the code step exactly 1: x.5 rounds to the even code."""
    row = np.array([127.0, 2.5, 3.5, -2.5, -0.5, 0.5, 1.5, -1.5, 126.5, 0.25, -3.5, 4.5], dtype=np.float32)
    want = np.array([127, 2, 4, -2, 0, 0, 2, -2, 126, 0, -4, 4], dtype=np.int8)
    bits = f32_to_bf16_bits(row)[None, None, :]
    k, v, ks, vs = _int8_pool(1, 1, 1, row.size)
    orc.kv_cache_write_int8(bits, bits, k, v, ks, vs, np.array([0], dtype=np.int64))
    assert np.array_equal(k[0, 0, 0], want), k[0, 0, 0]
    assert ks[0, 0, 0] == np.float32(1.0)


def pin_int8_error_within_half_step(orc):
    """Round to nearest: |code * scale - x| <= scale / 2, every code in
    [-127, 127], and the largest |code| is 127.  Slack: x * inv and the stored
    scale are fp32, each off by <= 2^-24 relative, i.e. <= 127 * 2^-23 of a
    code step near a tie; 2^-14 of the half step covers it, far below the
    whole step a truncating rounding would miss by."""
    rng = np.random.default_rng(32)
    T, Hkv, D, bs, NB = 40, 3, 64, 8, 6
    bits = rand_bits(rng, (T, Hkv, D), std=2.0)
    k, v, ks, vs = _int8_pool(NB, Hkv, bs, D)
    slots = rng.permutation(NB * bs)[:T].astype(np.int64)
    orc.kv_cache_write_int8(bits, bits, k, v, ks, vs, slots)
    x = bf16_bits_to_f64(bits)
    for t, sl in enumerate(slots):
        blk, off = sl // bs, sl % bs
        c = k[blk, :, off, :].astype(np.float64)
        sc = ks[blk, :, off].astype(np.float64)[:, None]
        assert np.abs(c).max() <= 127
        assert np.all(np.abs(c).max(axis=-1) == 127)
        assert np.all(np.abs(c * sc - x[t]) <= 0.5 * sc * (1 + 2.0 ** -14))


def pin_int8_zero_row_and_slots(orc):
    """A zero row gives codes 0 and scale 0; negative slots are skipped and
    every other slot keeps its canary."""
    D, bs, NB = 16, 4, 2
    key = np.zeros((3, 1, D), dtype=np.uint16)
    key[1] = f32_to_bf16_bits(np.linspace(-1, 1, D, dtype=np.float32))[None]
    k, v, ks, vs = _int8_pool(NB, 1, bs, D)
    orc.kv_cache_write_int8(key, key, k, v, ks, vs, np.array([6, -1, 1], dtype=np.int64))
    assert np.array_equal(k[1, 0, 2], np.zeros(D, np.int8)) and ks[1, 0, 2] == 0.0
    assert np.array_equal(k[0, 0, 1], np.zeros(D, np.int8)) and ks[0, 0, 1] == 0.0
    touched = {(1, 2), (0, 1)}
    for blk in range(NB):
        for off in range(bs):
            if (blk, off) not in touched:
                assert np.all(k[blk, 0, off] == 99) and np.isnan(ks[blk, 0, off])


def _random_int8_paged(rng, lens, Hkv, D, bs, extra=2):
    pages = [-(-L // bs) for L in lens]
    NB = sum(pages) + extra
    perm = rng.permutation(NB)
    MB = max(pages + [1])
    bt = np.full((len(lens), MB), -1, dtype=np.int32)
    o = 0
    for b, n in enumerate(pages):
        bt[b, :n] = perm[o:o + n]
        o += n
    k = rng.integers(-127, 128, size=(NB, Hkv, bs, D)).astype(np.int8)
    v = rng.integers(-127, 128, size=(NB, Hkv, bs, D)).astype(np.int8)
    ks = np.exp(rng.uniform(np.log(1e-3), np.log(3e-2), size=(NB, Hkv, bs))).astype(np.float32)
    vs = np.exp(rng.uniform(np.log(1e-3), np.log(3e-2), size=(NB, Hkv, bs))).astype(np.float32)
    return k, v, ks, vs, bt, np.array(lens, dtype=np.int32)


def pin_int8_attention_brute_force(orc):
    """NumPy full-matrix attention over the dequantised pool (code * scale)."""
    rng = np.random.default_rng(33)
    for lens, Hq, Hkv in (([5, 17, 1, 33], 4, 2), ([40, 9], 6, 3), ([16], 2, 2)):
        D, bs = 16, 4
        k, v, ks, vs, bt, cl = _random_int8_paged(rng, lens, Hkv, D, bs)
        q = rand_bits(rng, (len(lens), Hq, D))
        got = orc.paged_attention_int8(q, k, v, ks, vs, bt, cl, 0.3)
        kd = k.astype(np.float64) * ks.astype(np.float64)[..., None]
        vd = v.astype(np.float64) * vs.astype(np.float64)[..., None]
        G = Hq // Hkv
        for b, L in enumerate(lens):
            pages = bt[b, :-(-L // bs)]
            K = np.transpose(kd[pages], (0, 2, 1, 3)).reshape(-1, Hkv, D)[:L]
            V = np.transpose(vd[pages], (0, 2, 1, 3)).reshape(-1, Hkv, D)[:L]
            K, V = np.repeat(K, G, axis=1), np.repeat(V, G, axis=1)
            S = np.einsum("hd,jhd->hj", bf16_bits_to_f64(q[b]), K) * np.float64(np.float32(0.3))
            P = np.exp(S - S.max(axis=1, keepdims=True))
            ref = np.einsum("hj,jhd->hd", P / P.sum(axis=1, keepdims=True), V)
            assert np.allclose(got[b], ref, rtol=1e-12, atol=1e-14), np.abs(got[b] - ref).max()


def pin_int8_equals_bf16_path_on_exact_values(orc):
    """Power-of-two scales make code * scale bf16-exact; the int8 decode then
    equals the (pinned) bf16 decode of the same values bit for bit."""
    rng = np.random.default_rng(34)
    lens, Hq, Hkv, D, bs = [23, 7, 40], 8, 2, 32, 8
    k, v, ks, vs, bt, cl = _random_int8_paged(rng, lens, Hkv, D, bs)
    ks = np.ldexp(1.0, -rng.integers(4, 9, size=ks.shape)).astype(np.float32)
    vs = np.ldexp(1.0, -rng.integers(4, 9, size=vs.shape)).astype(np.float32)
    kb = f32_to_bf16_bits(k.astype(np.float32) * ks[..., None])
    vb = f32_to_bf16_bits(v.astype(np.float32) * vs[..., None])
    assert np.array_equal(bf16_bits_to_f64(kb), k.astype(np.float64) * ks[..., None])
    q = rand_bits(rng, (len(lens), Hq, D))
    a = orc.paged_attention_int8(q, k, v, ks, vs, bt, cl, 0.125)
    b = orc.paged_attention(q, kb, vb, bt, cl, 0.125)
    assert np.array_equal(a, b)


# --------------------------------------------------------------------------- #
# sliding window                                                               #
# --------------------------------------------------------------------------- #

def pin_window_covering_all_is_full_attention(orc):
    rng = np.random.default_rng(41)
    lens = [1, 9, 30, 17]
    k, v, bt, cl = make_paged(rng, lens, 2, 16, 4)
    q = rand_bits(rng, (4, 4, 16))
    full = orc.paged_attention(q, k, v, bt, cl, 0.4)
    for W in (30, 31, 1000):
        assert np.array_equal(orc.paged_attention_window(q, k, v, bt, cl, 0.4, W), full)


def pin_window_one_returns_last_v(orc):
    rng = np.random.default_rng(42)
    lens = [5, 12, 33]
    k, v, bt, cl = make_paged(rng, lens, 1, 8, 4)
    q = rand_bits(rng, (3, 2, 8))
    out = orc.paged_attention_window(q, k, v, bt, cl, 0.7, 1)
    for b, L in enumerate(lens):
        blk = bt[b, (L - 1) // 4]
        last_v = bf16_bits_to_f64(v[blk, 0, (L - 1) % 4])
        assert np.array_equal(out[b, 0], last_v) and np.array_equal(out[b, 1], last_v)


def pin_window_equals_truncated_context(orc):
    """Windowed decode over L keys == full decode of a contiguous cache that
    holds only the last W of them (same rows, same order: bit for bit)."""
    rng = np.random.default_rng(43)
    lens, Hq, Hkv, D, bs, W = [50, 7, 33, 16], 6, 3, 16, 4, 13
    k, v, bt, cl = make_paged(rng, lens, Hkv, D, bs)
    q = rand_bits(rng, (len(lens), Hq, D))
    got = orc.paged_attention_window(q, k, v, bt, cl, 0.3, W)
    n = [min(L, W) for L in lens]
    kc = np.zeros((len(lens), max(n), Hkv, D), np.uint16)
    vc = np.zeros_like(kc)
    for b, L in enumerate(lens):
        for i, j in enumerate(range(L - n[b], L)):
            blk, row = bt[b, j // bs], j % bs
            kc[b, i] = k[blk, :, row]
            vc[b, i] = v[blk, :, row]
    ref = orc.contiguous_attention(q, kc, vc, np.array(n, np.int32), 0.3)
    assert np.array_equal(got, ref)


def pin_int8_window_brute_force(orc):
    """INT8 cache under a sliding window: NumPy full-matrix attention over the
    dequantised last W keys; a window covering the context equals the
    unwindowed INT8 decode bit for bit."""
    rng = np.random.default_rng(45)
    for lens, Hq, Hkv, W in (([5, 17, 1, 33], 4, 2, 7), ([40, 9], 6, 3, 16), ([16], 2, 2, 1)):
        D, bs = 16, 4
        k, v, ks, vs, bt, cl = _random_int8_paged(rng, lens, Hkv, D, bs)
        q = rand_bits(rng, (len(lens), Hq, D))
        got = orc.paged_attention_int8(q, k, v, ks, vs, bt, cl, 0.3, window=W)
        kd = k.astype(np.float64) * ks.astype(np.float64)[..., None]
        vd = v.astype(np.float64) * vs.astype(np.float64)[..., None]
        G = Hq // Hkv
        for b, L in enumerate(lens):
            pages = bt[b, :-(-L // bs)]
            K = np.transpose(kd[pages], (0, 2, 1, 3)).reshape(-1, Hkv, D)[:L][max(0, L - W):]
            V = np.transpose(vd[pages], (0, 2, 1, 3)).reshape(-1, Hkv, D)[:L][max(0, L - W):]
            K, V = np.repeat(K, G, axis=1), np.repeat(V, G, axis=1)
            S = np.einsum("hd,jhd->hj", bf16_bits_to_f64(q[b]), K) * np.float64(np.float32(0.3))
            P = np.exp(S - S.max(axis=1, keepdims=True))
            ref = np.einsum("hj,jhd->hd", P / P.sum(axis=1, keepdims=True), V)
            assert np.allclose(got[b], ref, rtol=1e-12, atol=1e-14), np.abs(got[b] - ref).max()
        full = orc.paged_attention_int8(q, k, v, ks, vs, bt, cl, 0.3)
        assert np.array_equal(orc.paged_attention_int8(q, k, v, ks, vs, bt, cl, 0.3, window=max(lens)), full)


def pin_int8_window_equals_bf16_window_on_exact_values(orc):
    """Power-of-two scales make code * scale bf16-exact: the INT8 window decode
    then equals the (pinned) bf16 window decode of the same values bit for bit."""
    rng = np.random.default_rng(46)
    lens, Hq, Hkv, D, bs = [23, 7, 40], 8, 2, 32, 8
    k, v, ks, vs, bt, cl = _random_int8_paged(rng, lens, Hkv, D, bs)
    ks = np.ldexp(1.0, -rng.integers(4, 9, size=ks.shape)).astype(np.float32)
    vs = np.ldexp(1.0, -rng.integers(4, 9, size=vs.shape)).astype(np.float32)
    kb = f32_to_bf16_bits(k.astype(np.float32) * ks[..., None])
    vb = f32_to_bf16_bits(v.astype(np.float32) * vs[..., None])
    q = rand_bits(rng, (len(lens), Hq, D))
    for W in (1, 5, 17, 64):
        a = orc.paged_attention_int8(q, k, v, ks, vs, bt, cl, 0.125, window=W)
        b = orc.paged_attention_window(q, kb, vb, bt, cl, 0.125, W)
        assert np.array_equal(a, b), W


def pin_window_prefill_brute_force_and_last_row(orc):
    rng = np.random.default_rng(44)
    lens, qlens, Hq, Hkv, D, bs = [40, 9, 25], [12, 9, 1], 4, 2, 16, 4
    k, v, bt, cl = make_paged(rng, lens, Hkv, D, bs)
    qsl = np.concatenate([[0], np.cumsum(qlens)]).astype(np.int32)
    q = rand_bits(rng, (int(qsl[-1]), Hq, D))
    for W in (1, 5, 16, 100):
        got = orc.paged_attention_prefill_window(q, qsl, k, v, bt, cl, 0.25, W)
        for b, (L, Q) in enumerate(zip(lens, qlens)):
            K = brute.dense_kv(k, bt[b], L)
            V = brute.dense_kv(v, bt[b], L)
            G = Hq // Hkv
            K, V = np.repeat(K, G, axis=1), np.repeat(V, G, axis=1)
            qb = bf16_bits_to_f64(q[qsl[b]:qsl[b + 1]])
            S = np.einsum("ihd,jhd->hij", qb, K) * np.float64(np.float32(0.25))
            pos = L - Q + np.arange(Q)[:, None]
            j = np.arange(L)[None, :]
            S = np.where((j <= pos) & (j > pos - W), S, -np.inf)
            P = np.exp(S - S.max(axis=-1, keepdims=True))
            ref = np.einsum("hij,jhd->ihd", P / P.sum(axis=-1, keepdims=True), V)
            assert np.allclose(got[qsl[b]:qsl[b + 1]], ref, rtol=1e-12, atol=1e-14)
            last = orc.paged_attention_window(q[qsl[b + 1] - 1][None], k, v, bt[b:b + 1], cl[b:b + 1], 0.25, W)
            assert np.array_equal(got[qsl[b + 1] - 1], last[0])


# --------------------------------------------------------------------------- #
# RoPE in the cache write                                                      #
# --------------------------------------------------------------------------- #

def pin_rope_position_zero_is_identity(orc):
    rng = np.random.default_rng(51)
    x = rand_bits(rng, (5, 3, 16))
    y = orc.rope_rows(x, np.zeros(5, np.int64), 10000.0)
    assert np.array_equal(y, bf16_bits_to_f64(x))


def pin_rope_unit_vectors_d4(orc):
    """D = 4, base 100: pair (0, 2) turns at pos * 1, pair (1, 3) at pos * 0.1."""
    for pos in (1, 7, 123):
        e0 = np.zeros((1, 1, 4), np.uint16)
        e0[0, 0, 0] = 0x3F80                          # 1.0
        y = orc.rope_rows(e0, np.array([pos]), 100.0)[0, 0]
        assert np.allclose(y, [np.cos(pos), 0.0, np.sin(pos), 0.0], rtol=0, atol=1e-15), y
        e1 = np.zeros((1, 1, 4), np.uint16)
        e1[0, 0, 1] = 0x3F80
        y = orc.rope_rows(e1, np.array([pos]), 100.0)[0, 0]
        assert np.allclose(y, [0.0, np.cos(0.1 * pos), 0.0, np.sin(0.1 * pos)], rtol=0, atol=1e-15), y


def pin_rope_keeps_norms_and_relative_position(orc):
    rng = np.random.default_rng(52)
    D = 32
    q = rand_bits(rng, (1, 1, D))
    k = rand_bits(rng, (1, 1, D))
    x = bf16_bits_to_f64(q)[0, 0]
    y = orc.rope_rows(q, np.array([4321]), 500000.0)[0, 0]
    h = D // 2
    assert np.allclose(y[:h] ** 2 + y[h:] ** 2, x[:h] ** 2 + x[h:] ** 2, rtol=1e-13, atol=0)
    for m, n, sft in ((5, 2, 100), (1000, 17, 3), (0, 99, 12345)):
        a = np.dot(orc.rope_rows(q, np.array([m]), 10000.0)[0, 0], orc.rope_rows(k, np.array([n]), 10000.0)[0, 0])
        b = np.dot(orc.rope_rows(q, np.array([m + sft]), 10000.0)[0, 0],
                   orc.rope_rows(k, np.array([n + sft]), 10000.0)[0, 0])
        assert abs(a - b) <= 1e-11 * max(1.0, abs(a)), (a, b)


def pin_rope_cache_write(orc):
    rng = np.random.default_rng(53)
    T, Hkv, D, bs, NB = 9, 2, 16, 4, 5
    key = rand_bits(rng, (T, Hkv, D))
    val = rand_bits(rng, (T, Hkv, D))
    k = rand_bits(rng, (NB, Hkv, bs, D))
    v = rand_bits(rng, (NB, Hkv, bs, D))
    k0, v0 = k.copy(), v.copy()
    slots = np.array([3, -1, 0, 19, 7, 8, -1, 12, 1], np.int64)
    pos = rng.integers(0, 100000, size=T).astype(np.int64)
    orc.kv_cache_write_rope(key, val, k, v, slots, pos, 500000.0)
    want = orc.rope_rows(key, pos, 500000.0)
    for t, sl in enumerate(slots):
        if sl < 0:
            continue
        blk, off = sl // bs, sl % bs
        got = bf16_bits_to_f64(k[blk, :, off])
        # bf16 of the fp64 value: within half a bf16 step, 8 significant bits,
        # i.e. at most 2^-8 relative (at the bottom of a binade)
        assert np.all(np.abs(got - want[t]) <= np.abs(want[t]) * 2.0 ** -8 + 1e-300)
        # and it is the nearest bf16: the neighbours one step away are farther
        bits = k[blk, :, off].astype(np.int64)
        for nb in (bits - 1, bits + 1):
            other = bf16_bits_to_f64(nb.astype(np.uint16))
            ok = np.isnan(other) | (np.abs(other - want[t]) >= np.abs(got - want[t]))
            assert np.all(ok)
        assert np.array_equal(v[blk, :, off], val[t])
        k0[blk, :, off] = k[blk, :, off]
        v0[blk, :, off] = v[blk, :, off]
    assert np.array_equal(k, k0) and np.array_equal(v, v0)   # nothing else touched


def pin_negative_scale(orc):
    """A negative scale is legal attention: the scores scale * q.k reverse
    their order.  Closed form: keys (1, 0) and (-1, 0), q = (1, 0) and
    scale -1 give scores -1 and 1, so the weights are sigmoid(-2) and
    sigmoid(2) (the first query of a two-token chunk sees only key 0).
    Negating q and the scale together changes nothing, bit for bit, and the
    NumPy brute force agrees on random chunks."""
    rng = np.random.default_rng(41)
    kc = f32_to_bf16_bits(np.array([[1.0, 0.0], [-1.0, 0.0]], np.float32))[None, :, None, :]
    vc = f32_to_bf16_bits(np.array([[1.0, 0.0], [0.0, 1.0]], np.float32))[None, :, None, :]
    k, v, bt = scatter_contiguous(orc, kc, vc, [2], 2, rng)
    q = f32_to_bf16_bits(np.array([[1.0, 0.0], [1.0, 0.0]], np.float32))[:, None, :]
    lo, hi = 1.0 / (1.0 + np.exp(2.0)), 1.0 / (1.0 + np.exp(-2.0))
    out = orc.paged_attention_prefill(q, np.array([0, 2], np.int32), k, v, bt, np.array([2], np.int32), -1.0)
    np.testing.assert_allclose(out[0, 0], [1.0, 0.0], rtol=0, atol=1e-15)
    np.testing.assert_allclose(out[1, 0], [lo, hi], rtol=0, atol=1e-15)
    dec = orc.paged_attention(q[1:], k, v, bt, np.array([2], np.int32), -1.0)
    np.testing.assert_allclose(dec[0, 0], [lo, hi], rtol=0, atol=1e-15)
    for (lens, qlens, Hq, Hkv, D, bs) in [([40, 19], [7, 19], 4, 2, 32, 16), ([9, 33], [9, 5], 6, 2, 16, 4)]:
        k, v, bt, cl = make_paged(rng, lens, Hkv, D, bs)
        qsl = np.concatenate([[0], np.cumsum(qlens)]).astype(np.int32)
        q = rand_bits(rng, (int(qsl[-1]), Hq, D))
        got = orc.paged_attention_prefill(q, qsl, k, v, bt, cl, -0.3)
        np.testing.assert_allclose(got, brute.paged_attention_prefill(q, qsl, k, v, bt, cl, -0.3), rtol=0,
                                   atol=1e-12)
        flipped = orc.paged_attention_prefill(q ^ np.uint16(0x8000), qsl, k, v, bt, cl, 0.3)
        assert np.array_equal(got, flipped)


ALL_PINS = [
    pin_golden_closed_form,
    pin_brute_force_decode,
    pin_brute_force_prefill,
    pin_paged_equals_contiguous,
    pin_scatter_gather_identity,
    pin_single_key_returns_v,
    pin_identical_keys_mean_v,
    pin_scale_zero_mean_v,
    pin_softmax_row_sums_to_one,
    pin_causal_mask,
    pin_gqa_equals_materialised_mha,
    pin_split_merge_equals_plain,
    pin_empty_context_is_zero,
    pin_int8_exact_grid_rows,
    pin_int8_ties_round_to_even,
    pin_int8_error_within_half_step,
    pin_int8_zero_row_and_slots,
    pin_int8_attention_brute_force,
    pin_int8_equals_bf16_path_on_exact_values,
    pin_window_covering_all_is_full_attention,
    pin_window_one_returns_last_v,
    pin_window_equals_truncated_context,
    pin_window_prefill_brute_force_and_last_row,
    pin_int8_window_brute_force,
    pin_int8_window_equals_bf16_window_on_exact_values,
    pin_rope_position_zero_is_identity,
    pin_rope_unit_vectors_d4,
    pin_rope_keeps_norms_and_relative_position,
    pin_rope_cache_write,
    pin_negative_scale,
]
