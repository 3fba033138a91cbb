"""Pins of the CPU oracle against what the pages and the mathematics fix.

Each check here comes from somewhere other than the oracle itself: the
worked row and the storage arithmetic printed on the pages (fixtures under
tests/golden/), brute-force enumeration of the selection rule, a stable
library sort, numpy's float64 matmul as the closed form of the GEMM, an
explicit permutation matrix, and special cases (identity permutation, all
dense / all 2:4 tile maps) that reduce one function to another.
"""
import itertools
import json
import os

import numpy as np
import pytest

import oracle
import workloads as wl

PATTERNS = [(2, 4), (1, 4), (1, 8), (3, 4), (1, 2), (4, 8), (3, 8), (2, 8), (5, 16), (1, 16)]


def f64(bits):
    return wl.bf16_to_f32(bits).astype(np.float64)


def bits_of(values):
    return wl.bf16_bits(np.asarray(values, dtype=np.float32))


def positions(meta, R, K, n, m):
    """Survivor positions read back from the packed metadata (list of rows)."""
    return oracle.positions(meta, R, K, n, m).astype(int).tolist()


# ---------------------------------------------------------------------------
# The worked row of the pages
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("v", [1.0, -3.5, 0.0078125, 65280.0])
def test_worked_row(golden_dir, v):
    g = json.load(open(os.path.join(golden_dir, "worked_row_2of4.json")))
    row = [v if c == "v" else 0.0 for c in g["row_template"]]
    W = bits_of([row])
    vals, meta = oracle.compress(W, 2, 4)
    pos = positions(meta, 1, 8, 2, 4)[0]
    assert [pos[0:2], pos[2:4]] == g["metadata"]
    assert int(meta[0]) & 0xFF == g["packed_low_byte"]
    # the rest of the tile is padding: all-zero groups, positions (0,1), nibble 0x4
    assert int(meta[0]) >> 8 == 0x444444
    assert np.all(meta[1:] == 0x44444444)
    assert np.array_equal(vals[0], bits_of([v, v, v, v]))


# ---------------------------------------------------------------------------
# Selection rule
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("n,m", PATTERNS)
def test_exactly_n_survivors(n, m):
    W = wl.normal_bf16((37, 16 * m), 1.0, seed=n * 100 + m)
    mask = oracle.prune_mask(W, n, m)
    assert np.all(mask.reshape(37, -1, m).sum(axis=2) == n)


def _preferred(w, i, j):
    """i is kept ahead of j: larger |w|, equal magnitudes to the lower index."""
    return (abs(w[i]), -i) > (abs(w[j]), -j)


@pytest.mark.parametrize("n,m", [(2, 4), (1, 4), (3, 4), (1, 8), (2, 8), (5, 8), (1, 2)])
def test_selection_bruteforce(n, m):
    """Exactly one N-subset dominates its complement, and it is the oracle's."""
    rng = np.random.default_rng(7 + n + m)
    groups = rng.integers(-3, 4, size=(300, m)).astype(np.float32)  # many ties
    W = bits_of(groups.reshape(1, -1))
    mask = oracle.prune_mask(W, n, m).reshape(-1, m)
    for gi, grp in enumerate(groups):
        w = [float(x) for x in grp]
        winners = [S for S in itertools.combinations(range(m), n)
                   if all(_preferred(w, i, j) for i in S for j in range(m) if j not in S)]
        assert len(winners) == 1
        assert [p for p in range(m) if mask[gi, p]] == list(winners[0])


def _stable_sort_select(w, n):
    order = sorted(range(len(w)), key=lambda i: -abs(w[i]))  # stable: ties keep lower index first
    return sorted(order[:n])


@pytest.mark.parametrize("n,m,alphabet", [
    (2, 4, [-2.0, -1.0, -0.0, 0.0, 1.0, 2.0]),
    (1, 4, [-2.0, -1.0, -0.0, 0.0, 1.0, 2.0]),
    (3, 4, [-2.0, -1.0, -0.0, 0.0, 1.0, 2.0]),
    (1, 8, [0.0, 1.0, 2.0]),
    (2, 8, [0.0, -1.0, 2.0]),
])
def test_exhaustive_alphabet(n, m, alphabet):
    groups = np.array(list(itertools.product(alphabet, repeat=m)), dtype=np.float32)
    W = bits_of(groups.reshape(1, -1))
    vals, meta = oracle.compress(W, n, m)
    pos = positions(meta, 1, W.shape[1], n, m)[0]
    for gi, grp in enumerate(groups):
        want = _stable_sort_select([float(x) for x in grp], n)
        assert pos[gi * n:(gi + 1) * n] == want
        # values are the exact bit patterns at those positions (-0.0 kept as -0.0)
        assert np.array_equal(vals[0, gi * n:(gi + 1) * n], bits_of(grp[want]))


def test_nan_inf_order():
    """Reading for non-finite inputs: NaN above Inf, Inf above finite, ties to the lower index."""
    nan, inf = float("nan"), float("inf")
    rows = [[nan, inf, 1.0, -inf], [1.0, nan, nan, 5.0], [-inf, 3.0, inf, 2.0], [0.0, -0.0, 0.0, -0.0]]
    want = [[0, 1], [1, 2], [0, 2], [0, 1]]
    W = bits_of(rows)
    mask = oracle.prune_mask(W, 2, 4)
    for r, w in enumerate(want):
        assert [p for p in range(4) if mask[r, p]] == w


# ---------------------------------------------------------------------------
# Storage format
# ---------------------------------------------------------------------------
def test_storage_36_bits(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "storage_bits.json")))
    R, K = 64, 4096
    W = wl.normal_bf16((R, K), 1.0, seed=3)
    vals, meta = oracle.compress(W, 2, 4)
    groups = R * K // 4
    bits_per_group = (vals.nbytes + meta.nbytes) * 8 / groups
    assert bits_per_group == g["fp16_2of4_bits"]
    assert W.nbytes * 8 / groups == g["fp16_dense_bits"]
    assert round(100 * (1 - bits_per_group / g["fp16_dense_bits"])) == g["fp16_saving_percent_about"]
    # value block R x C/2, index block R x C/2 positions of 2 bits
    assert vals.shape == (R, K // 2)
    assert meta.size * 32 == R * (K // 2) * 2
    # the 2-bit index against a 16-bit and an 8-bit value; the INT8 saving
    assert 100 * 2 / 16 == g["index_overhead_fp16_percent"]
    assert 100 * 2 / 8 == g["index_overhead_int8_percent"]
    assert 100 * (1 - (2 * 8 + 2 * 2) / (4 * 8)) == g["int8_saving_percent"]


@pytest.mark.parametrize("R,K,n,m,words", [(16, 128, 2, 4, 64), (16, 24, 2, 4, 64), (17, 128, 2, 4, 128),
                                           (1, 24, 1, 8, 1), (1, 768, 1, 8, 10), (1, 256, 1, 4, 4),
                                           (4096, 4096, 2, 4, 4096 * 4096 // 32),
                                           (11008, 4096, 2, 4, 11008 * 4096 // 32), (3, 768, 1, 8, 30)])
def test_meta_sizes(R, K, n, m, words):
    assert oracle.meta_words(R, K, n, m) == words
    assert oracle.value_cols(K, n, m) == K * n // m


@pytest.mark.parametrize("m,bits,per_word", [(2, 1, 32), (4, 2, 16), (8, 3, 10), (16, 4, 8)])
def test_position_width_and_packing(m, bits, per_word):
    """b = ceil(log2 M) bits per survivor (the 2-bit positions of 2:4, generalised) and floor(32 / b) positions
    per 32-bit word, no position straddling two words; a row's words cover its K*N/M survivors."""
    assert oracle.index_bits(m) == bits == (m - 1).bit_length()
    assert oracle.positions_per_word(m) == per_word == 32 // bits
    for K, n in ((m, 1), (24 * m, 1), (24 * m, m // 2), (1000 * m, 1)):
        survivors = K // m * n
        assert oracle.meta_cols(K, n, m) == -(-survivors // per_word)
        if not (n == 2 and m == 4):
            assert oracle.meta_words(7, K, n, m) == 7 * oracle.meta_cols(K, n, m)


def test_tiled_2of4_every_group_once():
    """Each group's nibble sits in its own slot; everything else is the padding nibble."""
    R, K = 21, 200                       # padded to 32 rows x 256 columns
    W = wl.normal_bf16((R, K), 1.0, seed=12)
    _, meta = oracle.compress(W, 2, 4)
    assert meta.size == 2 * 2 * 64
    nibbles = (meta[:, None] >> (4 * np.arange(8))) & 0xF
    real = nibbles[nibbles != 0x4]
    # valid 2:4 position pairs only, and no more non-padding nibbles than groups
    assert set(np.unique(real).tolist()) <= {0x8, 0xC, 0x9, 0xD, 0xE}
    assert real.size <= R * K // 4
    # the padded rows 21..31 and columns 200..255 decode as positions (0,1)
    wide = np.zeros((32, 256), np.uint16)
    wide[:R, :K] = W
    _, meta_wide = oracle.compress(wide, 2, 4)
    pos_wide = oracle.positions(meta_wide, 32, 256, 2, 4)
    assert np.all(pos_wide[R:] == np.tile([0, 1], 64))


# The 64 words of one tiled 2:4 metadata block (16 rows x 128 columns), written
# out by hand from the layout description: lane l = 0..15 holds rows l mod 8
# (bits 0-15) and 8 + l mod 8 (bits 16-31); its word q = 0..3 covers the
# 16 columns starting at 32q + 16 (l / 8); four nibbles per row half, in column
# order.  Entry: (row in bits 0-15, row in bits 16-31, first column).
TILED_BLOCK_WORDS = [
    (0, 8, 0), (0, 8, 32), (0, 8, 64), (0, 8, 96),           # words 0-3, lane 0
    (1, 9, 0), (1, 9, 32), (1, 9, 64), (1, 9, 96),           # words 4-7, lane 1
    (2, 10, 0), (2, 10, 32), (2, 10, 64), (2, 10, 96),       # words 8-11, lane 2
    (3, 11, 0), (3, 11, 32), (3, 11, 64), (3, 11, 96),       # words 12-15, lane 3
    (4, 12, 0), (4, 12, 32), (4, 12, 64), (4, 12, 96),       # words 16-19, lane 4
    (5, 13, 0), (5, 13, 32), (5, 13, 64), (5, 13, 96),       # words 20-23, lane 5
    (6, 14, 0), (6, 14, 32), (6, 14, 64), (6, 14, 96),       # words 24-27, lane 6
    (7, 15, 0), (7, 15, 32), (7, 15, 64), (7, 15, 96),       # words 28-31, lane 7
    (0, 8, 16), (0, 8, 48), (0, 8, 80), (0, 8, 112),         # words 32-35, lane 8
    (1, 9, 16), (1, 9, 48), (1, 9, 80), (1, 9, 112),         # words 36-39, lane 9
    (2, 10, 16), (2, 10, 48), (2, 10, 80), (2, 10, 112),     # words 40-43, lane 10
    (3, 11, 16), (3, 11, 48), (3, 11, 80), (3, 11, 112),     # words 44-47, lane 11
    (4, 12, 16), (4, 12, 48), (4, 12, 80), (4, 12, 112),     # words 48-51, lane 12
    (5, 13, 16), (5, 13, 48), (5, 13, 80), (5, 13, 112),     # words 52-55, lane 13
    (6, 14, 16), (6, 14, 48), (6, 14, 80), (6, 14, 112),     # words 56-59, lane 14
    (7, 15, 16), (7, 15, 48), (7, 15, 80), (7, 15, 112),     # words 60-63, lane 15
]


def _slot_from_table(r, g):
    """(word, bit) of group g (columns 4g..4g+3) of row r inside one block, by table lookup."""
    hits = [(w, 16 * (r == hi) + 4 * ((4 * g - c) // 4))
            for w, (lo, hi, c) in enumerate(TILED_BLOCK_WORDS) if r in (lo, hi) and c <= 4 * g < c + 16]
    assert len(hits) == 1
    return hits[0]


def _planted_slot(R, K, r, g):
    """Compress a matrix that is zero except group g of row r = [0, 0, 1, 1]
    (positions 2, 3: nibble 0xE); every other group is all-zero (nibble 0x4).
    Returns the (word, bit) of the only 0xE nibble."""
    W = np.zeros((R, K), np.uint16)
    W[r, 4 * g + 2:4 * g + 4] = bits_of([1.0, 1.0])
    _, meta = oracle.compress(W, 2, 4)
    nib = (meta[:, None] >> (4 * np.arange(8))) & 0xF
    assert np.count_nonzero(nib == 0xE) == 1 and np.count_nonzero(nib == 0x4) == nib.size - 1
    w, j = np.argwhere(nib == 0xE)[0]
    return int(w), int(4 * j)


def test_tiled_2of4_slot_map_matches_hand_table():
    """Every (row, group) of one block lands at the word and bit of the hand-written table."""
    for r in range(16):
        for g in range(32):
            assert _planted_slot(16, 128, r, g) == _slot_from_table(r, g), (r, g)


@pytest.mark.parametrize("r,g", [(21, 67), (16, 0), (31, 95), (3, 40), (30, 33)])
def test_tiled_2of4_block_order(r, g):
    """Blocks follow one another row block by row block: block (rb, cb) of a
    32 x 384 matrix (three 128-column blocks per row block) starts at word
    (3 rb + cb) * 64."""
    rb, cb = r // 16, g // 32
    w, bit = _slot_from_table(r % 16, g % 32)
    assert _planted_slot(32, 384, r, g) == ((3 * rb + cb) * 64 + w, bit)


# ---------------------------------------------------------------------------
# Decompression
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("n,m", PATTERNS)
def test_roundtrip(n, m):
    W = wl.integer_bf16((19, 8 * m), -2, 2, seed=11)  # many zeros and ties
    W[0, :m] = bits_of([-0.0] * m)                    # a group of negative zeros
    vals, meta = oracle.compress(W, n, m)
    mask = oracle.prune_mask(W, n, m)
    D = oracle.decompress(vals, meta, W.shape[1], n, m)
    assert np.array_equal(D, np.where(mask == 1, W, np.uint16(0)))
    vals2, meta2 = oracle.compress(D, n, m)
    assert np.array_equal(vals2, vals) and np.array_equal(meta2, meta)


# ---------------------------------------------------------------------------
# Sparse GEMM
# ---------------------------------------------------------------------------
def test_k8_example(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "k8_example.json")))
    W = bits_of([g["a_row"]])
    vals, meta = oracle.compress(W, 2, 4)
    assert vals.shape[1] == g["sparse_products"] and W.shape[1] == g["dense_products"]
    assert np.array_equal(f64(vals[0]), np.array(g["expected_values"]))
    pos = positions(meta, 1, 8, 2, 4)[0]
    assert [pos[0:2], pos[2:4]] == g["expected_positions"]
    X = bits_of(np.array(g["b_col"], dtype=np.float32).reshape(8, 1))
    y = oracle.spmm(vals, meta, 2, 4, 8, X)
    assert y[0, 0] == g["expected_dot"]


@pytest.mark.parametrize("n,m", [(2, 4), (1, 4), (1, 8), (3, 8)])
def test_spmm_equals_dense_of_masked(n, m):
    R, K, T = 23, 64 * m // 4 + 8 * m, 19
    W = wl.normal_bf16((R, K), 1.0, seed=21)
    X = wl.normal_bf16((K, T), 1.0, seed=22)
    vals, meta = oracle.compress(W, n, m)
    Wm = np.where(oracle.prune_mask(W, n, m) == 1, f64(W), 0.0)
    ref = Wm @ f64(X)
    y = oracle.spmm(vals, meta, n, m, K, X)
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12)
    yd = oracle.dense_gemm(oracle.decompress(vals, meta, K, n, m), X)
    np.testing.assert_allclose(yd, ref, rtol=1e-12, atol=1e-12)


def test_spmm_integer_exact():
    """Integer inputs: every partial sum is an exact integer, so the result is exact."""
    R, K, T = 17, 96, 13
    W = wl.integer_bf16((R, K), -8, 8, seed=31)
    X = wl.integer_bf16((K, T), -8, 8, seed=32)
    vals, meta = oracle.compress(W, 2, 4)
    Wm = np.where(oracle.prune_mask(W, 2, 4) == 1, f64(W), 0.0).astype(np.int64)
    ref = Wm @ f64(X).astype(np.int64)
    assert np.array_equal(oracle.spmm(vals, meta, 2, 4, K, X), ref.astype(np.float64))


def test_spmm_bruteforce_tiny():
    """Tiny case worked by hand-rolled loops: subset selection, then pure-Python dot products."""
    rng = np.random.default_rng(5)
    for n, m in [(2, 4), (1, 4), (1, 8)]:
        Wf = rng.integers(-3, 4, size=(3, 2 * m)).astype(np.float32)
        Xf = rng.integers(-3, 4, size=(2 * m, 2)).astype(np.float32)
        W, X = bits_of(Wf), bits_of(Xf)
        vals, meta = oracle.compress(W, n, m)
        y = oracle.spmm(vals, meta, n, m, 2 * m, X)
        for r in range(3):
            kept = []
            for g0 in range(0, 2 * m, m):
                w = [float(v) for v in Wf[r, g0:g0 + m]]
                win = [S for S in itertools.combinations(range(m), n)
                       if all(_preferred(w, i, j) for i in S for j in range(m) if j not in S)]
                kept += [g0 + p for p in win[0]]
            for t in range(2):
                assert y[r, t] == sum(float(Wf[r, k]) * float(Xf[k, t]) for k in kept)


def test_sampled_matches_full():
    R, K, T = 31, 256, 40
    W = wl.normal_bf16((R, K), 0.02, seed=41)
    X = wl.normal_bf16((K, T), 1.0, seed=42)
    idx = wl.permutation(K, 43)
    vals, meta = oracle.compress(W, 2, 4)
    full = oracle.spmm(vals, meta, 2, 4, K, X, idx)
    rows = np.array([0, 30, 7, 15, 30]); cols = np.array([0, 39, 20, 1, 0])
    out, mag = oracle.spmm_sampled(vals, meta, 2, 4, K, X, rows, cols, idx)
    assert np.array_equal(out, full[rows, cols])
    Wm = np.abs(f64(oracle.decompress(vals, meta, K, 2, 4)))
    np.testing.assert_allclose(mag, (Wm @ np.abs(f64(X)[idx]))[rows, cols], rtol=1e-12)


def test_dense_gemm_matches_numpy():
    W = wl.normal_bf16((9, 40), 1.0, seed=51)
    X = wl.normal_bf16((40, 11), 1.0, seed=52)
    Y, A = oracle.dense_gemm(W, X, with_abs=True)
    np.testing.assert_allclose(Y, f64(W) @ f64(X), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(A, np.abs(f64(W)) @ np.abs(f64(X)), rtol=1e-12)


# ---------------------------------------------------------------------------
# Permuted input read, y = (W Pi) x
# ---------------------------------------------------------------------------
def test_identity_permutation_reduces_to_plain():
    R, K, T = 20, 128, 24
    W = wl.normal_bf16((R, K), 0.02, seed=61)
    X = wl.normal_bf16((K, T), 1.0, seed=62)
    vals, meta = oracle.compress(W, 2, 4)
    a = oracle.spmm(vals, meta, 2, 4, K, X)
    b = oracle.spmm(vals, meta, 2, 4, K, X, np.arange(K, dtype=np.int32))
    assert np.array_equal(a, b)


def test_permutation_matrix_form():
    """y = (W' Pi) X with an explicit K x K permutation matrix, Pi[k, idx[k]] = 1."""
    R, K, T = 6, 16, 5
    W = wl.integer_bf16((R, K), -4, 4, seed=71)
    X = wl.integer_bf16((K, T), -4, 4, seed=72)
    idx = wl.permutation(K, 73)
    vals, meta = oracle.compress(W, 2, 4)
    Wm = f64(oracle.decompress(vals, meta, K, 2, 4))
    Pi = np.zeros((K, K))
    Pi[np.arange(K), idx] = 1.0
    assert np.array_equal(oracle.spmm(vals, meta, 2, 4, K, X, idx), (Wm @ Pi) @ f64(X))


def test_permutation_equals_permuted_input():
    R, K, T = 12, 64, 9
    W = wl.normal_bf16((R, K), 1.0, seed=81)
    X = wl.normal_bf16((K, T), 1.0, seed=82)
    idx = wl.permutation(K, 83)
    vals, meta = oracle.compress(W, 1, 8)
    assert np.array_equal(oracle.spmm(vals, meta, 1, 8, K, X, idx),
                          oracle.spmm(vals, meta, 1, 8, K, np.ascontiguousarray(X[idx])))


# ---------------------------------------------------------------------------
# PATCH hybrid
# ---------------------------------------------------------------------------
def test_hybrid_special_cases():
    R, K, T, tile = 40, 96, 7, 32
    W = wl.integer_bf16((R, K), -5, 5, seed=91)
    X = wl.integer_bf16((K, T), -5, 5, seed=92)
    tiles = (-(-R // tile), -(-K // tile))
    dense = oracle.hybrid_spmm(W, np.zeros(tiles, np.uint8), X, tile)
    assert np.array_equal(dense, f64(W) @ f64(X))
    vals, meta = oracle.compress(W, 2, 4)
    sparse = oracle.hybrid_spmm(W, np.ones(tiles, np.uint8), X, tile)
    assert np.array_equal(sparse, oracle.spmm(vals, meta, 2, 4, K, X))


def test_hybrid_mixed_tiles():
    R, K, T, tile = 64, 128, 10, 32
    W = wl.normal_bf16((R, K), 0.02, seed=101)
    X = wl.normal_bf16((K, T), 1.0, seed=102)
    tm = wl.tile_map(2, 4, 0.5, seed=103)
    mask = oracle.prune_mask(W, 2, 4)
    sparse_el = np.kron(tm, np.ones((tile, tile), np.uint8)).astype(bool)
    Weff = np.where(sparse_el & (mask == 0), 0.0, f64(W))
    np.testing.assert_allclose(oracle.hybrid_spmm(W, tm, X, tile), Weff @ f64(X), rtol=1e-12, atol=1e-14)
    assert np.array_equal(f64(oracle.hybrid_weights(W, tm, tile)), Weff)


def test_rejects_bad_arguments():
    W = wl.normal_bf16((4, 10), 1.0, seed=1)
    with pytest.raises(ValueError):
        oracle.compress(W, 2, 4)      # K % M != 0
    with pytest.raises(ValueError):
        oracle.compress(wl.normal_bf16((4, 12), 1.0, 1), 4, 4)  # N must be below M
    with pytest.raises(ValueError):
        oracle.compress(wl.normal_bf16((4, 12), 1.0, 1), 1, 3)  # M not a power of two
