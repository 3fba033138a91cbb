"""Pins of the diagonal-pattern oracle functions.

* planted structure: a weight that is zero off D chosen diagonals selects
  exactly those D offsets, whatever their values;
* ties: equal scores keep the lowest offsets; D = K keeps every offset;
* NaN: a diagonal holding a NaN ranks first;
* expand/compress round trip, one entry per row and diagonal, wrapping
  rows when R > K;
* the GEMM equals the oracle's dense GEMM of the expanded matrix and numpy's
  float64 matmul of it, with and without an index map.
"""
import numpy as np
import pytest

import oracle
import workloads as wl


def f64(bits):
    return wl.bf16_to_f32(bits).astype(np.float64)


@pytest.mark.parametrize("R,K,D", [(32, 32, 5), (48, 16, 3), (16, 40, 7)])
def test_planted_diagonals_are_selected(R, K, D):
    rng = np.random.default_rng(R + K)
    planted = np.sort(rng.choice(K, D, replace=False)).astype(np.int32)
    W = np.zeros((R, K), np.uint16)
    vals = wl.integer_bf16((D, R), 1, 9, seed=3)
    for d, o in enumerate(planted):
        for r in range(R):
            W[r, (r + o) % K] = vals[d, r]
    assert np.array_equal(oracle.diag_select(W, D), planted)
    V = oracle.diag_compress(W, planted)
    assert np.array_equal(V, vals)
    assert np.array_equal(oracle.diag_expand(V, planted, K), W)


def test_ties_and_full_selection():
    W = wl.bf16_bits(np.ones((8, 12), np.float32))  # every diagonal scores 8
    assert np.array_equal(oracle.diag_select(W, 5), np.arange(5, dtype=np.int32))
    assert np.array_equal(oracle.diag_select(W, 12), np.arange(12, dtype=np.int32))


def test_nan_diagonal_ranks_first():
    W = wl.bf16_bits(np.full((8, 12), 100.0, np.float32))
    W[2, (2 + 7) % 12] = 0x7FC0  # NaN on diagonal 7
    assert 7 in oracle.diag_select(W, 1)


@pytest.mark.parametrize("R,K,D,T", [(24, 16, 4, 5), (16, 24, 6, 3), (40, 40, 9, 7)])
def test_gemm_equals_dense_product(R, K, D, T):
    W = wl.integer_bf16((R, K), -5, 5, seed=R * K)
    offs = oracle.diag_select(W, D)
    V = oracle.diag_compress(W, offs)
    Wd = oracle.diag_expand(V, offs, K)
    assert np.count_nonzero(f64(Wd)) <= R * D
    X = wl.integer_bf16((K, T), -4, 4, seed=T)
    idx = np.random.default_rng(1).permutation(K).astype(np.int32)
    for ix in (None, idx):
        y = oracle.diag_spmm(V, offs, K, X, ix)
        Xp = X if ix is None else X[ix]
        assert np.array_equal(y, oracle.dense_gemm(Wd, X, ix))
        assert np.array_equal(y, f64(Wd) @ f64(Xp))
