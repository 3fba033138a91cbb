"""Pins of the diagonal-pattern oracle functions.

* planted structure: a weight that is zero off D chosen diagonals selects
  exactly those D offsets, whatever their values;
* ties: equal scores keep the lowest offsets; D = K keeps every offset;
* scores on non-integer weights equal the float64 sums numpy takes along each
  diagonal (within double rounding), and the selection is the top D of a
  library sort of them;
* two diagonals whose scores differ by less than float32 can resolve: the
  exactly larger one is kept (a float32 score would tie them);
* the selection checker used by the GPU tests accepts the oracle's choice and
  a near-tie swap, and rejects a clearly wrong one;
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


def _diag(W, o):
    R, K = W.shape
    r = np.arange(R)
    return W[r, (r + o) % K]


@pytest.mark.parametrize("R,K,D", [(200, 64, 9), (37, 90, 20), (512, 48, 5)])
def test_scores_equal_numpy_float64_sums(R, K, D):
    W = wl.normal_bf16((R, K), 0.02, seed=R * 7 + K)
    s = oracle.diag_scores(W)
    ref = np.array([np.abs(f64(_diag(W, o))).sum() for o in range(K)])
    assert np.allclose(s, ref, rtol=R * 2.0 ** -52, atol=0)
    order = np.lexsort((np.arange(K), -ref))  # library sort: score descending, then lower offset
    assert np.array_equal(oracle.diag_select(W, D), np.sort(order[:D]).astype(np.int32))


def test_gap_below_float32_resolution_goes_to_the_exactly_larger():
    # diagonal 0 sums 63 ones; diagonal 1 sums 63 ones and 2^-20.  The gap is a
    # quarter of float32's spacing at 63, so any float32 sum ties them (and the
    # tie rule would keep offset 0); the exact scores keep offset 1.
    R, K = 64, 16
    Wf = np.zeros((R, K), np.float32)
    for r in range(63):
        Wf[r, r % K] = 1.0
        Wf[r, (r + 1) % K] = 1.0
    Wf[63, (63 + 1) % K] = 2.0 ** -20
    W = wl.bf16_bits(Wf)
    assert np.float32(np.sum(f64(_diag(W, 1)), dtype=np.float32)) == np.float32(63.0)  # float32 cannot tell
    s = oracle.diag_scores(W)
    assert s[1] - s[0] == 2.0 ** -20
    assert oracle.diag_select(W, 1).tolist() == [1]
    # a float32 evaluation keeping offset 0 is still a valid selection; offset 2 is not
    assert oracle.diag_selection_errors(W, 1, [1]) == []
    assert oracle.diag_selection_errors(W, 1, [0]) == []
    assert oracle.diag_selection_errors(W, 1, [2]) != []
    assert oracle.diag_selection_errors(W, 1, [0], terms_exact=True) != []


def test_selection_checker():
    R, K, D = 96, 40, 8
    W = wl.normal_bf16((R, K), 0.02, seed=5)
    good = oracle.diag_select(W, D)
    assert oracle.diag_selection_errors(W, D, good) == []
    s = oracle.diag_scores(W)
    worst = np.argsort(s)[:D]
    assert oracle.diag_selection_errors(W, D, np.sort(worst)) != []
    assert oracle.diag_selection_errors(W, D, good[::-1]) != []          # not ascending
    assert oracle.diag_selection_errors(W, D, good[:-1]) != []           # too few
    # NaN diagonals must come first
    Wn = W.copy()
    Wn[3, (3 + 11) % K] = 0x7FC0
    assert 11 in oracle.diag_select(Wn, 1)
    assert oracle.diag_selection_errors(Wn, 1, oracle.diag_select(Wn, 1)) == []
    assert oracle.diag_selection_errors(Wn, 1, [int(np.argmax(s))] if np.argmax(s) != 11 else [0]) != []
    # exact small-integer data: ties must go to the lower offset
    Wt = wl.bf16_bits(np.ones((8, 12), np.float32))
    assert oracle.diag_selection_errors(Wt, 3, [0, 1, 2], terms_exact=True) == []
    assert oracle.diag_selection_errors(Wt, 3, [0, 1, 3], terms_exact=True) != []
