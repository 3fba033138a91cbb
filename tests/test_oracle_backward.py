"""Pins of the backward oracle functions (input gradient and value gradient).

Both are pinned through the forward GEMM oracle, which has its own pins, and
through identities of linear algebra that hold exactly on small-integer data
(every product and sum is an exact integer in fp64):

  * adjoint:  <dY, (W' Pi) X> = <spmm_t(dY), X>  for any X and dY;
  * values:   <dY, (W' Pi) X> = sum_rj dV[r][j] V[r][j];
  * gradient: adding 1 to one input entry (or one stored value) changes
    <dY, y> by exactly that entry of spmm_t (or of sddmm).

A swapped gather/scatter direction, a wrong survivor column, a dropped or
doubled term, or a transposed operand each breaks one of them.
"""
import numpy as np
import pytest

import oracle
import workloads as wl

PATTERNS = [(2, 4), (1, 4), (1, 8), (3, 8), (5, 16)]


def f64(bits):
    return wl.bf16_to_f32(bits).astype(np.float64)


def layer(n, m, R=13, K=48, T=5, seed=0):
    W = wl.integer_bf16((R, K), -4, 4, seed=seed)
    vals, meta = oracle.compress(W, n, m)
    X = wl.integer_bf16((K, T), -3, 3, seed=seed + 1)
    dY = wl.integer_bf16((R, T), -3, 3, seed=seed + 2)
    return vals, meta, X, dY


def index_maps(K, seed):
    rng = np.random.default_rng(seed)
    perm = rng.permutation(K).astype(np.int32)
    rough = rng.integers(0, K, K).astype(np.int32)  # repeated entries
    rough[[1, 7]] = [-1, K + 3]  # entries outside [0, K) read zero rows
    return [None, perm, rough]


@pytest.mark.parametrize("n,m", PATTERNS)
def test_adjoint_identity(n, m):
    vals, meta, X, dY = layer(n, m, seed=n * 10 + m)
    K = X.shape[0]
    for idx in index_maps(K, m):
        y = oracle.spmm(vals, meta, n, m, K, X, idx)
        dX = oracle.spmm_t(vals, meta, n, m, K, dY, idx)
        assert np.sum(f64(dY) * y) == np.sum(dX * f64(X))


@pytest.mark.parametrize("n,m", PATTERNS)
def test_value_gradient_identity(n, m):
    vals, meta, X, dY = layer(n, m, seed=n * 10 + m + 100)
    R, K = vals.shape[0], X.shape[0]
    for idx in index_maps(K, m + 1):
        y = oracle.spmm(vals, meta, n, m, K, X, idx)
        dV = oracle.sddmm(meta, n, m, R, K, dY, X, idx)
        assert np.sum(f64(dY) * y) == np.sum(dV * f64(vals))


@pytest.mark.parametrize("n,m", [(2, 4), (1, 8), (3, 8)])
def test_input_gradient_by_finite_difference(n, m):
    vals, meta, X, dY = layer(n, m, seed=n * 10 + m + 200)
    K, T = X.shape
    rng = np.random.default_rng(3)
    for idx in index_maps(K, m + 2):
        base = np.sum(f64(dY) * oracle.spmm(vals, meta, n, m, K, X, idx))
        dX = oracle.spmm_t(vals, meta, n, m, K, dY, idx)
        for _ in range(12):
            i, t = int(rng.integers(0, K)), int(rng.integers(0, T))
            Xp = X.copy()
            Xp[i, t] = wl.bf16_bits(np.array([f64(X[i:i + 1, t])[0] + 1.0], np.float32))[0]
            moved = np.sum(f64(dY) * oracle.spmm(vals, meta, n, m, K, Xp, idx))
            assert moved - base == dX[i, t]


@pytest.mark.parametrize("n,m", [(2, 4), (1, 4), (5, 16)])
def test_value_gradient_by_finite_difference(n, m):
    vals, meta, X, dY = layer(n, m, seed=n * 10 + m + 300)
    R, K = vals.shape[0], X.shape[0]
    rng = np.random.default_rng(4)
    for idx in index_maps(K, m + 3):
        base = np.sum(f64(dY) * oracle.spmm(vals, meta, n, m, K, X, idx))
        dV = oracle.sddmm(meta, n, m, R, K, dY, X, idx)
        for _ in range(12):
            r, j = int(rng.integers(0, R)), int(rng.integers(0, vals.shape[1]))
            V2 = vals.copy()
            V2[r, j] = wl.bf16_bits(np.array([f64(vals[r:r + 1, j])[0] + 1.0], np.float32))[0]
            moved = np.sum(f64(dY) * oracle.spmm(V2, meta, n, m, K, X, idx))
            assert moved - base == dV[r, j]


def test_tolerance_scales_bound_the_results():
    vals, meta, X, dY = layer(2, 4, seed=7)
    R, K = vals.shape[0], X.shape[0]
    dX, aX = oracle.spmm_t(vals, meta, 2, 4, K, dY, None, with_abs=True)
    dV, aV = oracle.sddmm(meta, 2, 4, R, K, dY, X, None, with_abs=True)
    assert np.all(np.abs(dX) <= aX) and np.all(np.abs(dV) <= aV)
    assert np.any(aX > np.abs(dX)) and np.any(aV > np.abs(dV))  # mixed signs do cancel somewhere
