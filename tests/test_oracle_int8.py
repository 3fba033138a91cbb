"""Pins of the INT8 oracle functions (2:4 on int8 weights).

* the pages' INT8 storage arithmetic (2-bit index = 25 % of an 8-bit value,
  37.5 % saving), from the golden fixture;
* the selection rule by brute force over an alphabet that holds -128, +-127,
  zeros and ties, and equal to the bf16 selection on the same values (every
  int8 is exact in bf16, so the two rules must agree, including |-128| = 128);
* decompress(compress(W)) == W where kept, 0 elsewhere;
* the GEMM equals numpy's int64 matmul of the decompressed matrix.
"""
import itertools
import json
import os

import numpy as np
import pytest

import oracle
import workloads as wl


def test_int8_storage_arithmetic(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "storage_bits.json")))
    R, K = 32, 1024
    W = wl.integer_i8((R, K), -128, 127, seed=1)
    vals, meta = oracle.compress_i8(W)
    groups = R * K // 4
    bits_per_group = (vals.nbytes + meta.nbytes) * 8 / groups
    assert bits_per_group == 2 * 8 + 2 * 2
    assert 100 * (1 - bits_per_group / (W.nbytes * 8 / groups)) == g["int8_saving_percent"]
    assert 100 * 2 / (8 * vals.itemsize) == g["index_overhead_int8_percent"]


def test_int8_selection_brute_force():
    alphabet = [-128, -127, -1, 0, 1, 5, -5, 127]
    groups = np.array(list(itertools.product(alphabet, repeat=4)), np.int8)  # 4096 groups, one per row
    mask = oracle.prune_mask_i8(groups, 2, 4)
    for g, mk in zip(groups, mask):
        mags = [abs(int(v)) for v in g]
        order = sorted(range(4), key=lambda i: (-mags[i], i))  # larger first, lower index on ties
        want = np.zeros(4, np.uint8)
        want[order[:2]] = 1
        assert np.array_equal(mk, want), (g, mk, want)


@pytest.mark.parametrize("n,m", [(2, 4), (1, 4), (1, 8), (3, 8)])
def test_int8_selection_equals_bf16_selection(n, m):
    W = wl.integer_i8((37, 64), -128, 127, seed=n + m)
    W[3, :8] = [-128, 127, 127, -128, 0, 0, 0, 0]
    as_bf16 = wl.bf16_bits(W.astype(np.float32))
    assert np.array_equal(oracle.prune_mask_i8(W, n, m), oracle.prune_mask(as_bf16, n, m))
    vals, meta = oracle.compress_i8(W, n, m)
    bvals, bmeta = oracle.compress(as_bf16, n, m)
    assert np.array_equal(meta, bmeta)
    assert np.array_equal(wl.bf16_bits(vals.astype(np.float32)), bvals)


@pytest.mark.parametrize("n,m", [(2, 4), (1, 8)])
def test_int8_roundtrip_and_gemm(n, m):
    R, K, T = 33, 128, 7
    W = wl.integer_i8((R, K), -128, 127, seed=11)
    X = wl.integer_i8((K, T), -128, 127, seed=12)
    vals, meta = oracle.compress_i8(W, n, m)
    Wd = oracle.decompress_i8(vals, meta, K, n, m)
    mask = oracle.prune_mask_i8(W, n, m).astype(bool)
    assert np.array_equal(Wd[mask], W[mask]) and np.all(Wd[~mask] == 0)
    assert np.all(mask.reshape(R, K // m, m).sum(axis=2) == n)
    Y = oracle.spmm_i8(vals, meta, K, X, n, m)
    assert np.array_equal(Y, Wd.astype(np.int64) @ X.astype(np.int64))
