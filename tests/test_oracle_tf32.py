"""Pins of the float32 (TF32-path) oracle functions: 1:2 selection, push-left
values, metadata, round trip and the GEMM.

"M:N sparsity on NVIDIA tensor cores" (the passage on the formats the sparse
tensor cores take): for TF32 the 2:4 block halves to 1:2.  The rule is the
one of the bf16 path on the float32 value: the larger magnitude survives,
equal magnitudes go to the lower index, a NaN ranks above every number.

Pins: the survivor of every ordered pair over an alphabet with signed zeros,
infinities and NaN, written out by hand below; the bf16 oracle on values that
are exactly bf16 (an independent selection and packing of the same rule);
the round trip; the 1-bit LSB-first metadata of a row built by hand; and the
GEMM against a float64 matmul of the written-out matrix.
"""
import math

import numpy as np
import pytest

import oracle
import workloads as wl

ALPHABET = [-2.0, -1.0, -0.0, 0.0, 1.0, 2.0, math.inf, -math.inf, math.nan]


def expected_survivor(a: float, b: float) -> int:
    """Position (0 or 1) of the survivor of the pair (a, b), from the rule as stated."""
    if math.isnan(a):
        return 0
    if math.isnan(b):
        return 1
    return 0 if abs(a) >= abs(b) else 1


def test_every_pair_of_the_alphabet():
    pairs = [(a, b) for a in ALPHABET for b in ALPHABET]
    W = np.array([x for ab in pairs for x in ab], np.float32).reshape(1, -1)
    mask = oracle.prune_mask_f32(W)
    vals, meta = oracle.compress_f32(W)
    for i, (a, b) in enumerate(pairs):
        p = expected_survivor(a, b)
        assert mask[0, 2 * i + p] == 1 and mask[0, 2 * i + 1 - p] == 0, (a, b)
        assert vals[0, i] == W.view(np.uint32)[0, 2 * i + p], (a, b)  # bits copied, -0.0 and NaN included
        assert (meta[i // 32] >> (i % 32)) & 1 == p, (a, b)


def test_metadata_of_a_hand_built_row():
    # survivors at positions 1, 0, 0, 1, 1 of five pairs, then 35 pairs won by the first element
    row = [0.0, 3.0, 4.0, 1.0, 5.0, -5.0, 1.0, -2.0, 0.5, 0.75] + [1.0, 0.0] * 35
    W = np.array([row], np.float32)
    vals, meta = oracle.compress_f32(W)
    assert meta.shape == (2,)  # 40 survivors, 32 per word
    assert meta[0] == 0b11001 and meta[1] == 0
    assert vals.view(np.float32)[0, :5].tolist() == [3.0, 4.0, 5.0, -2.0, 0.75]


def test_agrees_with_the_bf16_oracle_on_bf16_values():
    Wb = wl.normal_bf16((37, 64), 1.0, seed=5)
    Wb[0, :8] = [0x0000, 0x8000, 0x3F80, 0xBF80, 0x7FC0, 0x3F80, 0x7F80, 0xFF80]  # ties, NaN, +-Inf
    Wf = (Wb.astype(np.uint32) << 16)
    vb, mb = oracle.compress(Wb, 1, 2)
    vf, mf = oracle.compress_f32(Wf, 1, 2)
    assert np.array_equal(mb, mf)
    assert np.array_equal(vf, vb.astype(np.uint32) << 16)


@pytest.mark.parametrize("n,m", [(1, 2), (2, 4), (1, 4)])
def test_round_trip(n, m):
    W = wl.normal_f32((29, 48), 1.0, seed=n + m)
    W[3, :4] = [0.0, -0.0, 0.0, -0.0]
    mask = oracle.prune_mask_f32(W, n, m)
    assert np.all(mask.reshape(29, -1, m).sum(axis=2) == n)  # exactly N per group
    vals, meta = oracle.compress_f32(W, n, m)
    back = oracle.decompress_f32(vals, meta, 48, n, m)
    assert np.array_equal(back, np.where(mask == 1, W.view(np.uint32), np.uint32(0)))
    v2, m2 = oracle.compress_f32(back, n, m)
    assert np.array_equal(v2, vals) and np.array_equal(m2, meta)


def test_gemm_equals_the_dense_product():
    rng = np.random.default_rng(11)
    W = rng.normal(size=(23, 40)).astype(np.float32)
    X = rng.normal(size=(40, 13)).astype(np.float32)
    vals, meta = oracle.compress_f32(W)
    dense = oracle.decompress_f32(vals, meta, 40).view(np.float32).astype(np.float64)
    Y, A = oracle.spmm_f32(vals, meta, 40, X, with_abs=True)
    ref = dense @ X.astype(np.float64)
    assert np.allclose(Y, ref, rtol=1e-13, atol=1e-13)
    assert np.allclose(A, np.abs(dense) @ np.abs(X.astype(np.float64)), rtol=1e-13, atol=1e-13)
    Wi = rng.integers(-8, 9, size=(9, 16)).astype(np.float32)
    Xi = rng.integers(-8, 9, size=(16, 7)).astype(np.float32)
    vi, mi = oracle.compress_f32(Wi)
    Yi = oracle.spmm_f32(vi, mi, 16, Xi)
    assert np.array_equal(Yi, oracle.decompress_f32(vi, mi, 16).view(np.float32).astype(np.float64) @ Xi)
