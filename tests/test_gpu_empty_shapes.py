"""Degenerate sizes on every GEMM entry point: no rows, no columns or an empty reduction.

An output with no elements (R = 0 or T = 0) is left alone and nothing is
launched; an empty reduction (K = 0, or no kept diagonals) gives exact zeros
over the R x T output and leaves the padding columns of its rows untouched.
The output buffers start filled with a sentinel so that both are visible.
"""
import numpy as np
import pytest
import torch

import sparse_gemm_nm_b200 as nm
from gpu_helpers import DEV

pytestmark = pytest.mark.gpu

SENTINEL = 5.0
LD = 64  # row stride of every buffer (elements); the calls use at most 48 columns


def bf16(rows, cols=LD, value=0.0):
    return torch.full((rows, cols), value, dtype=torch.bfloat16, device=DEV)


def check(Y, R, T, zero_filled):
    """Y's first R rows x T columns are zeros when zero_filled, else untouched; the rest untouched."""
    y = Y.float().cpu().numpy()
    expect = np.full(y.shape, SENTINEL, np.float32)
    if zero_filled:
        expect[:R, :T] = 0.0
    assert np.array_equal(y, expect)


def launches(fn):
    torch.cuda.synchronize()
    before = nm.nm_launch_count()
    fn()
    torch.cuda.synchronize()
    nm.nm_device_status()
    return nm.nm_launch_count() - before


# (R, K, T) of each case and whether the output is an empty sum
CASES = [((0, 64, 32), False), ((48, 64, 0), False), ((48, 0, 32), True)]


@pytest.mark.parametrize("dims,zero", CASES)
def test_spmm_plain_permuted_and_hybrid(dims, zero):
    R, K, T = dims
    W = bf16(48, 64, 0.5)
    vals = bf16(48, 32, 0.5)
    meta = torch.zeros((nm.nm_meta_words(48, 64, 2, 4),), dtype=torch.int32, device=DEV)
    X = bf16(64, LD, 1.0)
    idx = torch.arange(64, dtype=torch.int32, device=DEV)
    tmap = torch.ones((1, 1), dtype=torch.uint8, device=DEV)
    calls = {
        "spmm": lambda Y: nm.nm_spmm(vals, meta, 2, 4, R, K, X, LD, T, Y, LD),
        "permuted": lambda Y: nm.nm_spmm_permuted(vals, meta, 2, 4, R, K, idx, X, LD, T, Y, LD),
        "hybrid": lambda Y: nm.nm_hybrid_spmm(W, 64, vals, meta, tmap, 128, R, K, X, LD, T, Y, LD),
        "prune_spmm": lambda Y: nm.nm_prune_spmm(W, 64, 2, 4, R, K, idx, X, LD, T, Y, LD),
    }
    for name, call in calls.items():
        Y = bf16(48, LD, SENTINEL)
        n = launches(lambda: call(Y))
        assert n == (1 if zero else 0), name
        check(Y, R, T, zero)


@pytest.mark.parametrize("dims,zero", CASES)
def test_spmm_int8_and_tf32(dims, zero):
    R, K, T = dims
    v8 = torch.ones((48, 32), dtype=torch.int8, device=DEV)
    m8 = torch.zeros((nm.nm_meta_words(48, 64, 2, 4),), dtype=torch.int32, device=DEV)
    X8 = torch.ones((64, LD), dtype=torch.int8, device=DEV)
    Y8 = torch.full((48, LD), int(SENTINEL), dtype=torch.int32, device=DEV)
    n = launches(lambda: nm.nm_spmm_i8(v8, m8, R, K, X8, LD, T, Y8, LD))
    assert n == (1 if zero else 0)
    check(Y8, R, T, zero)
    vf = torch.ones((48, 32), dtype=torch.float32, device=DEV)
    mf = torch.zeros((nm.nm_meta_words(48, 64, 1, 2),), dtype=torch.int32, device=DEV)
    Xf = torch.ones((64, LD), dtype=torch.float32, device=DEV)
    Yf = torch.full((48, LD), SENTINEL, dtype=torch.float32, device=DEV)
    n = launches(lambda: nm.nm_spmm_tf32(vf, mf, R, K, Xf, LD, T, Yf, LD))
    assert n == (1 if zero else 0)
    check(Yf, R, T, zero)


@pytest.mark.parametrize("dims,zero", [((0, 64, 32), True),     # dX = W'^T dY with no rows of W': zeros
                                       ((48, 64, 0), False),    # no columns of dY: nothing
                                       ((48, 0, 32), False)])   # dX has no rows: nothing
def test_spmm_t(dims, zero):
    R, K, T = dims
    vals = bf16(48, 32, 0.5)
    meta = torch.zeros((nm.nm_meta_words(48, 64, 2, 4),), dtype=torch.int32, device=DEV)
    dY = bf16(48, LD, 1.0)
    dX = bf16(64, LD, SENTINEL)
    n = launches(lambda: nm.nm_spmm_t(vals, meta, 2, 4, R, K, None, dY, LD, T, dX, LD))
    assert n == (1 if zero else 0)
    check(dX, K, T, zero)


@pytest.mark.parametrize("dims,D,zero", [((0, 64, 32), 4, False), ((48, 64, 0), 4, False),
                                         ((48, 64, 32), 0, True)])  # no kept diagonal: zeros
def test_diag_spmm(dims, D, zero):
    R, K, T = dims
    V = bf16(max(D, 1), 48, 0.5)
    offsets = torch.arange(max(D, 1), dtype=torch.int32, device=DEV)
    X = bf16(64, LD, 1.0)
    Y = bf16(48, LD, SENTINEL)
    n = launches(lambda: nm.nm_diag_spmm(V, offsets, D, R, K, None, X, LD, T, Y, LD))
    assert n == (1 if zero else 0)
    check(Y, R, T, zero)
