"""The allocation-free permuted GEMM (nm_spmm_permuted_noalloc) against the oracle.

nm_spmm_permuted_noalloc is for callers that cannot let the library take
device memory; it stages the gathered input in a fixed array inside the
library instead of a pool allocation.  Each case calls
it twice in a row with different inputs (the array keeps the previous call's
contents) and compares both outputs with nm_spmm_permuted's and with the
oracle, within the acceptance rule the other GEMM tests use.  This file is collected last on purpose.
"""
import numpy as np
import pytest
import torch

import oracle
import sparse_gemm_nm_b200 as nm
import workloads as wl
from gpu_helpers import DEV, assert_gemm_close, to_dev, to_dev_i32, values_f64

pytestmark = pytest.mark.gpu


def _bound(W, X, idx):
    """sum_k |w'_rk| |x_{idx[k],t}| in float64 (scale of the tolerance)."""
    vals, meta = oracle.compress(W, 2, 4)
    Wd = wl.bf16_to_f32(oracle.decompress(vals, meta, W.shape[1], 2, 4)).astype(np.float64)
    Xp = wl.bf16_to_f32(np.ascontiguousarray(X[idx])).astype(np.float64)
    return np.abs(Wd) @ np.abs(Xp)


def _run_noalloc(W, X, idx):
    """Run the allocation-free call and nm_spmm_permuted (the call that may
    allocate) on the same device inputs; return both outputs and the oracle's."""
    R, K = W.shape
    T = X.shape[1]
    vals, meta = nm.prune_compress(to_dev(W), 2, 4)
    Xd, idxd = to_dev(X), to_dev_i32(idx)
    y = torch.full((R, T), 5.0, dtype=torch.bfloat16, device=DEV)
    y_pool = torch.empty((R, T), dtype=torch.bfloat16, device=DEV)
    nm.nm_spmm_permuted_noalloc(vals, meta, 2, 4, R, K, idxd, Xd, T, T, y, T)
    nm.nm_spmm_permuted(vals, meta, 2, 4, R, K, idxd, Xd, T, T, y_pool, T)
    torch.cuda.synchronize()
    nm.nm_device_status()
    ov, om = oracle.compress(W, 2, 4)
    ref = oracle.dense_gemm(oracle.decompress(ov, om, K, 2, 4), X, idx)
    return values_f64(y), values_f64(y_pool), ref


@pytest.mark.parametrize("R,K,T,pair_cols", [
    (512, 1024, 512, 512),     # one chunk
    (128, 8192, 2304, 2304),   # chunks of 2048 + 256 columns (the array holds 2048 columns of K = 8192)
    (128, 8192, 2104, 2048),   # 2048 + a 56-column tail, too narrow for the two-SM kernel
    (128, 8192, 2248, 2248),   # 2048 + a 200-column tail (two-SM kernel, partial column tile)
])
def test_noalloc_matches_permuted_and_oracle_twice(R, K, T, pair_cols):
    for call in range(2):  # second call: new inputs, array still holds the first call's chunks
        W = wl.normal_bf16((R, K), 0.02, seed=1000 + 10 * call + K)
        X = wl.normal_bf16((K, T), 1.0, seed=2000 + 10 * call + T)
        idx = wl.permutation(K, 3000 + call)
        y, y_pool, ref = _run_noalloc(W, X, idx)
        bound = _bound(W, X, idx)
        assert_gemm_close(y, ref, bound, f"no-alloc call {call + 1} vs oracle")
        assert_gemm_close(y, y_pool, bound, f"no-alloc call {call + 1} vs nm_spmm_permuted")
        # columns served by two-SM chunks run the same kernel on the same gathered rows
        assert np.array_equal(y[:, :pair_cols], y_pool[:, :pair_cols])


def test_noalloc_other_shapes_run_as_permuted():
    R, K, T = 136, 1040, 64  # not a two-SM shape: nothing is staged
    W = wl.normal_bf16((R, K), 0.02, seed=5)
    X = wl.normal_bf16((K, T), 1.0, seed=6)
    idx = wl.permutation(K, 7)
    y, y_pool, ref = _run_noalloc(W, X, idx)
    assert_gemm_close(y, ref, _bound(W, X, idx), "delegated shape")
    assert_gemm_close(y, y_pool, _bound(W, X, idx), "delegated shape vs nm_spmm_permuted")


def test_noalloc_rejects_k_beyond_the_array():
    R, K, T = 256, 65536 + 128, 256
    vals = torch.zeros((R, K // 2), dtype=torch.bfloat16, device=DEV)
    meta = torch.zeros((nm.nm_meta_words(R, K, 2, 4),), dtype=torch.int32, device=DEV)
    X = torch.zeros((K, T), dtype=torch.bfloat16, device=DEV)
    idx = torch.arange(K, dtype=torch.int32, device=DEV)
    Y = torch.zeros((R, T), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(nm.NmError) as e:
        nm.nm_spmm_permuted_noalloc(vals, meta, 2, 4, R, K, idx, X, T, T, Y, T)
    assert e.value.status == nm.NM_ERR_UNSUPPORTED
    assert "staging array" in str(e.value)


def test_noalloc_other_patterns_stage_nothing():
    """1:8 on a two-SM shape: nm_spmm_permuted re-encodes it into a staged
    operand; the allocation-free call must run the one-SM kernel instead (one
    launch) and give the same result within the tolerance."""
    R, K, T = 256, 512, 256
    W = wl.normal_bf16((R, K), 0.02, seed=8)
    X = wl.normal_bf16((K, T), 1.0, seed=9)
    idx = wl.permutation(K, 10)
    vals, meta = nm.prune_compress(to_dev(W), 1, 8)
    Xd, idxd = to_dev(X), to_dev_i32(idx)
    y_ref = torch.empty((R, T), dtype=torch.bfloat16, device=DEV)
    y_new = torch.empty((R, T), dtype=torch.bfloat16, device=DEV)
    nm.nm_spmm_permuted(vals, meta, 1, 8, R, K, idxd, Xd, T, T, y_ref, T)
    before = nm.nm_launch_count()
    nm.nm_spmm_permuted_noalloc(vals, meta, 1, 8, R, K, idxd, Xd, T, T, y_new, T)
    assert nm.nm_launch_count() - before == 1
    torch.cuda.synchronize()
    nm.nm_device_status()
    vals_o, meta_o = oracle.compress(W, 1, 8)
    Wd = wl.bf16_to_f32(oracle.decompress(vals_o, meta_o, K, 1, 8)).astype(np.float64)
    Xp = wl.bf16_to_f32(np.ascontiguousarray(X[idx])).astype(np.float64)
    assert_gemm_close(values_f64(y_new), values_f64(y_ref), np.abs(Wd) @ np.abs(Xp), "1:8 no-alloc")
