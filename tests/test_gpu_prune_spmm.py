"""GPU prune + GEMM in one call (nm_prune_spmm) against the oracle.

The fused kernel (2:4, K % 128 == 0, T <= 64) selects every W tile in shared
memory and feeds the sparse MMA; its optional compressed output must equal the
oracle's compress bit for bit, and Y must meet the GEMM tolerance against the
oracle's prune -> decompress -> GEMM.  Other shapes and patterns take the
compress-then-GEMM route of the same entry point.
"""
import numpy as np
import pytest
import torch

import oracle
import sparse_gemm_nm_b200 as nm
import workloads as wl
from gpu_helpers import DEV, assert_gemm_close, bf16_rne_of, bits, to_dev, to_dev_i32, values_f64, words

pytestmark = pytest.mark.gpu


def reference(W, X, n, m, idx=None):
    ov, om = oracle.compress(W, n, m)
    Wd = oracle.decompress(ov, om, W.shape[1], n, m)
    y, mag = oracle.dense_gemm(Wd, X, idx, with_abs=True)
    return y, mag, ov, om


def padded(X):
    """K x T on the device with rows padded to 16 bytes (a T-column view of a wider buffer)."""
    K, T = X.shape
    buf = np.zeros((K, (T + 7) // 8 * 8), np.uint16)
    buf[:, :T] = X
    return to_dev(buf)[:, :T]


def run(W, X, n, m, idx=None, out_dtype=torch.bfloat16, keep=True):
    out = nm.prune_spmm(to_dev(W), n, m, padded(X), idx=None if idx is None else to_dev_i32(idx),
                        out_dtype=out_dtype, keep_compressed=keep)
    torch.cuda.synchronize()
    nm.nm_device_status()
    return out


# ----------------------------------------------------------------------------
# fused kernel
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("R,K,T", [(128, 128, 1), (300, 1024, 16), (200, 512, 33), (77, 384, 64),
                                   (640, 4096, 8), (1000, 2048, 24)])
@pytest.mark.parametrize("permuted", [False, True])
def test_fused_matches_oracle(R, K, T, permuted):
    W = wl.normal_bf16((R, K), 0.02, seed=R + 3 * K + T)
    X = wl.normal_bf16((K, T), 1.0, seed=T + 11)
    idx = wl.permutation(K, R + 5) if permuted else None
    Y, v, mt = run(W, X, 2, 4, idx)
    ref, mag, ov, om = reference(W, X, 2, 4, idx)
    assert_gemm_close(values_f64(Y), ref, mag, f"fused {R}x{K}x{T} permuted={permuted}")
    assert np.array_equal(bits(v), ov)
    assert np.array_equal(words(mt), om)


@pytest.mark.parametrize("out", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("T", [16, 32, 64])  # four stages (bn 16); three (bn 32, 64): a slot's uses alternate groups
def test_fused_integer_exact(out, T):
    R, K = 384, 4096  # several K ranges; every partial sum is an exact integer
    W = wl.integer_bf16((R, K), -8, 8, seed=201)
    X = wl.integer_bf16((K, T), -8, 8, seed=202)
    ref, _, ov, om = reference(W, X, 2, 4)
    Y, v, mt = run(W, X, 2, 4, out_dtype=out)
    if out == torch.float32:
        assert np.array_equal(Y.cpu().numpy().astype(np.float64), ref)
    else:
        assert np.array_equal(bits(Y), bf16_rne_of(ref))
    assert np.array_equal(bits(v), ov) and np.array_equal(words(mt), om)


def test_fused_ties_zeros_and_nonfinite_selection():
    """Selection inside the GEMM follows the compress rules (ties low, -0 == +0, NaN first)."""
    R, K, T = 64, 256, 16
    W = wl.integer_bf16((R, K), -2, 2, seed=211)
    W[3, :] = wl.bf16_bits(np.full(K, -0.0, np.float32))
    W[4, :] = 0
    nan, inf = float("nan"), float("inf")
    W[5, :] = wl.bf16_bits(np.array([nan, inf, 1.0, -inf] * (K // 4), np.float32))
    W[6, :] = wl.bf16_bits(np.array([1.0, nan, nan, 5.0] * (K // 4), np.float32))
    X = wl.integer_bf16((K, T), -3, 3, seed=212)
    _, v, mt = run(W, X, 2, 4)
    ov, om = oracle.compress(W, 2, 4)
    assert np.array_equal(bits(v), ov) and np.array_equal(words(mt), om)


def test_fused_equals_compress_then_gemm():
    """Same operand, same K ranges and MMA order as the two-call path: identical Y."""
    R, K, T = 1000, 4096, 16
    W = wl.normal_bf16((R, K), 0.02, seed=221)
    X = wl.normal_bf16((K, T), 1.0, seed=222)
    Wd, Xd = to_dev(W), to_dev(X)
    vals, meta = nm.prune_compress(Wd, 2, 4)
    Y2 = nm.spmm(vals, meta, 2, 4, K, Xd, out_dtype=torch.float32)
    Y1 = nm.prune_spmm(Wd, 2, 4, Xd, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.equal(Y1, Y2)


def test_fused_without_compressed_output():
    R, K, T = 256, 1024, 16
    W = wl.normal_bf16((R, K), 0.02, seed=231)
    X = wl.normal_bf16((K, T), 1.0, seed=232)
    Y = run(W, X, 2, 4, keep=False)
    ref, mag, _, _ = reference(W, X, 2, 4)
    assert_gemm_close(values_f64(Y), ref, mag, "fused, no side output")


def test_fused_launch_counts():
    R, K = 256, 1024
    W = to_dev(wl.normal_bf16((R, K), 0.02, seed=241))
    X = to_dev(wl.normal_bf16((K, 16), 1.0, seed=242))
    idx = to_dev_i32(wl.permutation(K, 243))
    Y = torch.empty((R, 16), dtype=torch.bfloat16, device=DEV)
    torch.cuda.synchronize()

    def launches(**kw):
        c0 = nm.nm_launch_count()
        nm.nm_prune_spmm(W, K, 2, 4, R, K, kw.get("idx"), X, 16, 16, Y, 16)
        torch.cuda.synchronize()
        return nm.nm_launch_count() - c0

    # 2 row tiles on ~148 SMs: K is split, so the partials need a second launch
    assert launches() == 2
    assert launches(idx=idx) == 3  # + the gather of the permuted rows


def test_decode_full_size_sampled():
    L = wl.workload("decode")[0]
    d = wl.make_layer(L)
    Y, v, mt = run(d.W, d.X, 2, 4)
    ov, om = oracle.compress(d.W, 2, 4)
    assert np.array_equal(bits(v), ov) and np.array_equal(words(mt), om)
    R, T = Y.shape
    rng = np.random.default_rng(5)
    rows = np.concatenate([rng.integers(0, R, 20000), [0, R - 1, 0, R - 1]])
    cols = np.concatenate([rng.integers(0, T, 20000), [0, T - 1, T - 1, 0]])
    ref, mag = oracle.spmm_sampled(ov, om, 2, 4, L.K, d.X, rows, cols, None)
    assert_gemm_close(values_f64(Y)[rows, cols], ref, mag, "fused decode sampled")


# ----------------------------------------------------------------------------
# compress-then-GEMM route of the same call
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("n,m,R,K,T", [(2, 4, 200, 1024, 100), (2, 4, 130, 96, 16), (1, 4, 300, 1024, 16),
                                       (1, 8, 256, 512, 264), (3, 4, 70, 256, 24), (2, 4, 300, 1024, 264),
                                       (2, 4, 600, 384, 520)])
@pytest.mark.parametrize("keep", [False, True])
def test_unfused_routes(n, m, R, K, T, keep):
    W = wl.normal_bf16((R, K), 0.02, seed=R + K + T + n + m)
    X = wl.normal_bf16((K, T), 1.0, seed=T + 13)
    idx = wl.permutation(K, 251)
    out = run(W, X, n, m, idx, keep=keep)
    Y = out[0] if keep else out
    ref, mag, ov, om = reference(W, X, n, m, idx)
    assert_gemm_close(values_f64(Y), ref, mag, f"prune_spmm {n}:{m} {R}x{K}x{T}")
    if keep:
        assert np.array_equal(bits(out[1]), ov) and np.array_equal(words(out[2]), om)


def test_edge_cases():
    W = to_dev(wl.normal_bf16((64, 128), 1.0, seed=261))
    X = to_dev(wl.normal_bf16((128, 8), 1.0, seed=262))
    # T = 0: nothing to multiply, the compressed form is still written
    vals = torch.empty((64, 64), dtype=torch.bfloat16, device=DEV)
    meta = torch.empty((nm.nm_meta_words(64, 128, 2, 4),), dtype=torch.int32, device=DEV)
    Y = torch.empty((64, 8), dtype=torch.bfloat16, device=DEV)
    nm.nm_prune_spmm(W, 128, 2, 4, 64, 128, None, X, 8, 0, Y, 8, values=vals, meta=meta)
    torch.cuda.synchronize()
    ov, om = oracle.compress(bits(W), 2, 4)
    assert np.array_equal(bits(vals), ov) and np.array_equal(words(meta), om)
    # K = 0: Y is zero
    Y.fill_(1.0)
    nm.nm_prune_spmm(W, 128, 2, 4, 64, 0, None, X, 8, 8, Y, 8)
    torch.cuda.synchronize()
    assert torch.count_nonzero(Y).item() == 0
    # only one of values / meta
    with pytest.raises(nm.NmError):
        nm.nm_prune_spmm(W, 128, 2, 4, 64, 128, None, X, 8, 8, Y, 8, values=vals)


# ----------------------------------------------------------------------------
# CUDA graphs: the calls (staging allocations and gather passes included)
# capture and replay
# ----------------------------------------------------------------------------
def test_graph_capture_replays_permuted_calls():
    R, K, T = 512, 1024, 256
    W = wl.normal_bf16((R, K), 0.02, seed=271)
    X = wl.normal_bf16((K, T), 1.0, seed=272)
    idx = wl.permutation(K, 273)
    Wd, Xd, idxd = to_dev(W), to_dev(X), to_dev_i32(idx)
    direct, vals, meta = nm.prune_spmm(Wd, 2, 4, Xd, idx=idxd, keep_compressed=True)
    torch.cuda.synchronize()
    Y1 = torch.empty((R, T), dtype=torch.bfloat16, device=DEV)
    Y2 = torch.empty_like(Y1)
    v = torch.empty_like(vals)
    mt = torch.empty_like(meta)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        nm.nm_prune_spmm(Wd, K, 2, 4, R, K, idxd, Xd, T, T, Y1, T, values=v, meta=mt)
        nm.nm_spmm_permuted(vals, meta, 2, 4, R, K, idxd, Xd, T, T, Y2, T)
    for _ in range(2):
        Y1.zero_()
        Y2.zero_()
        g.replay()
        torch.cuda.synchronize()
        nm.nm_device_status()
        assert torch.equal(Y1, direct) and torch.equal(Y2, direct)
        assert torch.equal(v, vals) and torch.equal(mt, meta)
    ref, mag, _, _ = reference(W, X, 2, 4, idx)
    assert_gemm_close(values_f64(Y1), ref, mag, "graph replay")


def test_compress_and_gather_in_one_grid():
    """2:4, two-SM shape, index map: one compress grid that also gathers Xp, then the GEMM (two launches)."""
    R, K, T = 512, 1024, 256
    W = wl.normal_bf16((R, K), 0.02, seed=281)
    X = wl.normal_bf16((K, T), 1.0, seed=282)
    idx = wl.permutation(K, 283).astype(np.int32)
    idx[[4, 9]] = [-1, K]  # zero rows
    Wd, Xd, idxd = to_dev(W), to_dev(X), to_dev_i32(idx)
    vals = torch.empty((R, K // 2), dtype=torch.bfloat16, device=DEV)
    meta = torch.empty((nm.nm_meta_words(R, K, 2, 4),), dtype=torch.int32, device=DEV)
    Y = torch.empty((R, T), dtype=torch.bfloat16, device=DEV)
    torch.cuda.synchronize()
    c0 = nm.nm_launch_count()
    nm.nm_prune_spmm(Wd, K, 2, 4, R, K, idxd, Xd, T, T, Y, T, values=vals, meta=meta)
    assert nm.nm_launch_count() - c0 == 2
    torch.cuda.synchronize()
    nm.nm_device_status()
    ref, mag, ov, om = reference(W, X, 2, 4, idx)
    assert_gemm_close(values_f64(Y), ref, mag, "compress + gather grid")
    assert np.array_equal(bits(vals), ov) and np.array_equal(words(meta), om)
