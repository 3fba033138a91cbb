"""GPU diagonal sparsity (selection, gather, dense copy, GEMM) against the oracle.

The device adds the diagonal scores in float32 while the oracle's scores are
exact, so where two scores differ by less than float32 rounding the two may
keep different diagonals.  Selection is therefore checked for validity
(``oracle.diag_selection_errors``: no dropped diagonal beats a kept one by
more than the float32 error bound; exact ties and NaNs by the rule), and the
values, the dense copy and the GEMM are compared with the oracle on the
offsets the device chose.  On small-integer data every float32 partial sum is
exact, so there the device must take the oracle's own choice.
"""
import numpy as np
import pytest
import torch

import oracle
import sparse_gemm_nm_b200 as nm
import workloads as wl
from gpu_helpers import DEV, assert_gemm_close, bf16_rne_of, bits, to_dev, to_dev_i32, values_f64

pytestmark = pytest.mark.gpu


def padded(X):
    K, T = X.shape
    buf = np.zeros((K, (T + 7) // 8 * 8), np.uint16)
    buf[:, :T] = X
    return to_dev(buf)[:, :T]


@pytest.mark.parametrize("R,K,D", [(64, 64, 7), (300, 128, 13), (128, 300, 30), (3072, 768, 77), (768, 3072, 307)])
def test_selection_and_values_match_oracle(R, K, D):
    W = wl.normal_bf16((R, K), 0.02, seed=R + K + D)
    offs, V = nm.diag_prune_compress(to_dev(W), D)
    torch.cuda.synchronize()
    oo = offs.cpu().numpy()
    assert oracle.diag_selection_errors(W, D, oo) == []
    assert np.array_equal(bits(V), oracle.diag_compress(W, oo))
    Wd = torch.empty((R, K), dtype=torch.bfloat16, device=DEV)
    nm.nm_diag_expand(V, offs, D, R, K, Wd, K)
    torch.cuda.synchronize()
    assert np.array_equal(bits(Wd), oracle.diag_expand(oracle.diag_compress(W, oo), oo, K))


def test_selection_ties_and_nan():
    W = wl.bf16_bits(np.ones((40, 24), np.float32))  # all diagonals tie
    offs, _ = nm.diag_prune_compress(to_dev(W), 5)
    torch.cuda.synchronize()
    assert np.array_equal(offs.cpu().numpy(), np.arange(5))
    W[3, (3 + 17) % 24] = 0x7FC0
    offs, _ = nm.diag_prune_compress(to_dev(W), 1)
    torch.cuda.synchronize()
    assert offs.cpu().numpy().tolist() == [17]


def test_selection_near_tie_is_valid():
    # two diagonals 2^-20 apart at a score of 63: float32 cannot separate them, the
    # oracle keeps the exactly larger one; either is a valid selection
    R, K = 64, 16
    Wf = np.zeros((R, K), np.float32)
    for r in range(63):
        Wf[r, r % K] = 1.0
        Wf[r, (r + 1) % K] = 1.0
    Wf[63, (63 + 1) % K] = 2.0 ** -20
    W = wl.bf16_bits(Wf)
    offs, V = nm.diag_prune_compress(to_dev(W), 1)
    torch.cuda.synchronize()
    oo = offs.cpu().numpy()
    assert oo.tolist() in ([0], [1])
    assert oracle.diag_selection_errors(W, 1, oo) == []
    assert np.array_equal(bits(V), oracle.diag_compress(W, oo))


@pytest.mark.parametrize("R,K,D,T", [(300, 128, 13, 264), (128, 300, 30, 100), (256, 512, 51, 256), (64, 64, 64, 8)])
@pytest.mark.parametrize("permuted", [False, True])
def test_diag_spmm_matches_oracle(R, K, D, T, permuted):
    W = wl.normal_bf16((R, K), 0.02, seed=R * 3 + K)
    X = wl.normal_bf16((K, T), 1.0, seed=T + 1)
    idx = wl.permutation(K, R + 2) if permuted else None
    offs, V = nm.diag_prune_compress(to_dev(W), D)
    Y = nm.diag_spmm(V, offs, K, padded(X), idx=None if idx is None else to_dev_i32(idx))
    torch.cuda.synchronize()
    nm.nm_device_status()
    oo = offs.cpu().numpy()
    assert oracle.diag_selection_errors(W, D, oo) == []
    ref, mag = oracle.diag_spmm(oracle.diag_compress(W, oo), oo, K, X, idx, with_abs=True)
    assert_gemm_close(values_f64(Y), ref, mag, f"diag {R}x{K} D={D} T={T} permuted={permuted}")


@pytest.mark.parametrize("out", [torch.bfloat16, torch.float32])
def test_diag_spmm_integer_exact(out):
    R, K, D, T = 384, 512, 64, 256
    W = wl.integer_bf16((R, K), -8, 8, seed=401)
    X = wl.integer_bf16((K, T), -8, 8, seed=402)
    offs, V = nm.diag_prune_compress(to_dev(W), D)
    Y = nm.diag_spmm(V, offs, K, to_dev(X), out_dtype=out)
    torch.cuda.synchronize()
    oo = oracle.diag_select(W, D)
    assert np.array_equal(offs.cpu().numpy(), oo)  # float32 sums of small integers are exact
    ref = oracle.diag_spmm(oracle.diag_compress(W, oo), oo, K, X)
    if out == torch.float32:
        assert np.array_equal(Y.contiguous().cpu().numpy().astype(np.float64), ref)
    else:
        assert np.array_equal(bits(Y), bf16_rne_of(ref))


def test_vit_size_sampled():
    R, K, D, T = 3072, 768, 77, 197 * 256  # 90 % sparse ViT-B linear, 197 tokens x 256 images
    W = wl.normal_bf16((R, K), 0.02, seed=411)
    X = wl.normal_bf16((K, T), 1.0, seed=412)
    idx = wl.permutation(K, 413)
    offs, V = nm.diag_prune_compress(to_dev(W), D)
    Y = nm.diag_spmm(V, offs, K, to_dev(X), idx=to_dev_i32(idx))
    torch.cuda.synchronize()
    nm.nm_device_status()
    oo = offs.cpu().numpy()
    assert oracle.diag_selection_errors(W, D, oo) == []
    assert np.array_equal(bits(V), oracle.diag_compress(W, oo))
    cols = np.array([0, 1, 999, 30000, T - 1])
    ref, mag = oracle.diag_spmm(oracle.diag_compress(W, oo), oo, K, np.ascontiguousarray(X[:, cols]), idx,
                                with_abs=True)
    assert_gemm_close(values_f64(Y)[:, cols], ref, mag, "diag ViT sampled")


@pytest.mark.parametrize("kind", ["permutation", "repeats", "out_of_range"])
@pytest.mark.parametrize("out", [torch.bfloat16, torch.float32])
def test_diag_spmm_index_maps_integer_exact(kind, out):
    # A permutation takes the route that places the dense copy's columns through idx (the GEMM reads X
    # itself); any other map takes the gather of X[idx].  Both are exact on small integers.
    R, K, D, T = 320, 384, 40, 264
    W = wl.integer_bf16((R, K), -8, 8, seed=421)
    X = wl.integer_bf16((K, T), -8, 8, seed=422)
    rng = np.random.default_rng(423)
    idx = rng.permutation(K).astype(np.int32)
    if kind == "repeats":
        idx[[5, 77, 200]] = idx[[6, 6, 300]]
    elif kind == "out_of_range":
        idx[[0, 383]] = [-1, K]
    offs, V = nm.diag_prune_compress(to_dev(W), D)
    Y = nm.diag_spmm(V, offs, K, padded(X), idx=to_dev_i32(idx), out_dtype=out)
    torch.cuda.synchronize()
    nm.nm_device_status()
    oo = oracle.diag_select(W, D)
    assert np.array_equal(offs.cpu().numpy(), oo)  # float32 sums of small integers are exact
    ref = oracle.diag_spmm(oracle.diag_compress(W, oo), oo, K, X, idx)
    if out == torch.float32:
        assert np.array_equal(Y.contiguous().cpu().numpy().astype(np.float64), ref)
    else:
        assert np.array_equal(bits(Y), bf16_rne_of(ref))


def test_diag_expand_strides_and_foreign_offsets():
    R, K, D = 70, 45, 6
    W = wl.normal_bf16((R, K), 1.0, seed=431)
    oo = np.array([0, 3, 9, 20, 33, 44], np.int32)
    V = oracle.diag_compress(W, oo)
    ref = oracle.diag_expand(V, oo, K)
    for ldw in (K, K + 3, 56):  # rows that are not 16-byte multiples, and ones that are
        buf = torch.full((R, ldw), 5.0, dtype=torch.bfloat16, device=DEV)
        nm.nm_diag_expand(to_dev(V), to_dev_i32(oo), D, R, K, buf, ldw)
        torch.cuda.synchronize()
        got = bits(buf)
        assert np.array_equal(got[:, :K], ref)
        assert np.all(got[:, K:] == bits(torch.tensor([5.0], dtype=torch.bfloat16))[0])  # padding untouched
    bad = oo.copy()
    bad[2] = K + 7  # an offset outside [0, K) places nothing
    buf = torch.full((R, K), 5.0, dtype=torch.bfloat16, device=DEV)
    nm.nm_diag_expand(to_dev(V), to_dev_i32(bad), D, R, K, buf, K)
    torch.cuda.synchronize()
    keep = np.array([0, 1, 3, 4, 5])
    assert np.array_equal(bits(buf), oracle.diag_expand(V[keep], oo[keep], K))
    nm.nm_diag_expand(to_dev(V), to_dev_i32(oo), 0, R, K, buf, K)  # D = 0: all zero
    torch.cuda.synchronize()
    assert torch.count_nonzero(buf).item() == 0
