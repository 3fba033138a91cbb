"""GPU sparse GEMMs (plain, permuted, hybrid, 1:4 / 1:8) against the oracle.

Sizes the oracle finishes in seconds span several 128-row tiles, several
column tiles and ragged tails in R, K and T; the full workload sizes are
checked on sampled outputs computed one by one by the oracle.
"""
import numpy as np
import pytest
import torch

import oracle
import sparse_gemm_nm_b200 as nm
import workloads as wl
from gpu_helpers import (DEV, assert_gemm_close, bf16_rne_of, bits, to_dev, to_dev_i32, to_dev_u8,
                         values_f64)

pytestmark = pytest.mark.gpu


def run_spmm(W, X, n, m, idx=None, out_dtype=torch.bfloat16, algo=nm.NM_ALGO_AUTO):
    K = W.shape[1]
    vals, meta = nm.prune_compress(to_dev(W), n, m)
    Y = nm.spmm(vals, meta, n, m, K, to_dev(X), idx=None if idx is None else to_dev_i32(idx),
                out_dtype=out_dtype, algo=algo)
    torch.cuda.synchronize()
    nm.nm_device_status()
    return Y


def reference(W, X, n, m, idx=None):
    ov, om = oracle.compress(W, n, m)
    Wd = oracle.decompress(ov, om, W.shape[1], n, m)
    return oracle.dense_gemm(Wd, X, idx, with_abs=True)


def check(W, X, n, m, idx=None, algo=nm.NM_ALGO_AUTO, out_dtype=torch.bfloat16, what=""):
    Y = run_spmm(W, X, n, m, idx, out_dtype, algo)
    ref, mag = reference(W, X, n, m, idx)
    assert_gemm_close(values_f64(Y), ref, mag, what)
    return Y


# ----------------------------------------------------------------------------
def test_tiny_2of4():
    L = wl.workload("tiny")[0]
    d = wl.make_layer(L)
    Y = check(d.W, d.X, 2, 4, what="tiny")
    Yi = run_spmm(d.W, d.X, 2, 4, idx=np.arange(L.K, dtype=np.int32))
    assert torch.equal(Y, Yi)  # identity permutation reduces to the plain kernel


@pytest.mark.parametrize("name", ["rl_mlp_2of4", "rl_mlp_1of4", "rl_mlp_1of8"])
@pytest.mark.parametrize("algo", [nm.NM_ALGO_AUTO, nm.NM_ALGO_DENSE_TC])
def test_rl_mlp(name, algo):
    for L in wl.workload(name):
        d = wl.make_layer(L)
        check(d.W, d.X, L.n, L.m, algo=algo, what=L.name)


@pytest.mark.parametrize("n,m", [(2, 4), (1, 4), (1, 8), (1, 2), (2, 8), (3, 4), (3, 8)])
@pytest.mark.parametrize("R,K,T", [(300, 1040, 264), (129, 512, 40), (7, 64, 8)])
def test_ragged_multi_tile(n, m, R, K, T):
    if K % m:
        pytest.skip("K must be a multiple of M")
    W = wl.normal_bf16((R, K), 0.02, seed=R + K)
    X = wl.normal_bf16((K, T), 1.0, seed=T)
    check(W, X, n, m, what=f"{n}:{m} {R}x{K}x{T}")


@pytest.mark.parametrize("n,m", [(1, 4), (1, 8), (2, 4)])
def test_sparse_and_dense_designs_agree(n, m):
    R, K, T = 256, 1024, 128
    W = wl.normal_bf16((R, K), 0.02, seed=3)
    X = wl.normal_bf16((K, T), 1.0, seed=4)
    a = check(W, X, n, m, algo=nm.NM_ALGO_SPARSE_TC, what="sparse")
    b = check(W, X, n, m, algo=nm.NM_ALGO_DENSE_TC, what="dense")
    assert values_f64(a).shape == values_f64(b).shape


@pytest.mark.parametrize("n,m", [(2, 4), (1, 8)])
@pytest.mark.parametrize("algo", [nm.NM_ALGO_AUTO, nm.NM_ALGO_DENSE_TC])
def test_integer_inputs_exact(n, m, algo):
    """Integer weights and inputs: the fp32 accumulation is exact, so the results match bit for bit."""
    R, K, T = 200, 512, 96
    W = wl.integer_bf16((R, K), -8, 8, seed=11)
    X = wl.integer_bf16((K, T), -8, 8, seed=12)
    ref, _ = reference(W, X, n, m)
    Y32 = run_spmm(W, X, n, m, out_dtype=torch.float32, algo=algo)
    assert np.array_equal(Y32.cpu().numpy().astype(np.float64), ref)
    Y16 = run_spmm(W, X, n, m, algo=algo)
    assert np.array_equal(bits(Y16), bf16_rne_of(ref))


def test_fp32_output():
    W = wl.normal_bf16((160, 384), 0.02, seed=21)
    X = wl.normal_bf16((384, 200), 1.0, seed=22)
    check(W, X, 2, 4, out_dtype=torch.float32, what="fp32 out")


def test_unaligned_k_2of4_uses_built_tiles():
    """K = 24 (a 17-wide layer padded to a multiple of 8): values rows are not 16-byte aligned."""
    W = wl.normal_bf16((256, 24), 0.2, seed=31)
    X = wl.normal_bf16((24, 256), 1.0, seed=32)
    check(W, X, 2, 4, what="K=24")


def test_ragged_columns_with_padded_ld():
    R, K, T, ldx = 140, 256, 20, 24
    W = wl.normal_bf16((R, K), 0.02, seed=41)
    X = wl.normal_bf16((K, T), 1.0, seed=42)
    Xp = np.zeros((K, ldx), np.uint16)
    Xp[:, :T] = X
    vals, meta = nm.prune_compress(to_dev(W), 2, 4)
    Y = torch.full((R, 24), 7.0, dtype=torch.bfloat16, device=DEV)
    nm.nm_spmm(vals, meta, 2, 4, R, K, to_dev(Xp), ldx, T, Y, 24)
    torch.cuda.synchronize()
    ref, mag = reference(W, X, 2, 4)
    assert_gemm_close(values_f64(Y[:, :T]), ref, mag, "ragged T")
    assert torch.all(Y[:, T:] == 7.0)  # columns past T untouched


def test_k_zero_gives_zeros():
    Y = torch.full((8, 16), 3.0, dtype=torch.bfloat16, device=DEV)
    vals = torch.empty((8, 0), dtype=torch.bfloat16, device=DEV)
    meta = torch.empty((8, 0), dtype=torch.int32, device=DEV)
    X = torch.empty((0, 16), dtype=torch.bfloat16, device=DEV)
    nm.nm_spmm(vals, meta, 2, 4, 8, 0, X, 16, 16, Y, 16)
    torch.cuda.synchronize()
    assert torch.all(Y == 0)


def test_misaligned_arguments_are_refused():
    vals, meta = nm.prune_compress(torch.zeros((8, 64), dtype=torch.bfloat16, device=DEV), 2, 4)
    X = torch.zeros((64, 24), dtype=torch.bfloat16, device=DEV)
    Y = torch.zeros((8, 24), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(nm.NmError) as e:
        nm.nm_spmm(vals, meta, 2, 4, 8, 64, X, 20, 20, Y, 24)   # ldx % 8 != 0
    assert e.value.status == nm.NM_ERR_MISALIGNED


# ----------------------------------------------------------------------------
# Permuted input read
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("n,m", [(2, 4), (1, 8)])
def test_permuted_matches_oracle(n, m):
    R, K, T = 270, 1024, 296
    W = wl.normal_bf16((R, K), 0.02, seed=51)
    X = wl.normal_bf16((K, T), 1.0, seed=52)
    idx = wl.permutation(K, 53)
    check(W, X, n, m, idx=idx, what="permuted")


@pytest.mark.parametrize("K", [768, 2048])  # SM-pair kernel: 256 x 224 tiles (6 stages), 256 x 256 tiles (16)
def test_permuted_identity_equals_plain_and_host_permuted(K):
    R, T = 256, 256
    W = wl.normal_bf16((R, K), 0.02, seed=61)
    X = wl.normal_bf16((K, T), 1.0, seed=62)
    plain = run_spmm(W, X, 2, 4)
    ident = run_spmm(W, X, 2, 4, idx=np.arange(K, dtype=np.int32))
    assert torch.equal(plain, ident)
    idx = wl.permutation(K, 63)
    perm = run_spmm(W, X, 2, 4, idx=idx)
    host = run_spmm(W, np.ascontiguousarray(X[idx]), 2, 4)
    assert torch.equal(perm, host)  # same tiles, same MMA order: bitwise equal


@pytest.mark.parametrize("K,T", [(512, 256),    # gather pass + SM-pair kernel, 256 x 224 tiles
                                 (1280, 264),   # the same with 256 x 256 tiles and a ragged column tile
                                 (512, 16),     # gather pass + split-K skinny kernel
                                 (512, 100)])   # one-SM kernel gathering its own rows
def test_permuted_out_of_range_entries_read_zero_rows(K, T):
    R = 300
    W = wl.normal_bf16((R, K), 0.02, seed=74)
    X = wl.normal_bf16((K, T), 1.0, seed=75)
    idx = wl.permutation(K, 76).astype(np.int32)
    idx[[0, 5, 130, 257, K - 1]] = [-1, K, K + 1000, -(2 ** 31), 2 ** 31 - 1]
    ld = (T + 7) // 8 * 8
    Xbuf = np.zeros((K, ld), np.uint16)
    Xbuf[:, :T] = X
    vals, meta = nm.prune_compress(to_dev(W), 2, 4)
    Y = torch.empty((R, ld), dtype=torch.bfloat16, device=DEV)
    nm.nm_spmm_permuted(vals, meta, 2, 4, R, K, to_dev_i32(idx), to_dev(Xbuf), ld, T, Y, ld)
    torch.cuda.synchronize()
    nm.nm_device_status()
    Xp = np.zeros((K, T), np.uint16)  # the permuted input by its definition, zero rows for the bad entries
    ok = (idx >= 0) & (idx < K)
    Xp[ok] = X[idx[ok]]
    ref, mag = reference(W, Xp, 2, 4)
    assert_gemm_close(values_f64(Y[:, :T]), ref, mag, f"out-of-range idx, T={T}")


def test_permuted_ragged_k():
    R, K, T = 130, 1040, 64
    W = wl.normal_bf16((R, K), 0.02, seed=71)
    X = wl.normal_bf16((K, T), 1.0, seed=72)
    check(W, X, 2, 4, idx=wl.permutation(K, 73), what="permuted ragged K")


# ----------------------------------------------------------------------------
# PATCH hybrid
# ----------------------------------------------------------------------------
def run_hybrid(W, X, tmap):
    Wd = to_dev(W)
    vals, meta = nm.prune_compress(Wd, 2, 4)
    Y = nm.hybrid_spmm(Wd, vals, meta, to_dev_u8(tmap), to_dev(X))
    torch.cuda.synchronize()
    nm.nm_device_status()
    return Y


@pytest.mark.parametrize("p", [0.0, 0.25, 0.5, 1.0])
def test_hybrid_matches_oracle(p):
    R, K, T = 384, 640, 256
    W = wl.normal_bf16((R, K), 0.02, seed=81)
    X = wl.normal_bf16((K, T), 1.0, seed=82)
    tm = wl.tile_map(3, 5, p, seed=83)
    Y = run_hybrid(W, X, tm)
    ref, mag = oracle.hybrid_spmm(W, tm, X, 128, with_abs=True)
    assert_gemm_close(values_f64(Y), ref, mag, f"hybrid p={p}")


def test_hybrid_all_sparse_equals_spmm():
    R, K, T = 256, 512, 256
    W = wl.normal_bf16((R, K), 0.02, seed=91)
    X = wl.normal_bf16((K, T), 1.0, seed=92)
    Y = run_hybrid(W, X, np.ones((2, 4), np.uint8))
    assert torch.equal(Y, run_spmm(W, X, 2, 4))


def test_hybrid_integer_exact():
    R, K, T = 256, 512, 128
    W = wl.integer_bf16((R, K), -8, 8, seed=93)
    X = wl.integer_bf16((K, T), -8, 8, seed=94)
    tm = wl.tile_map(2, 4, 0.5, seed=95)
    Y = run_hybrid(W, X, tm)
    ref = oracle.hybrid_spmm(W, tm, X, 128)
    assert np.array_equal(bits(Y), bf16_rne_of(ref))


# ----------------------------------------------------------------------------
# Full workload sizes, sampled outputs
# ----------------------------------------------------------------------------
def sampled_check(vals, meta, n, m, W, X, Y, idx=None, count=3000, seed=0):
    """Compare sampled outputs of Y with the oracle's product of ITS OWN compressed
    form of W (oracle.compress), after asserting that the device's compressed
    operand (vals, meta) equals that form bit for bit."""
    R, T = Y.shape
    K = X.shape[0]
    ov, om = oracle.compress(W, n, m)
    assert np.array_equal(bits(vals), ov), "compressed values differ from the oracle's"
    assert np.array_equal(meta.cpu().numpy().view(np.uint32), om), "metadata differs from the oracle's"
    rng = np.random.default_rng(seed)
    rows = np.concatenate([rng.integers(0, R, count), [0, R - 1, 0, R - 1]])
    cols = np.concatenate([rng.integers(0, T, count), [0, T - 1, T - 1, 0]])
    ref, mag = oracle.spmm_sampled(ov, om, n, m, K, X, rows, cols, idx)
    got = values_f64(Y)[rows, cols]
    assert_gemm_close(got, ref, mag, "sampled")


@pytest.mark.parametrize("li", [0, 1, 2])
def test_llama_full_size_sampled(li):
    L = wl.workload("llama7b")[li]  # layer seeds 0, 10, 20
    d = wl.make_layer(L)
    Wd, Xd, idxd = to_dev(d.W), to_dev(d.X), to_dev_i32(d.idx)
    vals, meta = nm.prune_compress(Wd, 2, 4)
    Y = nm.spmm(vals, meta, 2, 4, L.K, Xd, idx=idxd)
    torch.cuda.synchronize()
    nm.nm_device_status()
    sampled_check(vals, meta, 2, 4, d.W, d.X, Y, idx=d.idx)
    # identity map at full size reduces to the plain kernel, bit for bit
    Yp = nm.spmm(vals, meta, 2, 4, L.K, Xd[idxd.long()].contiguous())
    assert torch.equal(Y, Yp)


def test_decode_full_size_sampled():
    L = wl.workload("decode")[0]
    d = wl.make_layer(L)
    vals, meta = nm.prune_compress(to_dev(d.W), 2, 4)
    Y = nm.spmm(vals, meta, 2, 4, L.K, to_dev(d.X))
    torch.cuda.synchronize()
    sampled_check(vals, meta, 2, 4, d.W, d.X, Y, count=20000)


@pytest.mark.parametrize("li", [0, 1])
def test_vit_full_size_sampled(li):
    L = wl.workload("vit")[li]  # layer seeds 0, 10
    d = wl.make_layer(L)
    vals, meta = nm.prune_compress(to_dev(d.W), 1, 8)
    Y = nm.spmm(vals, meta, 1, 8, L.K, to_dev(d.X))
    torch.cuda.synchronize()
    nm.nm_device_status()
    sampled_check(vals, meta, 1, 8, d.W, d.X, Y)


def test_patch_full_size_sampled():
    L = wl.workload("patch_p50")[0]
    d = wl.make_layer(L)
    Wd = to_dev(d.W)
    vals, meta = nm.prune_compress(Wd, 2, 4)
    Y = nm.hybrid_spmm(Wd, vals, meta, to_dev_u8(d.tmap), to_dev(d.X))
    torch.cuda.synchronize()
    nm.nm_device_status()
    rng = np.random.default_rng(1)
    rows, cols = rng.integers(0, L.R, 64), rng.integers(0, L.T, 64)
    Weff = oracle.hybrid_weights(d.W, d.tmap, 128)
    ref, mag = oracle.dense_gemm(np.ascontiguousarray(Weff[rows]), np.ascontiguousarray(d.X[:, cols]),
                                 with_abs=True)
    i = np.arange(rows.shape[0])
    assert_gemm_close(values_f64(Y)[rows, cols], ref[i, i], mag[i, i], "patch sampled")


# ----------------------------------------------------------------------------
# Shapes served by the two-SM (256 x 256 tile) kernel: 2:4, K % 128 == 0, T >= 192
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("R,K,T", [(600, 1024, 520), (256, 4096, 256), (1000, 384, 200), (130, 256, 1000)])
def test_pair_kernel_ragged(R, K, T):
    W = wl.normal_bf16((R, K), 0.02, seed=R * 3 + K)
    X = wl.normal_bf16((K, T), 1.0, seed=T * 5)
    check(W, X, 2, 4, what=f"pair {R}x{K}x{T}")


@pytest.mark.parametrize("out", [torch.bfloat16, torch.float32])
def test_pair_kernel_integer_exact(out):
    R, K, T = 512, 512, 384
    W = wl.integer_bf16((R, K), -8, 8, seed=111)
    X = wl.integer_bf16((K, T), -8, 8, seed=112)
    ref, _ = reference(W, X, 2, 4)
    Y = run_spmm(W, X, 2, 4, out_dtype=out)
    if out == torch.float32:
        assert np.array_equal(Y.cpu().numpy().astype(np.float64), ref)
    else:
        assert np.array_equal(bits(Y), bf16_rne_of(ref))


@pytest.mark.parametrize("n,m", [(2, 4), (1, 8)])
def test_permuted_pair_path_after_release_staging(n, m):
    """The two-SM permuted path stages Xp (and for 1:8 a re-encoded 2:4
    operand) in a library pool; handing the pool's memory back between calls
    must not change the result."""
    R, K, T = 512, 1024, 512
    W = wl.normal_bf16((R, K), 0.02, seed=121)
    X = wl.normal_bf16((K, T), 1.0, seed=122)
    idx = wl.permutation(K, 123)
    first = run_spmm(W, X, n, m, idx=idx)
    nm.nm_release_staging()
    second = run_spmm(W, X, n, m, idx=idx)
    nm.nm_release_staging()
    assert torch.equal(first, second)
    ref, mag = reference(W, X, n, m, idx)
    assert_gemm_close(values_f64(second), ref, mag, "permuted after release")


# ----------------------------------------------------------------------------
# 1:2 / 1:4 / 1:8 / 2:8 on two-SM shapes: re-encoded as 2:4, then the pair kernel
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("n,m", [(1, 2), (1, 4), (1, 8), (2, 8)])
@pytest.mark.parametrize("permuted", [False, True])
def test_reencoded_pair_path(n, m, permuted):
    R, K, T = 600, 1024, 264
    W = wl.normal_bf16((R, K), 0.02, seed=131 + m + n)
    X = wl.normal_bf16((K, T), 1.0, seed=132)
    idx = wl.permutation(K, 133) if permuted else None
    before = nm.nm_launch_count()
    check(W, X, n, m, idx=idx, what=f"re-encoded {n}:{m}")
    # prune_compress, re-encode, [gather,] pair GEMM
    assert nm.nm_launch_count() - before == (4 if permuted else 3)



def test_reencoded_pair_path_integer_exact():
    R, K, T = 512, 1024, 256
    W = wl.integer_bf16((R, K), -8, 8, seed=141)
    X = wl.integer_bf16((K, T), -8, 8, seed=142)
    ref, _ = reference(W, X, 1, 8)
    Y = run_spmm(W, X, 1, 8, out_dtype=torch.float32)
    assert np.array_equal(Y.cpu().numpy().astype(np.float64), ref)


# ----------------------------------------------------------------------------
# Few columns (T <= 64, K % 128 == 0): the split-K skinny kernel
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("R,K,T", [(200, 1024, 16), (128, 512, 8), (333, 2048, 40), (1000, 256, 64),
                                   (64, 128, 8), (13824 // 8, 5120, 24)])
def test_skinny_kernel(R, K, T):
    W = wl.normal_bf16((R, K), 0.02, seed=R + K + T)
    X = wl.normal_bf16((K, T), 1.0, seed=T + 7)
    check(W, X, 2, 4, what=f"skinny {R}x{K}x{T}")


@pytest.mark.parametrize("n,m", [(2, 4), (1, 8)])
def test_skinny_kernel_permuted(n, m):
    R, K, T = 300, 1024, 16
    W = wl.normal_bf16((R, K), 0.02, seed=151)
    X = wl.normal_bf16((K, T), 1.0, seed=152)
    check(W, X, n, m, idx=wl.permutation(K, 153), what=f"skinny permuted {n}:{m}")


@pytest.mark.parametrize("T", [1, 13, 33])
def test_skinny_kernel_permuted_ragged_columns(T):
    """T % 8 != 0: X rows padded to 16 bytes; the gathered copy must carry the partial last piece."""
    R, K = 200, 512
    W = wl.normal_bf16((R, K), 0.02, seed=155 + T)
    X = wl.normal_bf16((K, T), 1.0, seed=156)
    idx = wl.permutation(K, 157)
    ld = (T + 7) // 8 * 8
    Xbuf = np.zeros((K, ld), np.uint16)
    Xbuf[:, :T] = X
    vals, meta = nm.prune_compress(to_dev(W), 2, 4)
    Y = torch.empty((R, ld), dtype=torch.bfloat16, device=DEV)
    nm.nm_spmm_permuted(vals, meta, 2, 4, R, K, to_dev_i32(idx), to_dev(Xbuf), ld, T, Y, ld)
    torch.cuda.synchronize()
    nm.nm_device_status()
    ref, mag = reference(W, X, 2, 4, idx)
    assert_gemm_close(values_f64(Y[:, :T]), ref, mag, f"skinny permuted T={T}")


@pytest.mark.parametrize("out", [torch.bfloat16, torch.float32])
def test_skinny_kernel_integer_exact(out):
    R, K, T = 384, 4096, 16  # several K ranges: partial sums are exact integers
    W = wl.integer_bf16((R, K), -8, 8, seed=161)
    X = wl.integer_bf16((K, T), -8, 8, seed=162)
    ref, _ = reference(W, X, 2, 4)
    Y = run_spmm(W, X, 2, 4, out_dtype=out)
    if out == torch.float32:
        assert np.array_equal(Y.cpu().numpy().astype(np.float64), ref)
    else:
        assert np.array_equal(bits(Y), bf16_rne_of(ref))


# ----------------------------------------------------------------------------
# PATCH hybrid on SM pairs (K % 128 == 0, T >= 192): mixed stages run dense
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("p", [0.25, 0.75])
def test_hybrid_pair_ragged(p):
    R, K, T = 300, 384, 264
    W = wl.normal_bf16((R, K), 0.02, seed=171)
    X = wl.normal_bf16((K, T), 1.0, seed=172)
    tm = wl.tile_map(3, 3, p, seed=173)
    Y = run_hybrid(W, X, tm)
    ref, mag = oracle.hybrid_spmm(W, tm, X, 128, with_abs=True)
    assert_gemm_close(values_f64(Y), ref, mag, f"hybrid pair p={p}")


def test_hybrid_pair_integer_exact():
    R, K, T = 512, 512, 256
    W = wl.integer_bf16((R, K), -8, 8, seed=181)
    X = wl.integer_bf16((K, T), -8, 8, seed=182)
    tm = wl.tile_map(4, 4, 0.5, seed=183)
    Y = run_hybrid(W, X, tm)
    ref = oracle.hybrid_spmm(W, tm, X, 128)
    assert np.array_equal(bits(Y), bf16_rne_of(ref))


# ----------------------------------------------------------------------------
# Failure path: a bounded wait that runs out is reported, the context stays usable
# ----------------------------------------------------------------------------
def test_bounded_wait_timeout_is_reported():
    nm.nm_device_status()  # start from a clear status word
    nm.nm_selftest_wait_timeout(20000)  # 20 ms on a barrier that nothing completes
    with pytest.raises(nm.NmError) as e:
        nm.nm_device_status()
    assert e.value.status == nm.NM_ERR_TIMEOUT
    nm.nm_device_status()  # the word was cleared by the read
    # the context still runs kernels correctly
    R, K, T = 256, 512, 256
    W = wl.normal_bf16((R, K), 0.02, seed=191)
    X = wl.normal_bf16((K, T), 1.0, seed=192)
    check(W, X, 2, 4, what="after a reported timeout")


# ----------------------------------------------------------------------------
# Dense design on SM pairs: decompress into a staged dense operand, dense stages
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("n,m,algo", [(2, 4, nm.NM_ALGO_DENSE_TC), (1, 8, nm.NM_ALGO_DENSE_TC),
                                      (3, 4, nm.NM_ALGO_AUTO), (5, 8, nm.NM_ALGO_AUTO)])
@pytest.mark.parametrize("permuted", [False, True])
def test_dense_design_pair_path(n, m, algo, permuted):
    R, K, T = 600, 1024, 264
    W = wl.normal_bf16((R, K), 0.02, seed=201 + m)
    X = wl.normal_bf16((K, T), 1.0, seed=202)
    idx = wl.permutation(K, 203) if permuted else None
    check(W, X, n, m, idx=idx, algo=algo, what=f"dense design {n}:{m}")


def test_dense_design_pair_integer_exact():
    R, K, T = 512, 1024, 256
    W = wl.integer_bf16((R, K), -8, 8, seed=211)
    X = wl.integer_bf16((K, T), -8, 8, seed=212)
    ref, _ = reference(W, X, 3, 4)
    Y = run_spmm(W, X, 3, 4, out_dtype=torch.float32)
    assert np.array_equal(Y.cpu().numpy().astype(np.float64), ref)


# ----------------------------------------------------------------------------
# SM-pair kernel tile forms: 256 x 256 tiles with one accumulator (more than 8
# stages per tile) and 256 x 224 tiles with two accumulators (at most 8)
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("R,K,T", [(2560, 8192, 2048),   # 64 stages: 256 x 256 tiles
                                   (4096, 11008, 2048),  # the LLaMA 4096 x 11008 layer
                                   (1280, 512, 4096),    # 4 stages: 256 x 224 tiles, 19 column tiles, the last one 64 wide
                                   (2304, 768, 2560),    # 6 stages (the ViT depth), last column tile partial
                                   (300, 1024, 200)])    # 8 stages, one partial 224-column tile, ragged rows
@pytest.mark.parametrize("out", [torch.bfloat16, torch.float32])
def test_pair_tile_forms_integer_exact(R, K, T, out):
    """Small integers keep every fp32 sum exact: sampled rows equal the oracle bit for bit."""
    W = wl.integer_bf16((R, K), -8, 8, seed=R + 7)
    X = wl.integer_bf16((K, T), -8, 8, seed=T + 9)
    Y = run_spmm(W, X, 2, 4, out_dtype=out)
    ov, om = oracle.compress(W, 2, 4)
    rng = np.random.default_rng(3)
    rows = np.unique(np.concatenate([rng.integers(0, R, 96), [0, 127, 128, 255, R - 1]]))
    rows = rows[rows < R]
    Wd = oracle.decompress(ov, om, K, 2, 4)
    ref = oracle.dense_gemm(np.ascontiguousarray(Wd[rows]), X)
    if out == torch.float32:
        assert np.array_equal(Y.contiguous().cpu().numpy().astype(np.float64)[rows], ref)
    else:
        assert np.array_equal(bits(Y)[rows], bf16_rne_of(ref))


@pytest.mark.parametrize("R,K,T", [(2560, 8192, 2048),   # 256 x 256 tiles, row tiles fastest
                                   (4096, 11008, 2048),  # 256 x 256 tiles, column tiles fastest
                                   (1280, 512, 4096),    # 256 x 224 tiles
                                   (2304, 768, 2568),    # 256 x 224 tiles, last column tile partial
                                   (300, 1024, 200)])    # one partial 224-column tile, ragged rows
@pytest.mark.parametrize("out", [torch.bfloat16, torch.float32])
def test_pair_permuted_integer_exact(R, K, T, out):
    """The permuted two-SM path (gather pass, then the pair kernel) on small
    integers (every fp32 sum exact): sampled rows equal the oracle's permuted
    product bit for bit."""
    W = wl.integer_bf16((R, K), -8, 8, seed=R + 17)
    X = wl.integer_bf16((K, T), -8, 8, seed=T + 19)
    idx = wl.permutation(K, K + 23)
    Y = run_spmm(W, X, 2, 4, idx=idx, out_dtype=out)
    ov, om = oracle.compress(W, 2, 4)
    rng = np.random.default_rng(5)
    rows = np.unique(np.concatenate([rng.integers(0, R, 96), [0, 127, 128, 255, R - 1]]))
    rows = rows[rows < R]
    Wd = oracle.decompress(ov, om, K, 2, 4)
    ref = oracle.dense_gemm(np.ascontiguousarray(Wd[rows]), X, idx)
    if out == torch.float32:
        assert np.array_equal(Y.contiguous().cpu().numpy().astype(np.float64)[rows], ref)
    else:
        assert np.array_equal(bits(Y)[rows], bf16_rne_of(ref))


@pytest.mark.parametrize("R,K,T", [(1, 128, 192),      # one row, one stage, one partial 224-column tile
                                   (257, 128, 192),    # a 1-row second row tile
                                   (255, 1024, 200),   # 8 stages (the last of the 256 x 224 form), 8 columns in the last 32-column chunk
                                   (255, 1152, 200),   # 9 stages: the 256 x 256 form, one partial column tile
                                   (513, 1152, 392),   # three row tiles, ragged rows and columns
                                   (256, 1024, 184)])  # T < 192: the one-SM kernel
@pytest.mark.parametrize("out", [torch.bfloat16, torch.float32])
def test_pair_admission_boundaries_integer_exact(R, K, T, out):
    """Shapes at the edges of the SM-pair kernel's rules (T >= 192, the eight-stage limit of the
    two-accumulator form, ragged R): small integers, so the whole output equals the oracle bit for bit."""
    W = wl.integer_bf16((R, K), -8, 8, seed=R + K)
    X = wl.integer_bf16((K, T), -8, 8, seed=T + 1)
    Y = run_spmm(W, X, 2, 4, out_dtype=out)
    ref, _ = reference(W, X, 2, 4)
    if out == torch.float32:
        assert np.array_equal(Y.contiguous().cpu().numpy().astype(np.float64), ref)
    else:
        assert np.array_equal(bits(Y), bf16_rne_of(ref))


def test_pair_double_buffered_permuted_tolerance():
    """ViT-depth tiles (6 stages, two accumulators) with an index map, sampled at full width."""
    R, K, T = 3072, 768, 6144
    W = wl.normal_bf16((R, K), 0.02, seed=41)
    X = wl.normal_bf16((K, T), 1.0, seed=42)
    idx = wl.permutation(K, 43)
    vals, meta = nm.prune_compress(to_dev(W), 2, 4)
    Y = nm.spmm(vals, meta, 2, 4, K, to_dev(X), idx=to_dev_i32(idx))
    torch.cuda.synchronize()
    nm.nm_device_status()
    sampled_check(vals, meta, 2, 4, W, X, Y, idx=idx, count=4000)


def test_pair_repeatable():
    """Two runs of the same GEMM agree bit for bit (both tile forms)."""
    for R, K, T in ((2560, 8192, 2048), (1280, 768, 4096)):
        W = wl.normal_bf16((R, K), 0.02, seed=61)
        X = wl.normal_bf16((K, T), 1.0, seed=62)
        a = run_spmm(W, X, 2, 4)
        b = run_spmm(W, X, 2, 4)
        assert torch.equal(a, b)
