"""GPU backward products of y = (W' Pi) x against the oracle.

nm_spmm_t (input gradient, dX = (W' Pi)^T dY) and nm_sddmm (gradient of the
stored values, the survivor entries of dY Xp^T) run as dense tcgen05 GEMMs on
SM pairs.  Sizes span several 256 x 256 tiles with ragged edges in every
dimension; integer inputs give exact results; the LLaMA-size layer is checked
on sampled columns / rows computed by the oracle.
"""
import numpy as np
import pytest
import torch

import oracle
import sparse_gemm_nm_b200 as nm
import workloads as wl
from gpu_helpers import DEV, assert_gemm_close, bf16_rne_of, bits, to_dev, to_dev_i32, values_f64, words

pytestmark = pytest.mark.gpu


def padded(A):
    """rows x cols on the device with rows padded to 16 bytes (a view of a wider buffer)."""
    r, c = A.shape
    buf = np.zeros((r, (c + 7) // 8 * 8), np.uint16)
    buf[:, :c] = A
    return to_dev(buf)[:, :c]


def compressed(W, n, m):
    vals, meta = oracle.compress(W, n, m)
    return vals, meta, to_dev(vals), torch.from_numpy(meta.view(np.int32)).to(DEV)


@pytest.mark.parametrize("R,K,T", [(300, 512, 264), (256, 1024, 256), (130, 384, 100), (64, 128, 8),
                                   (520, 264, 40)])
@pytest.mark.parametrize("n,m", [(2, 4), (1, 8), (3, 4)])
@pytest.mark.parametrize("permuted", [False, True])
def test_input_gradient_matches_oracle(R, K, T, n, m, permuted):
    if K % m:
        pytest.skip("K must be a multiple of M")
    W = wl.normal_bf16((R, K), 0.02, seed=R + K + T + m)
    dY = wl.normal_bf16((R, T), 1.0, seed=T + 5)
    idx = wl.permutation(K, R + 7) if permuted else None
    vals, meta, vd, md = compressed(W, n, m)
    dX = nm.spmm_t(vd, md, n, m, K, padded(dY), idx=None if idx is None else to_dev_i32(idx))
    torch.cuda.synchronize()
    nm.nm_device_status()
    ref, mag = oracle.spmm_t(vals, meta, n, m, K, dY, idx, with_abs=True)
    assert_gemm_close(values_f64(dX), ref, mag, f"dX {n}:{m} {R}x{K}x{T} permuted={permuted}")


@pytest.mark.parametrize("R,K,T", [(300, 512, 264), (256, 1024, 256), (130, 384, 100), (64, 128, 8),
                                   (520, 264, 40)])
@pytest.mark.parametrize("n,m", [(2, 4), (1, 8), (3, 4)])
@pytest.mark.parametrize("permuted", [False, True])
def test_value_gradient_matches_oracle(R, K, T, n, m, permuted):
    if K % m:
        pytest.skip("K must be a multiple of M")
    W = wl.normal_bf16((R, K), 0.02, seed=R + K + T + m + 1)
    dY = wl.normal_bf16((R, T), 1.0, seed=T + 6)
    X = wl.normal_bf16((K, T), 1.0, seed=T + 8)
    idx = wl.permutation(K, R + 9) if permuted else None
    vals, meta, vd, md = compressed(W, n, m)
    dV = nm.sddmm(md, n, m, R, K, padded(dY), padded(X), idx=None if idx is None else to_dev_i32(idx))
    torch.cuda.synchronize()
    nm.nm_device_status()
    ref, mag = oracle.sddmm(meta, n, m, R, K, dY, X, idx, with_abs=True)
    assert_gemm_close(values_f64(dV), ref, mag, f"dV {n}:{m} {R}x{K}x{T} permuted={permuted}")


@pytest.mark.parametrize("out", [torch.bfloat16, torch.float32])
def test_backward_integer_exact(out):
    R, K, T = 384, 768, 512  # several reduction stages each way; every partial sum is an exact integer
    W = wl.integer_bf16((R, K), -8, 8, seed=301)
    dY = wl.integer_bf16((R, T), -8, 8, seed=302)
    X = wl.integer_bf16((K, T), -8, 8, seed=303)
    idx = wl.permutation(K, 304)
    vals, meta, vd, md = compressed(W, 2, 4)
    dX = nm.spmm_t(vd, md, 2, 4, K, to_dev(dY), idx=to_dev_i32(idx), out_dtype=out)
    dV = nm.sddmm(md, 2, 4, R, K, to_dev(dY), to_dev(X), idx=to_dev_i32(idx), out_dtype=out)
    torch.cuda.synchronize()
    nm.nm_device_status()
    rX = oracle.spmm_t(vals, meta, 2, 4, K, dY, idx)
    rV = oracle.sddmm(meta, 2, 4, R, K, dY, X, idx)
    if out == torch.float32:
        assert np.array_equal(dX.cpu().numpy().astype(np.float64), rX)
        assert np.array_equal(dV.cpu().numpy().astype(np.float64), rV)
    else:
        assert np.array_equal(bits(dX), bf16_rne_of(rX))
        assert np.array_equal(bits(dV), bf16_rne_of(rV))


def test_input_gradient_drops_out_of_range_rows():
    R, K, T = 256, 512, 64
    W = wl.normal_bf16((R, K), 0.02, seed=311)
    dY = wl.normal_bf16((R, T), 1.0, seed=312)
    idx = wl.permutation(K, 313).astype(np.int32)
    lost = idx[[3, 300]].copy()  # rows no entry names any more
    idx[[3, 300]] = [-5, K]
    vals, meta, vd, md = compressed(W, 2, 4)
    dX = torch.full((K, T), 7.0, dtype=torch.float32, device=DEV)
    nm.nm_spmm_t(vd, md, 2, 4, R, K, to_dev_i32(idx), to_dev(dY), T, T, dX, T, nm.NM_OUT_F32)
    torch.cuda.synchronize()
    nm.nm_device_status()
    ref, mag = oracle.spmm_t(vals, meta, 2, 4, K, dY, idx, with_abs=True)
    got = dX.cpu().numpy().astype(np.float64)
    keep = np.ones(K, bool)
    keep[lost] = False
    assert_gemm_close(got[keep], ref[keep], mag[keep], "dX with dropped rows")
    assert np.all(got[lost] == 7.0)  # not written


def test_degenerate_shapes():
    K, T = 128, 16
    vals = torch.zeros((0, K // 2), dtype=torch.bfloat16, device=DEV)
    meta = torch.zeros((1,), dtype=torch.int32, device=DEV)
    dY = torch.zeros((0, T), dtype=torch.bfloat16, device=DEV)
    dX = torch.full((K, T), 3.0, dtype=torch.bfloat16, device=DEV)
    nm.nm_spmm_t(vals, meta, 2, 4, 0, K, None, dY, T, T, dX, T)  # R = 0: the gradient is zero
    R = 32
    W = wl.normal_bf16((R, K), 1.0, seed=321)
    v, mt, vd, md = compressed(W, 2, 4)
    dV = torch.full((R, K // 2), 3.0, dtype=torch.bfloat16, device=DEV)
    X = torch.zeros((K, 8), dtype=torch.bfloat16, device=DEV)
    dY2 = torch.zeros((R, 8), dtype=torch.bfloat16, device=DEV)
    nm.nm_sddmm(md, 2, 4, R, K, None, dY2, 8, X, 8, 0, dV)  # T = 0: an empty sum
    torch.cuda.synchronize()
    nm.nm_device_status()
    assert torch.count_nonzero(dX).item() == 0 and torch.count_nonzero(dV).item() == 0
    with pytest.raises(nm.NmError):
        nm.nm_spmm_t(vd, md, 2, 4, R, K, None, dY2, 4, 8, dX, T)  # lddy < T


def test_llama_layer_sampled():
    L = wl.workload("llama7b")[0]
    d = wl.make_layer(L)
    R, K, T = L.R, L.K, L.T
    dY = wl.normal_bf16((R, T), 1.0, seed=331)
    vals, meta, vd, md = compressed(d.W, 2, 4)
    dYd, Xd, idxd = to_dev(dY), to_dev(d.X), to_dev_i32(d.idx)
    dX = nm.spmm_t(vd, md, 2, 4, K, dYd, idx=idxd)
    dV = nm.sddmm(md, 2, 4, R, K, dYd, Xd, idx=idxd)
    torch.cuda.synchronize()
    nm.nm_device_status()
    cols = np.array([0, 1, 777, 1500, T - 1])
    ref, mag = oracle.spmm_t(vals, meta, 2, 4, K, np.ascontiguousarray(dY[:, cols]), d.idx, with_abs=True)
    assert_gemm_close(values_f64(dX)[:, cols], ref, mag, "dX sampled columns")
    rows = 48  # the first three 16-row metadata blocks: a prefix of the tiled metadata
    cb = (K + 127) // 128
    refv, magv = oracle.sddmm(meta[: rows // 16 * cb * 64], 2, 4, rows, K, np.ascontiguousarray(dY[:rows]), d.X,
                              d.idx, with_abs=True)
    assert_gemm_close(values_f64(dV)[:rows], refv, magv, "dV first rows")
