"""GPU TF32 path (1:2 float32 weights) against the oracle.

Compress and decompress are compared bit for bit (values, metadata, dense
copy); the GEMM, which reads its operands as TF32 on the tensor cores, is
held to the GEMM tolerance, and to bit equality on small integers (exact in
TF32 and in the fp32 accumulator).  Sizes span several 256 x 256 tiles and
64-deep stages with ragged edges in R, K and T.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import sparse_gemm_nm_b200 as nm
import workloads as wl
from gpu_helpers import DEV, assert_gemm_close, bf16_rne_of, bits

pytestmark = pytest.mark.gpu


def f32_dev(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(DEV)


def u32(t):
    return t.contiguous().cpu().numpy().view(np.uint32)


def padded_x(X):
    K, T = X.shape
    buf = np.zeros((K, (T + 3) // 4 * 4), np.float32)
    buf[:, :T] = X
    return f32_dev(buf)[:, :T]


@pytest.mark.parametrize("R,K", [(300, 512), (64, 66), (1, 2), (130, 1000), (7, 64)])
def test_compress_and_decompress_bit_exact(R, K):
    W = wl.normal_f32((R, K), 1.0, seed=R + K)
    vals, meta = nm.prune_compress_tf32(f32_dev(W))
    torch.cuda.synchronize()
    ov, om = oracle.compress_f32(W)
    assert np.array_equal(u32(vals), ov)
    assert np.array_equal(u32(meta), om)
    back = nm.decompress_tf32(vals, meta, K)
    torch.cuda.synchronize()
    assert np.array_equal(u32(back), oracle.decompress_f32(ov, om, K))


def test_compress_special_values():
    alphabet = [-2.0, -1.0, -0.0, 0.0, 1.0, 2.0, math.inf, -math.inf, math.nan]
    row = [x for a in alphabet for b in alphabet for x in (a, b)]
    W = np.array([row, row[::-1]], np.float32)
    W.view(np.uint32)[0, 1] = 0xFFC00001  # a negative NaN with a payload
    vals, meta = nm.prune_compress_tf32(f32_dev(W))
    torch.cuda.synchronize()
    ov, om = oracle.compress_f32(W)
    assert np.array_equal(u32(vals), ov)
    assert np.array_equal(u32(meta), om)


def test_compress_strided_rows():
    R, K, ldw = 40, 96, 100
    buf = wl.normal_f32((R, ldw), 1.0, seed=7)
    vals, meta = nm.prune_compress_tf32(f32_dev(buf)[:, :K])
    torch.cuda.synchronize()
    ov, om = oracle.compress_f32(np.ascontiguousarray(buf[:, :K]))
    assert np.array_equal(u32(vals), ov) and np.array_equal(u32(meta), om)


# T >= 192 with K % 8 == 0 runs on the sparse tensor cores (kind::tf32, metadata re-laid out); other shapes
# on the decompressed dense operand.
@pytest.mark.parametrize("R,K,T", [(300, 512, 264), (256, 1024, 256), (130, 386, 100), (64, 130, 8),
                                   (520, 264, 40), (260, 600, 320), (200, 514, 256)])
@pytest.mark.parametrize("out", [torch.float32, torch.bfloat16])
def test_spmm_matches_oracle(R, K, T, out):
    W = wl.normal_f32((R, K), 0.05, seed=R * 3 + K)
    X = wl.normal_f32((K, T), 1.0, seed=T + 1)
    vals, meta = nm.prune_compress_tf32(f32_dev(W))
    Y = nm.spmm_tf32(vals, meta, K, padded_x(X), out_dtype=out)
    torch.cuda.synchronize()
    nm.nm_device_status()
    ov, om = oracle.compress_f32(W)
    ref, mag = oracle.spmm_f32(ov, om, K, X, with_abs=True)
    assert_gemm_close(Y.float().cpu().numpy().astype(np.float64), ref, mag, f"tf32 {R}x{K}x{T} {out}")


@pytest.mark.parametrize("out", [torch.float32, torch.bfloat16])
def test_spmm_integer_exact(out):
    R, K, T = 384, 640, 264  # ten 64-deep stages, ragged T
    W = wl.integer_f32((R, K), -8, 8, seed=501)
    X = wl.integer_f32((K, T), -8, 8, seed=502)
    vals, meta = nm.prune_compress_tf32(f32_dev(W))
    Y = nm.spmm_tf32(vals, meta, K, padded_x(X), out_dtype=out)
    torch.cuda.synchronize()
    ov, om = oracle.compress_f32(W)
    ref = oracle.spmm_f32(ov, om, K, X)
    if out == torch.float32:
        assert np.array_equal(Y.contiguous().cpu().numpy().astype(np.float64), ref)
    else:
        assert np.array_equal(bits(Y), bf16_rne_of(ref))


def test_llama_layer_sampled():
    R, K, T = 4096, 4096, 2048
    W = wl.normal_f32((R, K), 0.02, seed=511)
    X = wl.normal_f32((K, T), 1.0, seed=512)
    vals, meta = nm.prune_compress_tf32(f32_dev(W))
    Y = nm.spmm_tf32(vals, meta, K, f32_dev(X))
    torch.cuda.synchronize()
    nm.nm_device_status()
    rows = np.array([0, 1, 2047, 4095])
    cols = np.array([0, 5, 1000, 2047])
    ov, om = oracle.compress_f32(W[rows])
    ref, mag = oracle.spmm_f32(ov, om, K, np.ascontiguousarray(X[:, cols]), with_abs=True)
    got = Y.cpu().numpy().astype(np.float64)[np.ix_(rows, cols)]
    assert_gemm_close(got, ref, mag, "tf32 LLaMA sampled")


def test_argument_errors():
    W = torch.zeros((4, 6), dtype=torch.float32, device=DEV)
    vals = torch.zeros((4, 3), dtype=torch.float32, device=DEV)
    meta = torch.zeros((4,), dtype=torch.int32, device=DEV)
    with pytest.raises(nm.NmError):
        nm.nm_prune_compress_tf32(W, 4, 5, 6, vals, meta)  # odd K
    X = torch.zeros((6, 8), dtype=torch.float32, device=DEV)
    Y = torch.zeros((4, 8), dtype=torch.float32, device=DEV)
    with pytest.raises(nm.NmError):
        nm.nm_spmm_tf32(vals, meta, 4, 6, X, 6, 8, Y, 8)  # ldx < T
    with pytest.raises(nm.NmError):
        nm.nm_spmm_tf32(vals, meta, 4, 6, X[:, 1:], 8, 7, Y, 8)  # X not 16-byte aligned
    nm.nm_spmm_tf32(vals, meta, 0, 6, X, 8, 8, Y, 8)  # R = 0: nothing to do
