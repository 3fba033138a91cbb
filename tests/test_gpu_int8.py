"""GPU INT8 2:4 (compress, decompress, exact int32 GEMM) against the oracle, bit for bit."""
import itertools

import numpy as np
import pytest
import torch

import oracle
import sparse_gemm_nm_b200 as nm
import workloads as wl
from gpu_helpers import DEV, words

pytestmark = pytest.mark.gpu


def dev_i8(a, ld=None):
    """int8 rows on the device; with ld, rows padded to ld (a view of a wider buffer)."""
    a = np.ascontiguousarray(a)
    if ld is None:
        return torch.from_numpy(a).to(DEV)
    buf = np.zeros((a.shape[0], ld), np.int8)
    buf[:, :a.shape[1]] = a
    return torch.from_numpy(buf).to(DEV)[:, :a.shape[1]]


@pytest.mark.parametrize("R,K", [(64, 128), (37, 256), (130, 1040), (300, 4096), (16, 16)])
@pytest.mark.parametrize("lo,hi", [(-128, 127), (-2, 2)])
def test_compress_i8_matches_oracle(R, K, lo, hi):
    W = wl.integer_i8((R, K), lo, hi, seed=R + K + hi)
    vals, meta = nm.prune_compress_i8(dev_i8(W))
    torch.cuda.synchronize()
    ov, om = oracle.compress_i8(W)
    assert np.array_equal(vals.cpu().numpy(), ov)
    assert np.array_equal(words(meta), om)


def test_compress_i8_strided_rows_and_alphabet():
    alphabet = [-128, -127, -1, 0, 1, 5, -5, 127]
    W = np.array(list(itertools.product(alphabet, repeat=4)), np.int8).reshape(-1, 128)  # every group, 32 rows
    R, K = W.shape
    vals = torch.empty((R, K // 2), dtype=torch.int8, device=DEV)
    meta = torch.empty((nm.nm_meta_words(R, K, 2, 4),), dtype=torch.int32, device=DEV)
    nm.nm_prune_compress_i8(dev_i8(W, ld=K + 8), R, K, K + 8, vals, meta)
    torch.cuda.synchronize()
    ov, om = oracle.compress_i8(W)
    assert np.array_equal(vals.cpu().numpy(), ov) and np.array_equal(words(meta), om)


@pytest.mark.parametrize("R,K", [(64, 128), (37, 256), (300, 1040)])
def test_decompress_i8_roundtrip(R, K):
    W = wl.integer_i8((R, K), -128, 127, seed=R * K)
    vals, meta = nm.prune_compress_i8(dev_i8(W))
    Wd = nm.decompress_i8(vals, meta, K)
    torch.cuda.synchronize()
    ov, om = oracle.compress_i8(W)
    assert np.array_equal(Wd.cpu().numpy(), oracle.decompress_i8(ov, om, K))


# T >= 192 with K % 32 == 0 runs on the sparse tensor cores (kind::i8, metadata re-laid out per row,
# 256 x 256 tiles, 256-deep stages); other shapes on the decompressed dense operand.
@pytest.mark.parametrize("R,K,T", [(300, 512, 264), (256, 1024, 256), (130, 384, 100), (64, 128, 16),
                                   (520, 256, 40), (600, 2048, 520), (260, 800, 320), (200, 1040, 256),
                                   (260, 8192, 264),    # 32 stages, a second column tile 8 wide
                                   (520, 2048, 2000),   # 8 column tiles, the last one 208 wide
                                   (260, 8448, 264)])   # 33 stages, ragged rows
def test_spmm_i8_exact(R, K, T):
    W = wl.integer_i8((R, K), -128, 127, seed=R + 7 * K)
    X = wl.integer_i8((K, T), -128, 127, seed=T + 3)
    vals, meta = nm.prune_compress_i8(dev_i8(W))
    Y = nm.spmm_i8(vals, meta, K, dev_i8(X, ld=(T + 15) // 16 * 16))
    torch.cuda.synchronize()
    nm.nm_device_status()
    ov, om = oracle.compress_i8(W)
    ref = oracle.spmm_i8(ov, om, K, X)
    assert np.array_equal(Y.cpu().numpy().astype(np.int64), ref)


def test_spmm_i8_meta_only_4_byte_aligned():
    """Metadata 4 bytes past a 16-byte boundary (the call asks for 4): the
    re-layout reads it word by word; the product is unchanged."""
    R, K, T = 300, 1024, 264
    W = wl.integer_i8((R, K), -128, 127, seed=31)
    X = wl.integer_i8((K, T), -128, 127, seed=32)
    vals, meta = nm.prune_compress_i8(dev_i8(W))
    Xd = dev_i8(X, ld=(T + 15) // 16 * 16)
    Y = nm.spmm_i8(vals, meta, K, Xd)
    buf = torch.zeros((meta.numel() + 4,), dtype=torch.int32, device=DEV)
    off = next(o for o in range(4) if (buf.data_ptr() + 4 * o) % 16 == 4)
    meta4 = buf[off:off + meta.numel()]
    meta4.copy_(meta)
    assert meta4.data_ptr() % 16 == 4
    Y4 = nm.spmm_i8(vals, meta4, K, Xd)
    torch.cuda.synchronize()
    nm.nm_device_status()
    assert torch.equal(Y, Y4)
    ov, om = oracle.compress_i8(W)
    assert np.array_equal(Y4.cpu().numpy().astype(np.int64), oracle.spmm_i8(ov, om, K, X))


def test_spmm_i8_llama_layer_sampled():
    R, K, T = 4096, 4096, 2048
    W = wl.normal_i8((R, K), 32.0, seed=21)
    X = wl.integer_i8((K, T), -128, 127, seed=22)
    vals, meta = nm.prune_compress_i8(dev_i8(W))
    Y = nm.spmm_i8(vals, meta, K, dev_i8(X))
    torch.cuda.synchronize()
    nm.nm_device_status()
    ov, om = oracle.compress_i8(W)
    assert np.array_equal(vals.cpu().numpy(), ov) and np.array_equal(words(meta), om)
    cols = np.array([0, 1, 513, 1500, T - 1])
    ref = oracle.spmm_i8(ov, om, K, np.ascontiguousarray(X[:, cols]))
    assert np.array_equal(Y.cpu().numpy()[:, cols].astype(np.int64), ref)


def test_int8_argument_checks():
    W = torch.zeros((16, 24), dtype=torch.int8, device=DEV)
    vals = torch.empty((16, 12), dtype=torch.int8, device=DEV)
    meta = torch.empty((64,), dtype=torch.int32, device=DEV)
    with pytest.raises(nm.NmError) as e:
        nm.nm_prune_compress_i8(W, 16, 24, 24, vals, meta)  # K % 16 != 0
    assert e.value.status == nm.NM_ERR_UNSUPPORTED
