"""GPU prune + compress and decompress against the oracle, bit for bit."""
import numpy as np
import pytest
import torch

import oracle
import sparse_gemm_nm_b200 as nm
import workloads as wl
from gpu_helpers import DEV, bits, to_dev, words

pytestmark = pytest.mark.gpu

PATTERNS = [(2, 4), (1, 4), (1, 8), (3, 4), (1, 2), (2, 8), (5, 8), (3, 16)]


def gpu_compress(W_bits, n, m, ldw=None):
    R, K = W_bits.shape
    if ldw is not None and ldw != K:  # strided rows
        buf = np.zeros((R, ldw), np.uint16)
        buf[:, :K] = W_bits
        Wd = to_dev(buf)
        vals = torch.empty((R, nm.nm_value_cols(K, n, m)), dtype=torch.bfloat16, device=DEV)
        meta = torch.empty((nm.nm_meta_words(R, K, n, m),), dtype=torch.int32, device=DEV)
        nm.nm_prune_compress(Wd, R, K, ldw, n, m, vals, meta)
    else:
        vals, meta = nm.prune_compress(to_dev(W_bits), n, m)
    torch.cuda.synchronize()
    return bits(vals), words(meta)


@pytest.mark.parametrize("n,m", PATTERNS)
@pytest.mark.parametrize("R,K", [(64, 128), (37, 96), (5, 48), (130, 1040), (3, 16)])
def test_compress_matches_oracle(n, m, R, K):
    if K % m:
        pytest.skip("K must be a multiple of M")
    W = wl.normal_bf16((R, K), 1.0, seed=R * 7 + K + n + m)
    v, mt = gpu_compress(W, n, m)
    ov, om = oracle.compress(W, n, m)
    assert np.array_equal(v, ov)
    assert np.array_equal(mt, om)


@pytest.mark.parametrize("n,m", [(2, 4), (1, 8), (3, 4)])
def test_compress_strided_rows(n, m):
    W = wl.normal_bf16((33, 256), 1.0, seed=5)
    v, mt = gpu_compress(W, n, m, ldw=264)
    ov, om = oracle.compress(W, n, m)
    assert np.array_equal(v, ov) and np.array_equal(mt, om)


@pytest.mark.parametrize("n,m", [(2, 4), (1, 4), (1, 8)])
def test_compress_ties_and_signed_zeros(n, m):
    """Small-integer weights (many ties), negative zeros and whole zero groups."""
    W = wl.integer_bf16((50, 64 * m), -2, 2, seed=17)
    W[3, :] = wl.bf16_bits(np.full(64 * m, -0.0, np.float32))
    W[4, :] = 0
    v, mt = gpu_compress(W, n, m)
    ov, om = oracle.compress(W, n, m)
    assert np.array_equal(v, ov) and np.array_equal(mt, om)


def test_compress_nonfinite():
    nan, inf = float("nan"), float("inf")
    rows = np.array([[nan, inf, 1.0, -inf] * 8, [1.0, nan, nan, 5.0] * 8, [-inf, 3.0, inf, 2.0] * 8,
                     [0.0, -0.0, 0.0, -0.0] * 8], np.float32)
    W = wl.bf16_bits(rows)
    W[1, 1] = 0x7FC1  # a second NaN payload ties with the first
    v, mt = gpu_compress(W, 2, 4)
    ov, om = oracle.compress(W, 2, 4)
    assert np.array_equal(v, ov) and np.array_equal(mt, om)


def test_worked_row_on_gpu():
    W = wl.bf16_bits(np.array([[1.5, 0, 0, -2.0, 0, 0.25, 3.0, 0] * 4], np.float32))
    _, mt = gpu_compress(W, 2, 4)
    # row 0, columns 0..15 -> word 0 low half; columns 16..31 -> word 0 of lane 8 (word 32)
    assert int(mt[0]) == 0x44449C9C and int(mt[32]) == 0x44449C9C


@pytest.mark.parametrize("n,m", PATTERNS)
def test_decompress_roundtrip(n, m):
    R, K = 45, 64 * m
    W = wl.normal_bf16((R, K), 1.0, seed=99 + m)
    vals, meta = nm.prune_compress(to_dev(W), n, m)
    D = nm.decompress(vals, meta, K, n, m)
    torch.cuda.synchronize()
    ov, om = oracle.compress(W, n, m)
    assert np.array_equal(bits(D), oracle.decompress(ov, om, K, n, m))
    assert np.array_equal(bits(D), np.where(oracle.prune_mask(W, n, m) == 1, W, np.uint16(0)))


@pytest.mark.parametrize("R,K", [(4096, 4096), (11008, 4096), (4096, 11008), (13824, 5120)])
def test_compress_full_size_2of4(R, K):
    """Full LLaMA-7B and decode weight shapes, whole arrays compared."""
    W = wl.normal_bf16((R, K), 0.02, seed=0)
    v, mt = gpu_compress(W, 2, 4)
    ov, om = oracle.compress(W, 2, 4)
    assert np.array_equal(v, ov) and np.array_equal(mt, om)


@pytest.mark.parametrize("R,K", [(3072, 768), (768, 3072)])
def test_compress_full_size_1of8(R, K):
    W = wl.normal_bf16((R, K), 0.02, seed=0)
    v, mt = gpu_compress(W, 1, 8)
    ov, om = oracle.compress(W, 1, 8)
    assert np.array_equal(v, ov) and np.array_equal(mt, om)


def test_empty_shapes():
    W = torch.empty((0, 64), dtype=torch.bfloat16, device=DEV)
    v, mt = nm.prune_compress(W, 2, 4)
    assert v.shape == (0, 32) and mt.shape == (0,)
    with pytest.raises(nm.NmError):
        nm.prune_compress(torch.zeros((4, 10), dtype=torch.bfloat16, device=DEV), 2, 4)


def test_selection_exhaustive_alphabet():
    """Every group of four over a 12-value alphabet (+-0, +-1, 1 + ulp, +-Inf, NaNs with different payloads and
    signs, denormals): the stream kernel (aligned rows), the other compress path (ldw % 8 != 0) and the fused
    prune + GEMM all select exactly as the oracle."""
    import itertools
    alphabet = [0x0000, 0x8000, 0x3F80, 0xBF80, 0x3F81, 0x7F80, 0xFF80, 0x7FC0, 0xFFC1, 0x7F81, 0x0001, 0x8001]
    groups = np.array(list(itertools.product(alphabet, repeat=4)), np.uint16)  # 20736 groups
    W = groups.reshape(-1, 128)  # 648 rows of 32 groups
    R, K = W.shape
    ov, om = oracle.compress(W, 2, 4)
    v, mt = gpu_compress(W, 2, 4)
    assert np.array_equal(v, ov) and np.array_equal(mt, om)
    v, mt = gpu_compress(W, 2, 4, ldw=132)
    assert np.array_equal(v, ov) and np.array_equal(mt, om)
    X = torch.zeros((K, 16), dtype=torch.bfloat16, device=DEV)
    _, fv, fm = nm.prune_spmm(to_dev(W), 2, 4, X, keep_compressed=True)
    torch.cuda.synchronize()
    assert np.array_equal(bits(fv), ov) and np.array_equal(words(fm), om)


# ----------------------------------------------------------------------------
# Row-wise patterns (warp kernel on aligned rows, per-word kernel otherwise)
# ----------------------------------------------------------------------------
def _alphabet_rows(alphabet, m, groups_per_row):
    import itertools
    groups = np.array(list(itertools.product(alphabet, repeat=m)), np.uint16)
    pad = (-len(groups)) % groups_per_row
    groups = np.concatenate([groups, np.zeros((pad, m), np.uint16)])
    return groups.reshape(-1, groups_per_row * m)


ALPHA12 = [0x0000, 0x8000, 0x3F80, 0xBF80, 0x3F81, 0x7F80, 0xFF80, 0x7FC0, 0xFFC1, 0x7F81, 0x0001, 0x8001]
ZERO_ONE_TWO = [0x0000, 0x3F80, 0x4000]       # {0, 1, 2}
ZERO_MINUS_ONE_TWO = [0x0000, 0xBF80, 0x4000]  # {0, -1, 2}


@pytest.mark.parametrize("n,m,alphabet", [(1, 8, ZERO_ONE_TWO), (2, 8, ZERO_ONE_TWO), (3, 8, ZERO_ONE_TWO),
                                          (4, 8, ZERO_ONE_TWO), (1, 8, ZERO_MINUS_ONE_TWO),
                                          (2, 8, ZERO_MINUS_ONE_TWO), (1, 4, ALPHA12), (3, 4, ALPHA12),
                                          (1, 2, ALPHA12)])
def test_rowwise_selection_exhaustive_alphabet(n, m, alphabet):
    """Every group of M over the alphabet ({0,1,2}^8 = 6561 groups of eight with their ties; the 12-value
    alphabet with NaN payloads, +-0, +-Inf and denormals for M = 4 and 2): the warp kernel (aligned rows) and
    the per-word kernel (row stride not a multiple of 8) both select exactly as the oracle."""
    W = _alphabet_rows(alphabet, m, 81 if m == 8 else 32)
    ov, om = oracle.compress(W, n, m)
    v, mt = gpu_compress(W, n, m)
    assert np.array_equal(v, ov) and np.array_equal(mt, om)
    v, mt = gpu_compress(W, n, m, ldw=W.shape[1] + 4)
    assert np.array_equal(v, ov) and np.array_equal(mt, om)


@pytest.mark.parametrize("n,m", [(1, 8), (2, 8), (1, 4)])
@pytest.mark.parametrize("R,K", [(7, 8), (3, 1032), (2, 10 * 8 * 33), (200, 5128)])
def test_rowwise_unit_tails(n, m, R, K):
    """Rows whose group count leaves a partial work unit and a partial last metadata word."""
    W = wl.normal_bf16((R, K), 1.0, seed=K + n)
    ov, om = oracle.compress(W, n, m)
    v, mt = gpu_compress(W, n, m)
    assert np.array_equal(v, ov) and np.array_equal(mt, om)


def test_compress_1of8_large_weight():
    """A 13824 x 5120 weight (141.6 MB) at 1:8, whole arrays compared."""
    W = wl.normal_bf16((13824, 5120), 0.02, seed=30)
    ov, om = oracle.compress(W, 1, 8)
    v, mt = gpu_compress(W, 1, 8)
    assert np.array_equal(v, ov) and np.array_equal(mt, om)
