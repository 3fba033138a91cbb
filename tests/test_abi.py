"""The C-ABI library loads on a CPU-only machine and exports what include/nm.h declares.

No call here reaches a device: only the size helpers and argument checks that
the library answers on the host before any CUDA call.
"""
import ctypes
import os
import re

import pytest

import sparse_gemm_nm_b200 as nm

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    src = open(os.path.join(ROOT, "include", "nm.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*NM_API\s+[^(]*?\b(nm_[a-z0-9_]+)\s*\(", src, flags=re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    from sparse_gemm_nm_b200 import build
    build.build()
    return nm.lib()


def test_header_declares_the_five_calls():
    names = declared_functions()
    for call in ["nm_prune_compress", "nm_decompress", "nm_spmm", "nm_spmm_permuted", "nm_hybrid_spmm"]:
        assert call in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert name in nm.SIGNATURES, f"binding lacks a signature for {name}"


def test_size_helpers_match_oracle(lib):
    import oracle
    for R, K, n, m in [(4096, 11008, 2, 4), (13824, 5120, 2, 4), (6, 24, 2, 4), (3072, 768, 1, 8),
                       (256, 24, 1, 4), (33, 96, 3, 4), (5, 48, 5, 8)]:
        assert nm.nm_meta_words(R, K, n, m) == oracle.meta_words(R, K, n, m)
        assert nm.nm_value_cols(K, n, m) == oracle.value_cols(K, n, m)


def test_size_helpers(lib):
    assert nm.nm_index_bits(4) == 2 and nm.nm_index_bits(8) == 3 and nm.nm_index_bits(2) == 1
    assert nm.nm_index_bits(3) == 0
    assert nm.nm_value_cols(4096, 2, 4) == 2048
    assert nm.nm_meta_words(4096, 4096, 2, 4) == 4096 * 4096 // 32   # tiled 2:4
    assert nm.nm_meta_words(16, 24, 2, 4) == 64                      # one padded block
    assert nm.nm_meta_words(17, 128, 2, 4) == 128
    assert nm.nm_meta_words(3, 768, 1, 8) == 30                      # row-wise, 10 words a row
    assert nm.nm_meta_words(4, 10, 2, 4) == -1     # K % M != 0
    assert nm.nm_value_cols(16, 4, 4) == -1        # N must be below M


def test_host_argument_checks(lib):
    L = lib
    # bad pattern, K % M, negative sizes and null pointers are refused before any launch
    assert L.nm_prune_compress(None, 4, 16, 16, 5, 4, None, None, None) == nm.NM_ERR_INVALID_ARG
    assert L.nm_prune_compress(None, 4, 18, 18, 2, 4, None, None, None) == nm.NM_ERR_INVALID_ARG
    assert L.nm_prune_compress(None, 4, 16, 8, 2, 4, None, None, None) == nm.NM_ERR_INVALID_ARG
    assert L.nm_prune_compress(None, -1, 16, 16, 2, 4, None, None, None) == nm.NM_ERR_INVALID_ARG
    assert L.nm_prune_compress(None, 4, 16, 16, 2, 4, None, None, None) == nm.NM_ERR_INVALID_ARG
    assert b"null" in L.nm_last_error()
    assert L.nm_decompress(None, None, 4, 16, 1, 3, None, 16, None) == nm.NM_ERR_INVALID_ARG
    assert L.nm_spmm(None, None, 2, 4, 8, 30, None, 8, 8, None, 8, 0, None) == nm.NM_ERR_INVALID_ARG
    assert L.nm_spmm(None, None, 2, 4, 8, 32, None, 8, 8, None, 4, 0, None) == nm.NM_ERR_INVALID_ARG
    assert L.nm_spmm(None, None, 2, 4, 8, 32, None, 8, 8, None, 8, 7, None) == nm.NM_ERR_INVALID_ARG
    assert L.nm_spmm_permuted(None, None, 2, 4, 8, 32, None, None, 8, 8, None, 8, 0, None) == nm.NM_ERR_INVALID_ARG
    # empty outputs are a no-op that never touches the device
    assert L.nm_spmm(None, None, 2, 4, 0, 32, None, 8, 8, None, 8, 0, None) == nm.NM_OK
    assert L.nm_spmm(None, None, 2, 4, 8, 32, None, 8, 0, None, 8, 0, None) == nm.NM_OK
    assert L.nm_prune_compress(None, 0, 16, 16, 2, 4, None, None, None) == nm.NM_OK


def test_status_strings(lib):
    for s in range(7):
        assert nm.lib().nm_status_string(s)
    assert nm.nm_version() >= 100


def test_product_package_does_not_touch_the_oracle():
    """The product path never imports, links or loads the oracle."""
    pkg = os.path.join(ROOT, "sparse_gemm_nm_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                text = open(os.path.join(dirpath, f)).read()
                assert "oracle" not in text.replace("oracle as the", ""), f


def test_host_argument_checks_of_the_format_calls(lib):
    """The TF32, INT8 and diagonal calls refuse bad shapes, leading dimensions and nulls before any launch."""
    L = lib
    I = nm.NM_ERR_INVALID_ARG
    assert L.nm_prune_compress_tf32(None, 4, 5, 6, None, None, None) == I          # odd K (1:2)
    assert L.nm_prune_compress_tf32(None, 4, 8, 6, None, None, None) == I          # ldw < K
    assert L.nm_prune_compress_tf32(None, 4, 8, 8, None, None, None) == I          # null pointers
    assert L.nm_prune_compress_tf32(None, 0, 8, 8, None, None, None) == nm.NM_OK   # empty
    assert L.nm_decompress_tf32(None, None, 4, 7, None, 8, None) == I
    assert L.nm_spmm_tf32(None, None, 4, 8, None, 8, 8, None, 8, 7, None) == I     # bad output dtype
    assert L.nm_spmm_tf32(None, None, 4, 8, None, 8, 8, None, 4, 0, None) == I     # ldy < T
    assert L.nm_spmm_tf32(None, None, 4, 8, None, 8, 8, None, 8, 0, None) == I     # Y null
    assert L.nm_spmm_tf32(None, None, 0, 8, None, 8, 8, None, 8, 0, None) == nm.NM_OK
    assert L.nm_diag_prune_compress(None, 4, 8, 8, 9, None, None, None) == I       # D > K
    assert L.nm_diag_prune_compress(None, 4, 8, 6, 2, None, None, None) == I       # ldw < K
    assert L.nm_diag_expand(None, None, 9, 4, 8, None, 8, None) == I               # D > K
    assert L.nm_diag_spmm(None, None, 9, 4, 8, None, None, 8, 8, None, 8, 0, None) == I
    assert L.nm_diag_spmm(None, None, 2, 4, 8, None, None, 8, 8, None, 4, 0, None) == I  # ldy < T
    assert L.nm_prune_compress_i8(None, 4, 16, 8, None, None, None) == I           # ldw < K
    assert L.nm_spmm_i8(None, None, 4, 16, None, 16, 16, None, 8, None) == I       # ldy < T
