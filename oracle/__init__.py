"""CPU oracle for N:M structured sparsity (test infrastructure only).

This package is the plain, slow, fp64 definition that the CUDA library is
checked against.  Only the tests, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may import it; the product package never does.

The arithmetic lives in ``nm_oracle.c`` (plain C, double accumulation).  This
module compiles it with gcc on first use (or via :func:`build`) and wraps each
function for numpy arrays.  bf16 values travel as their uint16 bit patterns.

Sources, by page title and passage:
  * "M:N sparsity on NVIDIA tensor cores" -- opening passage (2:4 definition
    and the worked row), "Fine-grained in what it removes, structured in how
    many" (2-bit positions, groups along the reduction axis), "Where this
    sits among the three case studies" (push-left format, 36-bit groups,
    sparse x dense = dense), "The recipe" (magnitude pruning).
  * "Technische Samenvatting: SHUFFLESPARSE", "2. Methodologie": y = (W Pi) x
    with Pi applied as an index map on the input read.
  * "Structured Sparsity" topic cards, PATCH abstract: per-tile dense / 2:4.
  * "M:N sparsity on NVIDIA tensor cores", the formats the sparse tensor cores
    take (INT8 among them) and the INT8 storage arithmetic: the ``*_i8`` functions.
  * The same passage: for TF32 the block halves to 1:2 -- the ``*_f32`` functions
    (float32 weights, 1:2 on the TF32 path).
  * SHUFFLESPARSE's contributions (block, N:M and diagonal patterns under one
    permutation) and the DynaDiag abstract: the ``diag_*`` functions (the pages
    give no format; see the readings in nm_oracle.c).
  * "Structured Sparsity" topic cards, RNM-TD3 abstract, and the DynaDiag
    page's abstract: N:M structure kept through training, sparse forward and
    backward passes (the gradients :func:`spmm_t` and :func:`sddmm`).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nm_oracle.c")
_LIB = os.path.join(_HERE, "libnm_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile nm_oracle.c into libnm_oracle.so next to it (gcc -O2)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P, I64, I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
            sig = {
                "oracle_index_bits": ([I], I),
                "oracle_positions_per_word": ([I], I),
                "oracle_value_cols": ([I64, I, I], I64),
                "oracle_meta_cols": ([I64, I, I], I64),
                "oracle_meta_words": ([I64, I64, I, I], I64),
                "oracle_positions": ([P, I64, I64, I, I, P], I),
                "oracle_prune_mask": ([P, I64, I64, I64, I, I, P], I),
                "oracle_compress": ([P, I64, I64, I64, I, I, P, P], I),
                "oracle_decompress": ([P, P, I64, I64, I, I, P, I64], I),
                "oracle_spmm": ([P, P, I, I, I64, I64, P, I64, I64, P, P, I64], I),
                "oracle_spmm_sampled": ([P, P, I, I, I64, I64, P, I64, I64, P, P, P, I64, P, P], I),
                "oracle_dense_gemm": ([P, I64, I64, I64, P, I64, I64, P, P, P, I64], I),
                "oracle_hybrid_weights": ([P, I64, I64, I64, P, I64, P], I),
                "oracle_hybrid_spmm": ([P, I64, I64, I64, P, I64, P, I64, I64, P, P, I64], I),
                "oracle_spmm_t": ([P, P, I, I, I64, I64, P, I64, I64, P, P, P, I64], I),
                "oracle_prune_mask_i8": ([P, I64, I64, I64, I, I, P], I),
                "oracle_diag_scores": ([P, I64, I64, I64, P], I),
                "oracle_diag_select": ([P, I64, I64, I64, I64, P], I),
                "oracle_diag_compress": ([P, I64, I64, I64, I64, P, P], I),
                "oracle_diag_expand": ([P, P, I64, I64, I64, P, I64], I),
                "oracle_diag_spmm": ([P, P, I64, I64, I64, P, I64, I64, P, P, P, I64], I),
                "oracle_compress_i8": ([P, I64, I64, I64, I, I, P, P], I),
                "oracle_decompress_i8": ([P, P, I64, I64, I, I, P, I64], I),
                "oracle_spmm_i8": ([P, P, I, I, I64, I64, P, I64, I64, P, I64], I),
                "oracle_sddmm": ([P, I, I, I64, I64, P, I64, P, I64, I64, P, P, P], I),
                "oracle_prune_mask_f32": ([P, I64, I64, I64, I, I, P], I),
                "oracle_compress_f32": ([P, I64, I64, I64, I, I, P, P], I),
                "oracle_decompress_f32": ([P, P, I64, I64, I, I, P, I64], I),
                "oracle_spmm_f32": ([P, P, I, I, I64, I64, P, I64, I64, P, P, I64], I),
            }
            for name, (args, res) in sig.items():
                fn = getattr(lib, name)
                fn.argtypes = args
                fn.restype = res
            _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data


def _u16(a):
    a = np.ascontiguousarray(a)
    assert a.dtype == np.uint16, "bf16 data travels as uint16 bit patterns"
    return a


def _check(rc, what):
    if rc != 0:
        raise ValueError(f"oracle {what} rejected its arguments (code {rc})")


def index_bits(m: int) -> int:
    return _load().oracle_index_bits(m)


def positions_per_word(m: int) -> int:
    return _load().oracle_positions_per_word(m)


def value_cols(K: int, n: int, m: int) -> int:
    return _load().oracle_value_cols(K, n, m)


def meta_cols(K: int, n: int, m: int) -> int:
    return _load().oracle_meta_cols(K, n, m)


def meta_words(R: int, K: int, n: int, m: int) -> int:
    """Total uint32 metadata words of an R x K matrix (tiled for 2:4, row-wise otherwise)."""
    return _load().oracle_meta_words(R, K, n, m)


def positions(meta: np.ndarray, R: int, K: int, n: int, m: int) -> np.ndarray:
    """R x K*n/m in-group positions of the survivors, read back from the metadata."""
    meta = np.ascontiguousarray(meta, dtype=np.uint32)
    out = np.zeros((R, value_cols(K, n, m)), np.uint8)
    _check(_load().oracle_positions(_ptr(meta), R, K, n, m, _ptr(out)), "positions")
    return out


def prune_mask(W: np.ndarray, n: int, m: int) -> np.ndarray:
    """uint8 R x K mask of the N:M survivors of bf16 W (R x K)."""
    W = _u16(W)
    R, K = W.shape
    mask = np.zeros((R, K), np.uint8)
    _check(_load().oracle_prune_mask(_ptr(W), R, K, K, n, m, _ptr(mask)), "prune_mask")
    return mask


def compress(W: np.ndarray, n: int, m: int):
    """(values R x K*n/m uint16, meta: meta_words uint32, flat) of bf16 W."""
    W = _u16(W)
    R, K = W.shape
    if K % m or not (1 <= n < m) or m not in (2, 4, 8, 16):
        raise ValueError(f"oracle compress rejected its arguments (K={K}, {n}:{m})")
    vals = np.zeros((R, value_cols(K, n, m)), np.uint16)
    meta = np.zeros(meta_words(R, K, n, m), np.uint32)
    _check(_load().oracle_compress(_ptr(W), R, K, K, n, m, _ptr(vals), _ptr(meta)), "compress")
    return vals, meta


def decompress(values: np.ndarray, meta: np.ndarray, K: int, n: int, m: int) -> np.ndarray:
    values = _u16(values)
    meta = np.ascontiguousarray(meta, dtype=np.uint32)
    R = values.shape[0]
    out = np.zeros((R, K), np.uint16)
    _check(_load().oracle_decompress(_ptr(values), _ptr(meta), R, K, n, m, _ptr(out), K), "decompress")
    return out


def spmm(values, meta, n, m, K, X, idx=None) -> np.ndarray:
    """fp64 y = (W' Pi) X from the compressed operand (idx = None: Pi = I)."""
    values = _u16(values)
    meta = np.ascontiguousarray(meta, dtype=np.uint32)
    X = _u16(X)
    R = values.shape[0]
    T = X.shape[1]
    if idx is not None:
        idx = np.ascontiguousarray(idx, dtype=np.int32)
    Y = np.zeros((R, T), np.float64)
    _check(_load().oracle_spmm(_ptr(values), _ptr(meta), n, m, R, K, _ptr(X), T, T,
                               _ptr(idx), _ptr(Y), T), "spmm")
    return Y


def spmm_sampled(values, meta, n, m, K, X, rows, cols, idx=None):
    """fp64 y[rows[i], cols[i]] and sum |w||x| for each sampled coordinate."""
    values = _u16(values)
    meta = np.ascontiguousarray(meta, dtype=np.uint32)
    X = _u16(X)
    R = values.shape[0]
    T = X.shape[1]
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    cols = np.ascontiguousarray(cols, dtype=np.int64)
    if idx is not None:
        idx = np.ascontiguousarray(idx, dtype=np.int32)
    out = np.zeros(rows.shape[0], np.float64)
    mag = np.zeros(rows.shape[0], np.float64)
    _check(_load().oracle_spmm_sampled(_ptr(values), _ptr(meta), n, m, R, K, _ptr(X), T, T,
                                       _ptr(idx), _ptr(rows), _ptr(cols), rows.shape[0],
                                       _ptr(out), _ptr(mag)), "spmm_sampled")
    return out, mag


def dense_gemm(W, X, idx=None, with_abs=False):
    """fp64 y = W X[idx] for bf16 W (R x K) and X (K x T); optionally sum |w||x|."""
    W = _u16(W)
    X = _u16(X)
    R, K = W.shape
    T = X.shape[1]
    if idx is not None:
        idx = np.ascontiguousarray(idx, dtype=np.int32)
    Y = np.zeros((R, T), np.float64)
    A = np.zeros((R, T), np.float64) if with_abs else None
    _check(_load().oracle_dense_gemm(_ptr(W), R, K, K, _ptr(X), T, T, _ptr(idx), _ptr(Y),
                                     _ptr(A), T), "dense_gemm")
    return (Y, A) if with_abs else Y


def hybrid_weights(W, tile_map, tile=128):
    W = _u16(W)
    R, K = W.shape
    tile_map = np.ascontiguousarray(tile_map, dtype=np.uint8)
    out = np.zeros((R, K), np.uint16)
    _check(_load().oracle_hybrid_weights(_ptr(W), R, K, K, _ptr(tile_map), tile, _ptr(out)),
           "hybrid_weights")
    return out


def hybrid_spmm(W, tile_map, X, tile=128, with_abs=False):
    W = _u16(W)
    X = _u16(X)
    R, K = W.shape
    T = X.shape[1]
    tile_map = np.ascontiguousarray(tile_map, dtype=np.uint8)
    Y = np.zeros((R, T), np.float64)
    A = np.zeros((R, T), np.float64) if with_abs else None
    _check(_load().oracle_hybrid_spmm(_ptr(W), R, K, K, _ptr(tile_map), tile, _ptr(X), T, T,
                                      _ptr(Y), _ptr(A), T), "hybrid_spmm")
    return (Y, A) if with_abs else Y


def spmm_t(values, meta, n, m, K, dY, idx=None, with_abs=False):
    """fp64 input gradient of y = (W' Pi) X: dX (K x T) from dY (R x T), the adjoint of the gather."""
    values = _u16(values)
    meta = np.ascontiguousarray(meta, dtype=np.uint32)
    dY = _u16(dY)
    R, T = dY.shape
    if idx is not None:
        idx = np.ascontiguousarray(idx, dtype=np.int32)
    dX = np.zeros((K, T), np.float64)
    A = np.zeros((K, T), np.float64) if with_abs else None
    _check(_load().oracle_spmm_t(_ptr(values), _ptr(meta), n, m, R, K, _ptr(dY), T, T, _ptr(idx), _ptr(dX),
                                 _ptr(A), T), "spmm_t")
    return (dX, A) if with_abs else dX


def sddmm(meta, n, m, R, K, dY, X, idx=None, with_abs=False):
    """fp64 gradient of the stored values: dV[r][j] = sum_t dY[r][t] X[pi(k_j)][t] (R x K*n/m)."""
    meta = np.ascontiguousarray(meta, dtype=np.uint32)
    dY = _u16(dY)
    X = _u16(X)
    T = dY.shape[1]
    if idx is not None:
        idx = np.ascontiguousarray(idx, dtype=np.int32)
    dV = np.zeros((R, value_cols(K, n, m)), np.float64)
    A = np.zeros_like(dV) if with_abs else None
    _check(_load().oracle_sddmm(_ptr(meta), n, m, R, K, _ptr(dY), T, _ptr(X), X.shape[1], T, _ptr(idx),
                                _ptr(dV), _ptr(A)), "sddmm")
    return (dV, A) if with_abs else dV


def _i8(a):
    a = np.ascontiguousarray(a)
    assert a.dtype == np.int8, "int8 data"
    return a


def prune_mask_i8(W, n, m):
    W = _i8(W)
    R, K = W.shape
    mask = np.zeros((R, K), np.uint8)
    _check(_load().oracle_prune_mask_i8(_ptr(W), R, K, K, n, m, _ptr(mask)), "prune_mask_i8")
    return mask


def compress_i8(W, n=2, m=4):
    """(values R x K*n/m int8, meta uint32) of int8 W, same metadata packing as compress()."""
    W = _i8(W)
    R, K = W.shape
    if K % m or not (1 <= n < m) or m not in (2, 4, 8, 16):
        raise ValueError(f"oracle compress_i8 rejected its arguments (K={K}, {n}:{m})")
    vals = np.zeros((R, value_cols(K, n, m)), np.int8)
    meta = np.zeros(meta_words(R, K, n, m), np.uint32)
    _check(_load().oracle_compress_i8(_ptr(W), R, K, K, n, m, _ptr(vals), _ptr(meta)), "compress_i8")
    return vals, meta


def decompress_i8(values, meta, K, n=2, m=4):
    values = _i8(values)
    meta = np.ascontiguousarray(meta, dtype=np.uint32)
    R = values.shape[0]
    out = np.zeros((R, K), np.int8)
    _check(_load().oracle_decompress_i8(_ptr(values), _ptr(meta), R, K, n, m, _ptr(out), K), "decompress_i8")
    return out


def spmm_i8(values, meta, K, X, n=2, m=4):
    """Exact int64 y = W' X for int8 compressed W' and int8 X (K x T)."""
    values = _i8(values)
    meta = np.ascontiguousarray(meta, dtype=np.uint32)
    X = _i8(X)
    R, T = values.shape[0], X.shape[1]
    Y = np.zeros((R, T), np.int64)
    _check(_load().oracle_spmm_i8(_ptr(values), _ptr(meta), n, m, R, K, _ptr(X), T, T, _ptr(Y), T), "spmm_i8")
    return Y


def _u32(a):
    """float32 data as its uint32 bit patterns (float32 or uint32 arrays)."""
    a = np.ascontiguousarray(a)
    if a.dtype == np.float32:
        return a.view(np.uint32)
    assert a.dtype == np.uint32, "float32 data or its uint32 bits"
    return a


def prune_mask_f32(W, n=1, m=2):
    """uint8 R x K mask of the N:M survivors of float32 W (TF32 path: 1:2)."""
    W = _u32(W)
    R, K = W.shape
    mask = np.zeros((R, K), np.uint8)
    _check(_load().oracle_prune_mask_f32(_ptr(W), R, K, K, n, m, _ptr(mask)), "prune_mask_f32")
    return mask


def compress_f32(W, n=1, m=2):
    """(values R x K*n/m as uint32 float32 bits, meta uint32) of float32 W; same packing as compress()."""
    W = _u32(W)
    R, K = W.shape
    if K % m or not (1 <= n < m) or m not in (2, 4, 8, 16):
        raise ValueError(f"oracle compress_f32 rejected its arguments (K={K}, {n}:{m})")
    vals = np.zeros((R, value_cols(K, n, m)), np.uint32)
    meta = np.zeros(meta_words(R, K, n, m), np.uint32)
    _check(_load().oracle_compress_f32(_ptr(W), R, K, K, n, m, _ptr(vals), _ptr(meta)), "compress_f32")
    return vals, meta


def decompress_f32(values, meta, K, n=1, m=2):
    values = _u32(values)
    meta = np.ascontiguousarray(meta, dtype=np.uint32)
    R = values.shape[0]
    out = np.zeros((R, K), np.uint32)
    _check(_load().oracle_decompress_f32(_ptr(values), _ptr(meta), R, K, n, m, _ptr(out), K), "decompress_f32")
    return out


def spmm_f32(values, meta, K, X, n=1, m=2, with_abs=False):
    """y = W' X in fp64 for float32 compressed W' and float32 X (K x T); optionally sum |w||x|."""
    values = _u32(values)
    meta = np.ascontiguousarray(meta, dtype=np.uint32)
    X = _u32(X)
    R, T = values.shape[0], X.shape[1]
    Y = np.zeros((R, T), np.float64)
    A = np.zeros((R, T), np.float64) if with_abs else None
    _check(_load().oracle_spmm_f32(_ptr(values), _ptr(meta), n, m, R, K, _ptr(X), T, T, _ptr(Y), _ptr(A), T),
           "spmm_f32")
    return (Y, A) if with_abs else Y


def diag_scores(W):
    """float64 scores s(o) = sum_r |W[r][(r + o) mod K]| (r ascending; NaN if the diagonal holds one)."""
    W = _u16(W)
    R, K = W.shape
    out = np.zeros(K, np.float64)
    _check(_load().oracle_diag_scores(_ptr(W), R, K, K, _ptr(out)), "diag_scores")
    return out


def diag_selection_errors(W, D, offsets, terms_exact=False):
    """Why ``offsets`` is not a valid choice of the D highest-scoring diagonals of W (empty list: it is).

    Several selections are correct when a device adds the scores in float32:
    two diagonals whose exact scores differ by less than the float32 rounding
    error may come out in either order.  A selection is accepted when
    * it holds D distinct offsets in [0, K), ascending;
    * every diagonal holding a NaN is kept before any other (NaNs tie among
      themselves: lower offsets first);
    * no dropped diagonal beats a kept one by more than the rounding error:
      min over kept of s*(1 + g) >= max over dropped of s*(1 - g), where s is
      the exact score (``diag_scores``) and g = (n - 1) u / (1 - (n - 1) u),
      u = 2^-24, bounds the relative error of ANY float32 summation order of
      n = R non-negative terms that are exact in float32 (Higham, "Accuracy
      and Stability of Numerical Algorithms", recursive summation bound).
    With ``terms_exact`` (every partial sum is exact in float32, e.g. small
    integers) g = 0 and equal scores must go to the lower offset.  The bound
    assumes the float32 sums do not overflow.
    """
    W = _u16(W)
    R, K = W.shape
    offs = np.asarray(offsets)
    errs = []
    if offs.shape != (D,):
        return [f"expected {D} offsets, got shape {offs.shape}"]
    if D and (offs.min() < 0 or offs.max() >= K):
        return ["offset outside [0, K)"]
    if np.any(np.diff(offs.astype(np.int64)) <= 0):
        return ["offsets not strictly ascending"]
    s = diag_scores(W)
    kept = np.zeros(K, bool)
    kept[offs] = True
    nan = np.isnan(s)
    if np.any(nan & ~kept) and np.any(~nan & kept):
        errs.append("a diagonal without NaN kept while one with NaN was dropped")
    kn, dn = np.flatnonzero(nan & kept), np.flatnonzero(nan & ~kept)
    if kn.size and dn.size and kn.max() > dn.min():
        errs.append("NaN diagonals not kept in offset order")
    fk, fd = np.flatnonzero(~nan & kept), np.flatnonzero(~nan & ~kept)
    if fk.size and fd.size:
        if terms_exact:
            a = fk[np.lexsort((-fk, s[fk]))[0]]        # weakest kept: lowest score, then highest offset
            b = fd[np.lexsort((fd, -s[fd]))[0]]        # strongest dropped: highest score, then lowest offset
            if s[a] < s[b] or (s[a] == s[b] and a > b):
                errs.append(f"dropped offset {b} (score {s[b]!r}) beats kept offset {a} (score {s[a]!r})")
        else:
            u = 2.0 ** -24
            g = (R - 1) * u / (1.0 - (R - 1) * u)
            lo, hi = s[fk].min() * (1.0 + g), s[fd].max() * (1.0 - g)
            if lo < hi:
                errs.append(f"a dropped score {s[fd].max()!r} beats the lowest kept score {s[fk].min()!r} by more "
                            f"than the float32 bound (relative {g:.3g})")
    return errs


def diag_select(W, D):
    """Ascending int32 offsets of the D diagonals with the largest scores (ties to the lower offset)."""
    W = _u16(W)
    R, K = W.shape
    out = np.zeros(D, np.int32)
    _check(_load().oracle_diag_select(_ptr(W), R, K, K, D, _ptr(out)), "diag_select")
    return out


def diag_compress(W, offsets):
    """V (D x R uint16): V[d][r] = W[r][(r + o_d) mod K]."""
    W = _u16(W)
    R, K = W.shape
    offsets = np.ascontiguousarray(offsets, dtype=np.int32)
    V = np.zeros((len(offsets), R), np.uint16)
    _check(_load().oracle_diag_compress(_ptr(W), R, K, K, len(offsets), _ptr(offsets), _ptr(V)), "diag_compress")
    return V


def diag_expand(values, offsets, K):
    values = _u16(values)
    offsets = np.ascontiguousarray(offsets, dtype=np.int32)
    D, R = values.shape
    out = np.zeros((R, K), np.uint16)
    _check(_load().oracle_diag_expand(_ptr(values), _ptr(offsets), D, R, K, _ptr(out), K), "diag_expand")
    return out


def diag_spmm(values, offsets, K, X, idx=None, with_abs=False):
    values = _u16(values)
    offsets = np.ascontiguousarray(offsets, dtype=np.int32)
    X = _u16(X)
    D, R = values.shape
    T = X.shape[1]
    if idx is not None:
        idx = np.ascontiguousarray(idx, dtype=np.int32)
    Y = np.zeros((R, T), np.float64)
    A = np.zeros((R, T), np.float64) if with_abs else None
    _check(_load().oracle_diag_spmm(_ptr(values), _ptr(offsets), D, R, K, _ptr(X), T, T, _ptr(idx), _ptr(Y),
                                    _ptr(A), T), "diag_spmm")
    return (Y, A) if with_abs else Y
