"""sparse_gemm_nm_b200 -- N:M structured weight sparsity on NVIDIA B200 (sm_100a).

Python binding of the C ABI in ``include/nm.h`` (library ``libnm_b200.so``).
The functions named like the C entry points (``nm_prune_compress``,
``nm_decompress``, ``nm_spmm``, ``nm_spmm_permuted``, ``nm_hybrid_spmm``,
``nm_spmm_algo``, ``nm_prune_spmm``, ``nm_spmm_t``, ``nm_sddmm``) only marshal arguments: tensors become device pointers, the
stream defaults to torch's current stream, and a non-zero status raises
:class:`NmError`.  Every step of the computation runs in the library's CUDA
kernels; there is no fallback of any kind.  The convenience wrappers
(``prune_compress``, ``decompress``, ``spmm``, ``hybrid_spmm``, ``prune_spmm``, ``spmm_t``,
``sddmm``) also allocate
the outputs with torch.

bf16 data is accepted as ``torch.bfloat16`` tensors (or int16/uint16 views of
the same bits).  Matrices are row-major: W is R x K, X is K x T, Y is R x T.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libnm_b200.so")

NM_OK = 0
NM_ERR_INVALID_ARG = 1
NM_ERR_UNSUPPORTED = 2
NM_ERR_MISALIGNED = 3
NM_ERR_CUDA = 4
NM_ERR_TIMEOUT = 5
NM_ERR_NO_DEVICE = 6

NM_OUT_BF16 = 0
NM_OUT_F32 = 1

NM_ALGO_AUTO = 0
NM_ALGO_SPARSE_TC = 1
NM_ALGO_DENSE_TC = 2

# Every symbol include/nm.h declares, with its ctypes signature.
_P, _I64, _I, _U64 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_uint64
SIGNATURES = {
    "nm_index_bits": ([_I], _I),
    "nm_value_cols": ([_I64, _I, _I], _I64),
    "nm_meta_words": ([_I64, _I64, _I, _I], _I64),
    "nm_prune_compress": ([_P, _I64, _I64, _I64, _I, _I, _P, _P, _P], _I),
    "nm_decompress": ([_P, _P, _I64, _I64, _I, _I, _P, _I64, _P], _I),
    "nm_spmm": ([_P, _P, _I, _I, _I64, _I64, _P, _I64, _I64, _P, _I64, _I, _P], _I),
    "nm_spmm_permuted": ([_P, _P, _I, _I, _I64, _I64, _P, _P, _I64, _I64, _P, _I64, _I, _P], _I),
    "nm_hybrid_spmm": ([_P, _I64, _P, _P, _P, _I, _I64, _I64, _P, _I64, _I64, _P, _I64, _I, _P], _I),
    "nm_prune_spmm": ([_P, _I64, _I, _I, _I64, _I64, _P, _P, _I64, _I64, _P, _I64, _I, _P, _P, _P], _I),
    "nm_spmm_t": ([_P, _P, _I, _I, _I64, _I64, _P, _P, _I64, _I64, _P, _I64, _I, _P], _I),
    "nm_prune_compress_i8": ([_P, _I64, _I64, _I64, _P, _P, _P], _I),
    "nm_diag_prune_compress": ([_P, _I64, _I64, _I64, _I64, _P, _P, _P], _I),
    "nm_diag_expand": ([_P, _P, _I64, _I64, _I64, _P, _I64, _P], _I),
    "nm_diag_spmm": ([_P, _P, _I64, _I64, _I64, _P, _P, _I64, _I64, _P, _I64, _I, _P], _I),
    "nm_decompress_i8": ([_P, _P, _I64, _I64, _P, _I64, _P], _I),
    "nm_spmm_i8": ([_P, _P, _I64, _I64, _P, _I64, _I64, _P, _I64, _P], _I),
    "nm_prune_compress_tf32": ([_P, _I64, _I64, _I64, _P, _P, _P], _I),
    "nm_decompress_tf32": ([_P, _P, _I64, _I64, _P, _I64, _P], _I),
    "nm_spmm_tf32": ([_P, _P, _I64, _I64, _P, _I64, _I64, _P, _I64, _I, _P], _I),
    "nm_sddmm": ([_P, _I, _I, _I64, _I64, _P, _P, _I64, _P, _I64, _I64, _P, _I, _P], _I),
    "nm_spmm_algo": ([_P, _P, _I, _I, _I64, _I64, _P, _P, _I64, _I64, _P, _I64, _I, _I, _P], _I),
    "nm_spmm_permuted_noalloc": ([_P, _P, _I, _I, _I64, _I64, _P, _P, _I64, _I64, _P, _I64, _I, _P], _I),
    "nm_release_staging": ([], _I),
    "nm_selftest_wait_timeout": ([ctypes.c_uint32, _P], _I),
    "nm_device_status": ([_P], _I),
    "nm_status_string": ([_I], ctypes.c_char_p),
    "nm_last_error": ([], ctypes.c_char_p),
    "nm_launch_count": ([], _U64),
    "nm_version": ([], _I),
}


class NmError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str):
        super().__init__(f"{where}: status {status} ({_status_text(status)}): {detail}")
        self.status = status


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded libnm_b200.so.  Raises ImportError when it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with `python -m sparse_gemm_nm_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = res
        _lib = L
    return _lib


def _status_text(s: int) -> str:
    try:
        return lib().nm_status_string(s).decode()
    except Exception:  # pragma: no cover - only while reporting another failure
        return "?"


def _check(status: int, where: str) -> None:
    if status != NM_OK:
        raise NmError(status, where, lib().nm_last_error().decode())


def _ptr(x) -> Optional[int]:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


# ----------------------------------------------------------------------------
# C-ABI names (argument marshalling only)
# ----------------------------------------------------------------------------
def nm_index_bits(m: int) -> int:
    return lib().nm_index_bits(m)


def nm_value_cols(K: int, n: int, m: int) -> int:
    return lib().nm_value_cols(K, n, m)


def nm_meta_words(R: int, K: int, n: int, m: int) -> int:
    return lib().nm_meta_words(R, K, n, m)


def nm_prune_compress(W, R, K, ldw, n, m, values, meta, stream=None) -> None:
    _check(lib().nm_prune_compress(_ptr(W), R, K, ldw, n, m, _ptr(values), _ptr(meta), _stream(stream)),
           "nm_prune_compress")


def nm_decompress(values, meta, R, K, n, m, W_out, ldw, stream=None) -> None:
    _check(lib().nm_decompress(_ptr(values), _ptr(meta), R, K, n, m, _ptr(W_out), ldw, _stream(stream)),
           "nm_decompress")


def nm_spmm(values, meta, n, m, R, K, X, ldx, T, Y, ldy, y_dtype=NM_OUT_BF16, stream=None) -> None:
    _check(lib().nm_spmm(_ptr(values), _ptr(meta), n, m, R, K, _ptr(X), ldx, T, _ptr(Y), ldy, y_dtype,
                         _stream(stream)), "nm_spmm")


def nm_spmm_permuted(values, meta, n, m, R, K, idx, X, ldx, T, Y, ldy, y_dtype=NM_OUT_BF16,
                     stream=None) -> None:
    _check(lib().nm_spmm_permuted(_ptr(values), _ptr(meta), n, m, R, K, _ptr(idx), _ptr(X), ldx, T, _ptr(Y),
                                  ldy, y_dtype, _stream(stream)), "nm_spmm_permuted")


def nm_hybrid_spmm(W, ldw, values, meta, tile_map, tile, R, K, X, ldx, T, Y, ldy, y_dtype=NM_OUT_BF16,
                   stream=None) -> None:
    _check(lib().nm_hybrid_spmm(_ptr(W), ldw, _ptr(values), _ptr(meta), _ptr(tile_map), tile, R, K, _ptr(X),
                                ldx, T, _ptr(Y), ldy, y_dtype, _stream(stream)), "nm_hybrid_spmm")


def nm_prune_spmm(W, ldw, n, m, R, K, idx, X, ldx, T, Y, ldy, y_dtype=NM_OUT_BF16, values=None, meta=None,
                  stream=None) -> None:
    _check(lib().nm_prune_spmm(_ptr(W), ldw, n, m, R, K, _ptr(idx), _ptr(X), ldx, T, _ptr(Y), ldy, y_dtype,
                               _ptr(values), _ptr(meta), _stream(stream)), "nm_prune_spmm")


def nm_spmm_t(values, meta, n, m, R, K, idx, dY, lddy, T, dX, lddx, dtype=NM_OUT_BF16, stream=None) -> None:
    _check(lib().nm_spmm_t(_ptr(values), _ptr(meta), n, m, R, K, _ptr(idx), _ptr(dY), lddy, T, _ptr(dX), lddx,
                           dtype, _stream(stream)), "nm_spmm_t")


def nm_sddmm(meta, n, m, R, K, idx, dY, lddy, X, ldx, T, dV, dtype=NM_OUT_BF16, stream=None) -> None:
    _check(lib().nm_sddmm(_ptr(meta), n, m, R, K, _ptr(idx), _ptr(dY), lddy, _ptr(X), ldx, T, _ptr(dV), dtype,
                          _stream(stream)), "nm_sddmm")


def nm_prune_compress_i8(W, R, K, ldw, values, meta, stream=None) -> None:
    _check(lib().nm_prune_compress_i8(_ptr(W), R, K, ldw, _ptr(values), _ptr(meta), _stream(stream)),
           "nm_prune_compress_i8")


def nm_decompress_i8(values, meta, R, K, W_out, ldw, stream=None) -> None:
    _check(lib().nm_decompress_i8(_ptr(values), _ptr(meta), R, K, _ptr(W_out), ldw, _stream(stream)),
           "nm_decompress_i8")


def nm_spmm_i8(values, meta, R, K, X, ldx, T, Y, ldy, stream=None) -> None:
    _check(lib().nm_spmm_i8(_ptr(values), _ptr(meta), R, K, _ptr(X), ldx, T, _ptr(Y), ldy, _stream(stream)),
           "nm_spmm_i8")


def nm_prune_compress_tf32(W, R, K, ldw, values, meta, stream=None) -> None:
    _check(lib().nm_prune_compress_tf32(_ptr(W), R, K, ldw, _ptr(values), _ptr(meta), _stream(stream)),
           "nm_prune_compress_tf32")


def nm_decompress_tf32(values, meta, R, K, W_out, ldw, stream=None) -> None:
    _check(lib().nm_decompress_tf32(_ptr(values), _ptr(meta), R, K, _ptr(W_out), ldw, _stream(stream)),
           "nm_decompress_tf32")


def nm_spmm_tf32(values, meta, R, K, X, ldx, T, Y, ldy, y_dtype=NM_OUT_F32, stream=None) -> None:
    _check(lib().nm_spmm_tf32(_ptr(values), _ptr(meta), R, K, _ptr(X), ldx, T, _ptr(Y), ldy, y_dtype,
                              _stream(stream)), "nm_spmm_tf32")


def nm_diag_prune_compress(W, R, K, ldw, D, offsets, values, stream=None) -> None:
    _check(lib().nm_diag_prune_compress(_ptr(W), R, K, ldw, D, _ptr(offsets), _ptr(values), _stream(stream)),
           "nm_diag_prune_compress")


def nm_diag_expand(values, offsets, D, R, K, W_out, ldw, stream=None) -> None:
    _check(lib().nm_diag_expand(_ptr(values), _ptr(offsets), D, R, K, _ptr(W_out), ldw, _stream(stream)),
           "nm_diag_expand")


def nm_diag_spmm(values, offsets, D, R, K, idx, X, ldx, T, Y, ldy, y_dtype=NM_OUT_BF16, stream=None) -> None:
    _check(lib().nm_diag_spmm(_ptr(values), _ptr(offsets), D, R, K, _ptr(idx), _ptr(X), ldx, T, _ptr(Y), ldy,
                              y_dtype, _stream(stream)), "nm_diag_spmm")


def nm_spmm_algo(values, meta, n, m, R, K, idx, X, ldx, T, Y, ldy, y_dtype=NM_OUT_BF16, algo=NM_ALGO_AUTO,
                 stream=None) -> None:
    _check(lib().nm_spmm_algo(_ptr(values), _ptr(meta), n, m, R, K, _ptr(idx), _ptr(X), ldx, T, _ptr(Y), ldy,
                              y_dtype, algo, _stream(stream)), "nm_spmm_algo")


def nm_spmm_permuted_noalloc(values, meta, n, m, R, K, idx, X, ldx, T, Y, ldy, y_dtype=NM_OUT_BF16,
                             stream=None) -> None:
    _check(lib().nm_spmm_permuted_noalloc(_ptr(values), _ptr(meta), n, m, R, K, _ptr(idx), _ptr(X), ldx, T,
                                          _ptr(Y), ldy, y_dtype, _stream(stream)), "nm_spmm_permuted_noalloc")


def nm_selftest_wait_timeout(limit_us: int, stream=None) -> None:
    _check(lib().nm_selftest_wait_timeout(limit_us, _stream(stream)), "nm_selftest_wait_timeout")


def nm_release_staging() -> None:
    _check(lib().nm_release_staging(), "nm_release_staging")


def nm_device_status(stream=None) -> None:
    _check(lib().nm_device_status(_stream(stream)), "nm_device_status")


def nm_launch_count() -> int:
    return int(lib().nm_launch_count())


def nm_version() -> int:
    return int(lib().nm_version())


# ----------------------------------------------------------------------------
# Convenience wrappers that allocate outputs with torch
# ----------------------------------------------------------------------------
def _require_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("tensors must live on a CUDA device")


def prune_compress(W, n: int, m: int, stream=None):
    """(values R x K*n/m bf16, meta: nm_meta_words uint32 as int32, flat) of bf16 W (R x K)."""
    import torch
    _require_cuda(W)
    R, K = W.shape
    if nm_value_cols(K, n, m) < 0:  # let the library name the bad argument
        _check(lib().nm_prune_compress(None, R, K, K, n, m, None, None, None), "nm_prune_compress")
    vals = torch.empty((R, nm_value_cols(K, n, m)), dtype=torch.bfloat16, device=W.device)
    meta = torch.empty((max(nm_meta_words(R, K, n, m), 0),), dtype=torch.int32, device=W.device)
    nm_prune_compress(W, R, K, W.stride(0), n, m, vals, meta, stream)
    return vals, meta


def decompress(values, meta, K: int, n: int, m: int, stream=None):
    import torch
    _require_cuda(values, meta)
    R = values.shape[0]
    out = torch.empty((R, K), dtype=torch.bfloat16, device=values.device)
    nm_decompress(values, meta, R, K, n, m, out, K, stream)
    return out


def spmm(values, meta, n: int, m: int, K: int, X, idx=None, out_dtype=None, algo: int = NM_ALGO_AUTO,
         stream=None):
    """Y = (W' Pi) X from the compressed operand; idx=None means Pi = I."""
    import torch
    _require_cuda(values, meta, X, idx)
    out_dtype = out_dtype or torch.bfloat16
    R, T = values.shape[0], X.shape[1]
    Y = torch.empty((R, T), dtype=out_dtype, device=X.device)
    yt = NM_OUT_F32 if out_dtype == torch.float32 else NM_OUT_BF16
    if algo == NM_ALGO_AUTO and idx is None:
        nm_spmm(values, meta, n, m, R, K, X, X.stride(0), T, Y, T, yt, stream)
    elif algo == NM_ALGO_AUTO:
        nm_spmm_permuted(values, meta, n, m, R, K, idx, X, X.stride(0), T, Y, T, yt, stream)
    else:
        nm_spmm_algo(values, meta, n, m, R, K, idx, X, X.stride(0), T, Y, T, yt, algo, stream)
    return Y


def hybrid_spmm(W, values, meta, tile_map, X, tile: int = 128, out_dtype=None, stream=None):
    import torch
    _require_cuda(W, values, meta, tile_map, X)
    out_dtype = out_dtype or torch.bfloat16
    R, K = W.shape
    T = X.shape[1]
    Y = torch.empty((R, T), dtype=out_dtype, device=X.device)
    yt = NM_OUT_F32 if out_dtype == torch.float32 else NM_OUT_BF16
    nm_hybrid_spmm(W, W.stride(0), values, meta, tile_map, tile, R, K, X, X.stride(0), T, Y, T, yt, stream)
    return Y


def prune_spmm(W, n: int, m: int, X, idx=None, out_dtype=None, keep_compressed: bool = False, stream=None):
    """Y = (W' Pi) X with W' the n:m magnitude-pruned W, from the dense W in one call.

    With keep_compressed=True also returns (values, meta) as prune_compress would.
    Y's rows are padded to 16 bytes; the returned tensor is the R x T view.
    """
    import torch
    _require_cuda(W, X, idx)
    out_dtype = out_dtype or torch.bfloat16
    R, K = W.shape
    T = X.shape[1]
    per16 = 4 if out_dtype == torch.float32 else 8
    ldy = max((T + per16 - 1) // per16 * per16, per16)
    Y = torch.empty((R, ldy), dtype=out_dtype, device=X.device)
    yt = NM_OUT_F32 if out_dtype == torch.float32 else NM_OUT_BF16
    vals = meta = None
    if keep_compressed:
        if nm_value_cols(K, n, m) < 0:
            _check(lib().nm_prune_compress(None, R, K, K, n, m, None, None, None), "nm_prune_spmm")
        vals = torch.empty((R, nm_value_cols(K, n, m)), dtype=torch.bfloat16, device=W.device)
        meta = torch.empty((max(nm_meta_words(R, K, n, m), 0),), dtype=torch.int32, device=W.device)
    nm_prune_spmm(W, W.stride(0), n, m, R, K, idx, X, X.stride(0), T, Y, ldy, yt, vals, meta, stream)
    Y = Y[:, :T]
    return (Y, vals, meta) if keep_compressed else Y


def spmm_t(values, meta, n: int, m: int, K: int, dY, idx=None, out_dtype=None, stream=None):
    """dX = (W' Pi)^T dY (K x T) from the compressed operand; idx=None means Pi = I."""
    import torch
    _require_cuda(values, meta, dY, idx)
    out_dtype = out_dtype or torch.bfloat16
    R, T = dY.shape
    per16 = 4 if out_dtype == torch.float32 else 8
    ld = max((T + per16 - 1) // per16 * per16, per16)
    dX = torch.empty((K, ld), dtype=out_dtype, device=dY.device)
    yt = NM_OUT_F32 if out_dtype == torch.float32 else NM_OUT_BF16
    nm_spmm_t(values, meta, n, m, R, K, idx, dY, dY.stride(0), T, dX, ld, yt, stream)
    return dX[:, :T]


def sddmm(meta, n: int, m: int, R: int, K: int, dY, X, idx=None, out_dtype=None, stream=None):
    """dV[r][j] = sum_t dY[r][t] X[idx[k_j]][t] (R x K*n/m), the gradient of the stored values."""
    import torch
    _require_cuda(meta, dY, X, idx)
    out_dtype = out_dtype or torch.bfloat16
    T = dY.shape[1]
    dV = torch.empty((R, max(nm_value_cols(K, n, m), 0)), dtype=out_dtype, device=dY.device)
    yt = NM_OUT_F32 if out_dtype == torch.float32 else NM_OUT_BF16
    nm_sddmm(meta, n, m, R, K, idx, dY, dY.stride(0), X, X.stride(0), T, dV, yt, stream)
    return dV


def prune_compress_i8(W, stream=None):
    """2:4 (values R x K/2 int8, meta uint32 as int32) of int8 W (R x K)."""
    import torch
    _require_cuda(W)
    R, K = W.shape
    vals = torch.empty((R, K // 2), dtype=torch.int8, device=W.device)
    meta = torch.empty((max(nm_meta_words(R, K, 2, 4), 0),), dtype=torch.int32, device=W.device)
    nm_prune_compress_i8(W, R, K, W.stride(0), vals, meta, stream)
    return vals, meta


def decompress_i8(values, meta, K: int, stream=None):
    import torch
    _require_cuda(values, meta)
    R = values.shape[0]
    out = torch.empty((R, K), dtype=torch.int8, device=values.device)
    nm_decompress_i8(values, meta, R, K, out, K, stream)
    return out


def spmm_i8(values, meta, K: int, X, stream=None):
    """Y = W' X (int32, exact) from the int8 2:4 operand and int8 X (K x T)."""
    import torch
    _require_cuda(values, meta, X)
    R, T = values.shape[0], X.shape[1]
    ld = max((T + 3) // 4 * 4, 4)
    Y = torch.empty((R, ld), dtype=torch.int32, device=X.device)
    nm_spmm_i8(values, meta, R, K, X, X.stride(0), T, Y, ld, stream)
    return Y[:, :T]


def prune_compress_tf32(W, stream=None):
    """1:2 (values R x K/2 float32, meta uint32 as int32) of float32 W (R x K), for the TF32 path."""
    import torch
    _require_cuda(W)
    R, K = W.shape
    vals = torch.empty((R, K // 2), dtype=torch.float32, device=W.device)
    meta = torch.empty((max(nm_meta_words(R, K, 1, 2), 0),), dtype=torch.int32, device=W.device)
    nm_prune_compress_tf32(W, R, K, W.stride(0), vals, meta, stream)
    return vals, meta


def decompress_tf32(values, meta, K: int, stream=None):
    import torch
    _require_cuda(values, meta)
    R = values.shape[0]
    out = torch.empty((R, K), dtype=torch.float32, device=values.device)
    nm_decompress_tf32(values, meta, R, K, out, K, stream)
    return out


def spmm_tf32(values, meta, K: int, X, out_dtype=None, stream=None):
    """Y = W' X from the 1:2 float32 operand and float32 X (K x T) on the TF32 tensor cores (fp32 by default)."""
    import torch
    _require_cuda(values, meta, X)
    out_dtype = torch.float32 if out_dtype is None else out_dtype
    R, T = values.shape[0], X.shape[1]
    per = 4 if out_dtype == torch.float32 else 8
    ld = max((T + per - 1) // per * per, per)
    Y = torch.empty((R, ld), dtype=out_dtype, device=X.device)
    nm_spmm_tf32(values, meta, R, K, X, X.stride(0), T, Y, ld,
                 NM_OUT_F32 if out_dtype == torch.float32 else NM_OUT_BF16, stream)
    return Y[:, :T]


def diag_prune_compress(W, D: int, stream=None):
    """(offsets int32[D] ascending, values D x R bf16) of the D highest-scoring diagonals of bf16 W (R x K)."""
    import torch
    _require_cuda(W)
    R, K = W.shape
    offsets = torch.empty((D,), dtype=torch.int32, device=W.device)
    values = torch.empty((D, R), dtype=torch.bfloat16, device=W.device)
    nm_diag_prune_compress(W, R, K, W.stride(0), D, offsets, values, stream)
    return offsets, values


def diag_spmm(values, offsets, K: int, X, idx=None, out_dtype=None, stream=None):
    import torch
    _require_cuda(values, offsets, X, idx)
    out_dtype = out_dtype or torch.bfloat16
    D, R = values.shape
    T = X.shape[1]
    per16 = 4 if out_dtype == torch.float32 else 8
    ld = max((T + per16 - 1) // per16 * per16, per16)
    Y = torch.empty((R, ld), dtype=out_dtype, device=X.device)
    yt = NM_OUT_F32 if out_dtype == torch.float32 else NM_OUT_BF16
    nm_diag_spmm(values, offsets, D, R, K, idx, X, X.stride(0), T, Y, ld, yt, stream)
    return Y[:, :T]
