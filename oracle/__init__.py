"""CPU oracle for the packed 1-bit / balanced-ternary matmul (numpy wrappers).

TEST INFRASTRUCTURE ONLY: imported by tests/, by __graft_entry__.smoke() and by
bench.py's CPU-baseline leg.  The product path (the CUDA library and its
binding) never imports this package, and this package never imports it.

Every function takes and returns host numpy arrays and calls the plain C++
definitions in bnn_oracle.cpp (built on first use by oracle/build.py).  Which
passage of the pages each definition follows is stated beside it there.
"""
from __future__ import annotations

import ctypes as C

import numpy as np

from .build import build as _build
from .build import build_k1 as _build_k1

_lib = None


def _L():
    global _lib
    if _lib is None:
        lib = C.CDLL(_build())
        i64, vp = C.c_int64, C.c_void_p
        sig = {
            "oracle_pack_signs": ([vp, i64, i64, vp], None),
            "oracle_unpack_signs": ([vp, i64, i64, vp], None),
            "oracle_count_pad_bits": ([vp, i64, i64], i64),
            "oracle_binary_gemm": ([vp, vp, vp, i64, i64, i64, vp, vp], None),
            "oracle_binary_gemm_sampled": ([vp, vp, vp, i64, i64, i64, vp, vp, i64, vp, vp], None),
            "oracle_binary_linear": ([vp, vp, vp, vp, i64, i64, i64, vp, vp, vp], None),
            "oracle_ternary_linear": ([vp, vp, vp, vp, i64, i64, i64, vp, vp], None),
            "oracle_sparse_count": ([vp, i64, i64, vp], i64),
            "oracle_sparse_encode": ([vp, i64, i64, vp, vp], None),
            "oracle_sparse_decode": ([vp, vp, i64, i64, vp], i64),
            "oracle_sparse_gemm": ([vp, vp, vp, vp, vp, i64, i64, i64, vp, vp], None),
            "oracle_twn_ternarize": ([vp, i64, i64, vp, vp, vp], None),
            "oracle_twn_delta": ([vp, i64], C.c_float),
            "oracle_absmean_ternarize": ([vp, i64, i64, vp, vp, vp], None),
            "oracle_absmean_apply": ([vp, i64, i64, C.c_float, vp, vp], None),
            "oracle_twn_apply": ([vp, i64, i64, C.c_float, vp, vp], None),
            "oracle_base3_pack": ([vp, i64, i64, vp], None),
            "oracle_base3_unpack": ([vp, i64, i64, vp], i64),
            "oracle_ternary_gemm": ([vp, vp, vp, i64, i64, i64, vp, vp], None),
            "oracle_ternary_gemm_sampled": ([vp, vp, vp, i64, i64, i64, vp, vp, i64, vp, vp], None),
        }
        for name, (args, res) in sig.items():
            f = getattr(lib, name)
            f.argtypes = args
            f.restype = res
        _lib = lib
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def words_per_row(k: int) -> int:
    return (k + 63) // 64


def trit_words_per_row(k: int) -> int:
    return (k + 9) // 10


def pack_signs(x: np.ndarray, k: int | None = None) -> np.ndarray:
    """fp32 [rows, k] -> uint64 [rows, ceil(k/64)]; bit 1 iff !(x > 0)."""
    x = _c(x, np.float32)
    x2 = x.reshape(-1, x.shape[-1]) if x.ndim > 1 else x.reshape(1, -1)
    rows, kk = x2.shape
    out = np.zeros((rows, words_per_row(kk)), dtype=np.uint64)
    _L().oracle_pack_signs(_p(x2), rows, kk, _p(out))
    return out


def unpack_signs(p: np.ndarray, k: int) -> np.ndarray:
    p = _c(p, np.uint64).reshape(-1, words_per_row(k)) if k else _c(p, np.uint64).reshape(-1, 0)
    out = np.zeros((p.shape[0], k), dtype=np.int8)
    _L().oracle_unpack_signs(_p(p), p.shape[0], k, _p(out))
    return out


def count_pad_bits(p: np.ndarray, k: int) -> int:
    p = _c(p, np.uint64)
    rows = p.shape[0] if p.ndim > 1 else 1
    return int(_L().oracle_count_pad_bits(_p(p), rows, k))


def binary_gemm(xp, wp, alpha, m: int, n: int, k: int):
    """Returns (dots int32 [m,n], out float32 [m,n])."""
    xp, wp, alpha = _c(xp, np.uint64), _c(wp, np.uint64), _c(alpha, np.float32)
    dots = np.zeros((m, n), dtype=np.int32)
    out = np.zeros((m, n), dtype=np.float32)
    _L().oracle_binary_gemm(_p(xp), _p(wp), _p(alpha), m, n, k, _p(dots), _p(out))
    return dots, out


def binary_gemm_sampled(xp, wp, alpha, m: int, n: int, k: int, rows, cols):
    xp, wp, alpha = _c(xp, np.uint64), _c(wp, np.uint64), _c(alpha, np.float32)
    rows, cols = _c(rows, np.int64), _c(cols, np.int64)
    assert rows.shape == cols.shape
    assert rows.size == 0 or (rows.min() >= 0 and rows.max() < m and cols.min() >= 0 and cols.max() < n)
    dots = np.zeros(rows.shape, dtype=np.int32)
    out = np.zeros(rows.shape, dtype=np.float32)
    _L().oracle_binary_gemm_sampled(_p(xp), _p(wp), _p(alpha), m, n, k, _p(rows), _p(cols),
                                    rows.size, _p(dots), _p(out))
    return dots, out


def binary_linear(xp, wp, alpha, bias, m: int, n: int, k: int):
    """One binarised layer: (dots int32 [m,n], y float32 [m,n], next uint64 [m, ceil(n/64)]),
    y = fl32(fl32(alpha*dot) + bias) (bias may be None), next = sign pack of y."""
    xp, wp, alpha = _c(xp, np.uint64), _c(wp, np.uint64), _c(alpha, np.float32)
    bias = None if bias is None else _c(bias, np.float32)
    dots = np.zeros((m, n), dtype=np.int32)
    y = np.zeros((m, n), dtype=np.float32)
    nxt = np.zeros((m, words_per_row(n)), dtype=np.uint64)
    _L().oracle_binary_linear(_p(xp), _p(wp), _p(alpha), _p(bias), m, n, k, _p(dots), _p(y), _p(nxt))
    return dots, y, nxt


def ternary_linear(x_bf16, packed, scale, bias, m: int, n: int, k: int):
    """Ternary layer with bias, float64: (y [m,n], mag [m,n])."""
    x_bf16, packed, scale = _c(x_bf16, np.uint16), _c(packed, np.uint16), _c(scale, np.float32)
    bias = None if bias is None else _c(bias, np.float32)
    y = np.zeros((m, n), dtype=np.float64)
    mag = np.zeros((m, n), dtype=np.float64)
    _L().oracle_ternary_linear(_p(x_bf16), _p(packed), _p(scale), _p(bias), m, n, k, _p(y), _p(mag))
    return y, mag


def sparse_encode(trits):
    """int8 trits [n,k] -> (row_ptr int64 [n+1], entries uint16 [nnz]): index + sign
    entries (position in bits 0..14, bit 15 for -1), rows in order."""
    trits = _c(trits, np.int8)
    n, k = trits.shape
    row_ptr = np.zeros(n + 1, dtype=np.int64)
    nnz = int(_L().oracle_sparse_count(_p(trits), n, k, _p(row_ptr)))
    entries = np.zeros(max(nnz, 1), dtype=np.uint16)
    _L().oracle_sparse_encode(_p(trits), n, k, _p(row_ptr), _p(entries))
    return row_ptr, entries[:nnz]


def sparse_decode(row_ptr, entries, n: int, k: int):
    """Inverse of sparse_encode: (trits int8 [n,k], count of malformed entries)."""
    row_ptr, entries = _c(row_ptr, np.int64), _c(entries, np.uint16)
    trits = np.zeros((n, k), dtype=np.int8)
    bad = _L().oracle_sparse_decode(_p(row_ptr), _p(entries if entries.size else np.zeros(1, np.uint16)), n, k,
                                    _p(trits))
    return trits, int(bad)


def sparse_gemm(x_bf16, row_ptr, entries, scale, bias, m: int, n: int, k: int):
    """Sparse ternary layer in float64: (y [m,n], mag [m,n])."""
    x_bf16, row_ptr, scale = _c(x_bf16, np.uint16), _c(row_ptr, np.int64), _c(scale, np.float32)
    entries = _c(entries, np.uint16) if len(entries) else np.zeros(1, np.uint16)
    bias = None if bias is None else _c(bias, np.float32)
    y = np.zeros((m, n), dtype=np.float64)
    mag = np.zeros((m, n), dtype=np.float64)
    _L().oracle_sparse_gemm(_p(x_bf16), _p(row_ptr), _p(entries), _p(scale), _p(bias), m, n, k, _p(y), _p(mag))
    return y, mag


def twn_ternarize(w: np.ndarray):
    """fp32 [n,k] -> (trits int8 [n,k], scale float32 [n], delta float32)."""
    w = _c(w, np.float32)
    n, k = w.shape
    trits = np.zeros((n, k), dtype=np.int8)
    scale = np.zeros(n, dtype=np.float32)
    delta = np.zeros(1, dtype=np.float32)
    _L().oracle_twn_ternarize(_p(w), n, k, _p(trits), _p(scale), _p(delta))
    return trits, scale, np.float32(delta[0])


def twn_delta(w: np.ndarray) -> np.float32:
    w = _c(w, np.float32)
    return np.float32(_L().oracle_twn_delta(_p(w), w.size))


def twn_apply(w: np.ndarray, delta) -> tuple:
    """Trits and least-squares scales for a given threshold Delta (float32)."""
    w = _c(w, np.float32)
    n, k = w.shape
    trits = np.zeros((n, k), dtype=np.int8)
    scale = np.zeros(n, dtype=np.float32)
    _L().oracle_twn_apply(_p(w), n, k, C.c_float(np.float32(delta)), _p(trits), _p(scale))
    return trits, scale


def absmean_ternarize(w: np.ndarray):
    """fp32 [n,k] -> (trits int8 [n,k], scale float32 [n], gamma float32)."""
    w = _c(w, np.float32)
    n, k = w.shape
    trits = np.zeros((n, k), dtype=np.int8)
    scale = np.zeros(n, dtype=np.float32)
    gamma = np.zeros(1, dtype=np.float32)
    _L().oracle_absmean_ternarize(_p(w), n, k, _p(trits), _p(scale), _p(gamma))
    return trits, scale, np.float32(gamma[0])


def absmean_apply(w: np.ndarray, gamma) -> tuple:
    """Mode 'absmean' at a given gamma (float32): (trits int8 [n,k], scale float32 [n])."""
    w = _c(w, np.float32)
    n, k = w.shape
    trits = np.zeros((n, k), dtype=np.int8)
    scale = np.zeros(n, dtype=np.float32)
    _L().oracle_absmean_apply(_p(w), n, k, C.c_float(np.float32(gamma)), _p(trits), _p(scale))
    return trits, scale


def delta_ternarize(w: np.ndarray, threshold) -> tuple:
    """Mode 'delta': a given threshold F and least-squares scales (twn_apply at F)."""
    return twn_apply(w, threshold)


def base3_pack(trits: np.ndarray) -> np.ndarray:
    trits = _c(trits, np.int8)
    n, k = trits.shape
    out = np.zeros((n, trit_words_per_row(k)), dtype=np.uint16)
    _L().oracle_base3_pack(_p(trits), n, k, _p(out))
    return out


def base3_unpack(packed: np.ndarray, k: int):
    """-> (trits int8 [n,k], number of words >= 3^10)."""
    packed = _c(packed, np.uint16)
    n = packed.shape[0]
    trits = np.zeros((n, k), dtype=np.int8)
    bad = _L().oracle_base3_unpack(_p(packed), n, k, _p(trits))
    return trits, int(bad)


def ternary_gemm(x_bf16, packed, scale, m: int, n: int, k: int):
    """Returns (y float64 [m,n], mag float64 [m,n])."""
    x_bf16, packed, scale = _c(x_bf16, np.uint16), _c(packed, np.uint16), _c(scale, np.float32)
    y = np.zeros((m, n), dtype=np.float64)
    mag = np.zeros((m, n), dtype=np.float64)
    _L().oracle_ternary_gemm(_p(x_bf16), _p(packed), _p(scale), m, n, k, _p(y), _p(mag))
    return y, mag


def ternary_gemm_sampled(x_bf16, packed, scale, m: int, n: int, k: int, rows, cols):
    x_bf16, packed, scale = _c(x_bf16, np.uint16), _c(packed, np.uint16), _c(scale, np.float32)
    rows, cols = _c(rows, np.int64), _c(cols, np.int64)
    assert rows.size == 0 or (rows.min() >= 0 and rows.max() < m and cols.min() >= 0 and cols.max() < n)
    y = np.zeros(rows.shape, dtype=np.float64)
    mag = np.zeros(rows.shape, dtype=np.float64)
    _L().oracle_ternary_gemm_sampled(_p(x_bf16), _p(packed), _p(scale), m, n, k, _p(rows), _p(cols),
                                     rows.size, _p(y), _p(mag))
    return y, mag


# ----------------------------------------------------------------------------
# CPU baseline (not the oracle): the pages' binary_gemm_u64 restated, XOR +
# 64-bit popcount row by row (k1_popcount.cpp).  Checked against the oracle by
# the tests; timed by the bench on one core and on all cores.
# ----------------------------------------------------------------------------
_k1 = None


def _K1():
    global _k1
    if _k1 is None:
        lib = C.CDLL(_build_k1())
        i64, vp = C.c_int64, C.c_void_p
        lib.k1_binary_gemm.argtypes = [vp, vp, vp, i64, i64, i64, C.c_int, vp, vp]
        lib.k1_binary_gemm.restype = None
        lib.k1_threads_used.argtypes = [C.c_int]
        lib.k1_threads_used.restype = C.c_int
        _k1 = lib
    return _k1


def k1_binary_gemm(xp, wp, alpha, m: int, n: int, k: int, threads: int = 1):
    """(dots int32 [m,n], out float32 [m,n]) by XOR + popcount, on `threads` OpenMP threads."""
    xp, wp, alpha = _c(xp, np.uint64), _c(wp, np.uint64), _c(alpha, np.float32)
    dots = np.zeros((m, n), dtype=np.int32)
    out = np.zeros((m, n), dtype=np.float32)
    _K1().k1_binary_gemm(_p(xp), _p(wp), _p(alpha), m, n, k, int(threads), _p(dots), _p(out))
    return dots, out


def k1_threads_used(threads: int) -> int:
    return int(_K1().k1_threads_used(int(threads)))
