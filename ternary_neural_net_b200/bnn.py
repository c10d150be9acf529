"""Python binding of libbnn (the C ABI declared in include/bnn.h).

Argument marshalling only: every function checks shapes and dtypes, allocates
outputs with PyTorch when the caller does not pass them, and calls the
library entry point of the same name with raw device pointers and the current
CUDA stream.  Every step of the computation runs in the library's kernels;
there is no fallback.  Importing this module loads libbnn.so and raises
ImportError when it is missing (build it with
``python -m ternary_neural_net_b200.build``).

dtype conventions (PyTorch has no general-purpose unsigned tensors, so the
unsigned words travel in signed tensors of the same width, bit for bit):
  packed sign words   torch.int64  [rows, ceil(k/64)]   (uint64 in the ABI)
  base-3 trit words   torch.int16  [n, ceil(k/10)]      (uint16 in the ABI)
  bf16 activations    torch.bfloat16 [m, k]             (uint16 bit patterns in the ABI)
"""
from __future__ import annotations

import ctypes as C
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libbnn.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"libbnn.so not found at {LIB_PATH}; build it with "
                      "`python -m ternary_neural_net_b200.build` (needs nvcc)")
_lib = C.CDLL(LIB_PATH)

_vp, _i64, _int = C.c_void_p, C.c_int64, C.c_int
_SIGS = {
    "bnn_pack_signs": [_vp, _i64, _i64, _vp, _vp],
    "bnn_binary_gemm": [_vp, _vp, _vp, _i64, _i64, _i64, _vp, _vp, _vp],
    "bnn_binary_gemm_algo": [_vp, _vp, _vp, _i64, _i64, _i64, _vp, _vp, _int, _vp],
    "bnn_binary_linear": [_vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp, _vp, _vp, _vp],
    "bnn_ternary_pack": [_vp, _i64, _i64, _vp, _vp, _vp, _vp],
    "bnn_ternary_gemm": [_vp, _vp, _vp, _i64, _i64, _i64, _vp, _vp],
    "bnn_ternary_pack_mode": [_vp, _i64, _i64, _int, C.c_float, _vp, _vp, _vp, _vp],
    "bnn_ternary_gemm_algo": [_vp, _vp, _vp, _i64, _i64, _i64, _vp, _int, _vp],
    "bnn_ternary_pack_noalloc": [_vp, _i64, _i64, _vp, _vp, _vp, _vp],
    "bnn_ternary_linear": [_vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp, _vp],
    "bnn_ternary_sparse_count": [_vp, _i64, _i64, _vp, _vp],
    "bnn_ternary_sparse_encode": [_vp, _i64, _i64, _vp, _vp, _vp],
    "bnn_ternary_sparse_gemm": [_vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp, _vp],
}
class TbinRecord(C.Structure):
    """bnn_tbin_record (include/bnn.h)."""
    _fields_ = [("kind", C.c_uint32), ("name_len", C.c_uint32), ("name_offset", C.c_uint64),
                ("out_features", C.c_uint32), ("in_features", C.c_uint32), ("delta", C.c_float),
                ("sparsity", C.c_float), ("num_biases", C.c_uint32), ("reserved", C.c_uint32),
                ("scales_offset", C.c_uint64), ("biases_offset", C.c_uint64), ("weights_offset", C.c_uint64),
                ("weights_words", C.c_uint64), ("ndims", C.c_uint32), ("dims", C.c_uint32 * 8),
                ("data_offset", C.c_uint64), ("data_elems", C.c_uint64)]


_SIGS.update({
    "bnn_tbin_parse": [_vp, C.c_uint64, _vp, _vp, _vp, _vp, _i64, _vp],
    "bnn_tbin_load_ternary": [_vp, C.c_uint64, _vp, _vp, _vp, _vp, _vp],
    "bnn_tbin_load_raw": [_vp, C.c_uint64, _vp, _vp, _vp],
})

for _name, _args in _SIGS.items():
    _f = getattr(_lib, _name)
    _f.argtypes = _args
    _f.restype = _int
_lib.bnn_status_string.argtypes = [_int]
_lib.bnn_status_string.restype = C.c_char_p
_lib.bnn_last_cuda_error.argtypes = []
_lib.bnn_last_cuda_error.restype = _int
_lib.bnn_device_error_count.argtypes = [_int]
_lib.bnn_device_error_count.restype = _int

# Exported symbol names, as declared in include/bnn.h.
ABI_SYMBOLS = tuple(_SIGS) + ("bnn_status_string", "bnn_last_cuda_error", "bnn_device_error_count")


def device_error_count(reset: bool = False) -> int:
    """Bounded device-side waits that ran out since the last reset (0 when all is well)."""
    return int(_lib.bnn_device_error_count(1 if reset else 0))

BNN_OK, BNN_ERR_INVALID_ARG, BNN_ERR_MISALIGNED, BNN_ERR_CUDA, BNN_ERR_UNSUPPORTED = range(5)
ALGO_AUTO, ALGO_POPC, ALGO_MMA_S8, ALGO_TC = 0, 1, 2, 3
TERNARY_TWN, TERNARY_ABSMEAN, TERNARY_DELTA = 0, 1, 2
TALGO_AUTO, TALGO_CUDA_CORES, TALGO_MMA, TALGO_TC = 0, 1, 2, 3
MAX_K_BINARY = 1 << 24
MAX_K_SPARSE = 1 << 15


class BnnError(RuntimeError):
    def __init__(self, status: int, call: str):
        msg = _lib.bnn_status_string(status).decode()
        if status == BNN_ERR_CUDA:
            msg += f" (cudaError {_lib.bnn_last_cuda_error()})"
        super().__init__(f"{call}: {msg}")
        self.status = status


def lib() -> C.CDLL:
    """The loaded libbnn handle (for raw-pointer calls)."""
    return _lib


def _check(st: int, call: str):
    if st != BNN_OK:
        raise BnnError(st, call)


def _ptr(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def _stream(device):
    return C.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _dev(t: torch.Tensor, name: str, dtype=None, ndim=2):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must be {ndim}-D, got shape {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def words_per_row(k: int) -> int:
    return (k + 63) // 64


def trit_words_per_row(k: int) -> int:
    return (k + 9) // 10


def bnn_pack_signs(x: torch.Tensor, out: torch.Tensor | None = None) -> torch.Tensor:
    """float32 [rows, k] -> packed int64 [rows, ceil(k/64)] (bit 1 iff !(x > 0))."""
    _dev(x, "x", torch.float32)
    rows, k = x.shape
    if out is None:
        out = torch.empty((rows, words_per_row(k)), dtype=torch.int64, device=x.device)
    else:
        _dev(out, "out", torch.int64)
        if tuple(out.shape) != (rows, words_per_row(k)):
            raise ValueError("out has the wrong shape")
    _check(_lib.bnn_pack_signs(_ptr(x), rows, k, _ptr(out), _stream(x.device)), "bnn_pack_signs")
    return out


def bnn_binary_gemm(xp: torch.Tensor, wp: torch.Tensor, alpha: torch.Tensor | None, k: int,
                    want_dots: bool = True, want_out: bool = True,
                    dots: torch.Tensor | None = None, out: torch.Tensor | None = None, algo: int = ALGO_AUTO):
    """Packed XOR+popcount matmul.  Returns (dots int32 [m,n] or None, out float32 [m,n] or None).
    `algo` selects the kernel family (ALGO_AUTO, ALGO_POPC, ALGO_MMA_S8, ALGO_TC); all are bit-identical."""
    _dev(xp, "xp", torch.int64)
    _dev(wp, "wp", torch.int64)
    m, n = xp.shape[0], wp.shape[0]
    if xp.shape[1] != words_per_row(k) or wp.shape[1] != words_per_row(k):
        raise ValueError("packed rows must hold ceil(k/64) words")
    dev = xp.device
    if want_dots and dots is None:
        dots = torch.empty((m, n), dtype=torch.int32, device=dev)
    if want_out and out is None:
        out = torch.empty((m, n), dtype=torch.float32, device=dev)
    if dots is not None:
        _dev(dots, "dots", torch.int32)
    if out is not None:
        _dev(out, "out", torch.float32)
        _dev(alpha, "alpha", torch.float32, ndim=1)
    if algo == ALGO_AUTO:
        st = _lib.bnn_binary_gemm(_ptr(xp), _ptr(wp), _ptr(alpha), m, n, k, _ptr(dots), _ptr(out), _stream(dev))
    else:
        st = _lib.bnn_binary_gemm_algo(_ptr(xp), _ptr(wp), _ptr(alpha), m, n, k, _ptr(dots), _ptr(out),
                                       int(algo), _stream(dev))
    _check(st, "bnn_binary_gemm")
    return dots, out


def bnn_binary_linear(xp: torch.Tensor, wp: torch.Tensor, alpha: torch.Tensor | None,
                      bias: torch.Tensor | None, k: int, want_dots: bool = False, want_out: bool = True,
                      want_next: bool = True, dots: torch.Tensor | None = None,
                      out: torch.Tensor | None = None, nxt: torch.Tensor | None = None):
    """One binarised layer with the fused epilogue: returns (dots int32 [m,n] or None,
    y float32 [m,n] or None, next int64 [m, ceil(n/64)] or None), y = alpha*dot (+ bias),
    next = the sign pack of y (the next layer's packed input)."""
    _dev(xp, "xp", torch.int64)
    _dev(wp, "wp", torch.int64)
    m, n = xp.shape[0], wp.shape[0]
    if xp.shape[1] != words_per_row(k) or wp.shape[1] != words_per_row(k):
        raise ValueError("packed rows must hold ceil(k/64) words")
    dev = xp.device
    if want_dots and dots is None:
        dots = torch.empty((m, n), dtype=torch.int32, device=dev)
    if want_out and out is None:
        out = torch.empty((m, n), dtype=torch.float32, device=dev)
    if want_next and nxt is None:
        nxt = torch.empty((m, words_per_row(n)), dtype=torch.int64, device=dev)
    if dots is not None:
        _dev(dots, "dots", torch.int32)
    if out is not None:
        _dev(out, "out", torch.float32)
    if nxt is not None:
        _dev(nxt, "next", torch.int64)
    if out is not None or nxt is not None:
        _dev(alpha, "alpha", torch.float32, ndim=1)
    if bias is not None:
        _dev(bias, "bias", torch.float32, ndim=1)
    _check(_lib.bnn_binary_linear(_ptr(xp), _ptr(wp), _ptr(alpha), _ptr(bias), m, n, k, _ptr(dots), _ptr(out),
                                  _ptr(nxt), _stream(dev)), "bnn_binary_linear")
    return dots, out, nxt


def bnn_ternary_sparse_encode(packed: torch.Tensor, k: int):
    """Base-3 packed [n, ceil(k/10)] -> (row_ptr int64 [n+1], entries int16 [nnz]) of the index +
    sign sparse form.  An offline weight-preparation step: it reads the entry count back from
    the device between its two kernels, and synchronises the stream again after the encode, so
    the returned tensors are complete when it returns (the sparse matmul reads its weight
    operands before waiting for the kernel ahead of it; see "Weights are static data" in bnn.h)."""
    _dev(packed, "packed", torch.int16)
    n = packed.shape[0]
    if packed.shape[1] != trit_words_per_row(k):
        raise ValueError("packed rows must hold ceil(k/10) words")
    dev = packed.device
    row_ptr = torch.empty((n + 1,), dtype=torch.int64, device=dev)
    _check(_lib.bnn_ternary_sparse_count(_ptr(packed), n, k, _ptr(row_ptr), _stream(dev)), "bnn_ternary_sparse_count")
    nnz = int(row_ptr[n].item())
    entries = torch.empty((max(nnz, 1),), dtype=torch.int16, device=dev)
    _check(_lib.bnn_ternary_sparse_encode(_ptr(packed), n, k, _ptr(row_ptr), _ptr(entries), _stream(dev)),
           "bnn_ternary_sparse_encode")
    torch.cuda.current_stream(dev).synchronize()
    return row_ptr, entries[:nnz]


def bnn_ternary_sparse_gemm(x: torch.Tensor, row_ptr: torch.Tensor, entries: torch.Tensor, scale: torch.Tensor,
                            bias: torch.Tensor | None = None, out: torch.Tensor | None = None) -> torch.Tensor:
    """bf16 [m, k] x sparse ternary [n, k] -> float32 [m, n] (scale and bias applied)."""
    _dev(x, "x", torch.bfloat16)
    _dev(row_ptr, "row_ptr", torch.int64, ndim=1)
    _dev(scale, "scale", torch.float32, ndim=1)
    m, k = x.shape
    n = row_ptr.shape[0] - 1
    if bias is not None:
        _dev(bias, "bias", torch.float32, ndim=1)
    if out is None:
        out = torch.empty((m, n), dtype=torch.float32, device=x.device)
    _dev(out, "out", torch.float32)
    ent = _ptr(entries) if entries.numel() else None
    _check(_lib.bnn_ternary_sparse_gemm(_ptr(x), _ptr(row_ptr), ent, _ptr(scale), _ptr(bias), m, n, k, _ptr(out),
                                        _stream(x.device)), "bnn_ternary_sparse_gemm")
    return out


def bnn_tbin_parse(data: bytes):
    """Parse a .tbin file held in host memory: (version, metadata bytes, [TbinRecord, ...])."""
    buf = C.create_string_buffer(bytes(data), len(data))
    ver, moff, mlen, count = C.c_uint32(), C.c_uint64(), C.c_uint64(), C.c_int64()
    _check(_lib.bnn_tbin_parse(buf, len(data), C.byref(ver), C.byref(moff), C.byref(mlen), None, 0,
                               C.byref(count)), "bnn_tbin_parse")
    recs = (TbinRecord * max(count.value, 1))()
    _check(_lib.bnn_tbin_parse(buf, len(data), None, None, None, recs, count.value, C.byref(count)),
           "bnn_tbin_parse")
    meta = bytes(data[moff.value:moff.value + mlen.value])
    return ver.value, meta, [recs[i] for i in range(count.value)]


def tbin_record_name(data: bytes, rec: TbinRecord) -> str:
    return bytes(data[rec.name_offset:rec.name_offset + rec.name_len]).decode()


def bnn_tbin_load_ternary(file_dev: torch.Tensor, rec: TbinRecord):
    """A ternary record from the file's bytes on the device (uint8 tensor) ->
    (packed int16 [out, ceil(in/10)], scale float32 [out], bias float32 [out] or None)."""
    _dev(file_dev, "file", torch.uint8, ndim=1)
    dev = file_dev.device
    out_f, kt = rec.out_features, trit_words_per_row(rec.in_features)
    packed = torch.empty((out_f, kt), dtype=torch.int16, device=dev)
    scale = torch.empty((out_f,), dtype=torch.float32, device=dev)
    bias = torch.empty((out_f,), dtype=torch.float32, device=dev) if rec.num_biases else None
    _check(_lib.bnn_tbin_load_ternary(_ptr(file_dev), file_dev.numel(), C.byref(rec), _ptr(packed), _ptr(scale),
                                      _ptr(bias), _stream(dev)), "bnn_tbin_load_ternary")
    return packed, scale, bias


def bnn_tbin_load_raw(file_dev: torch.Tensor, rec: TbinRecord) -> torch.Tensor:
    """A raw float16 record from the file's bytes on the device -> float32 tensor of its dims."""
    _dev(file_dev, "file", torch.uint8, ndim=1)
    out = torch.empty((int(rec.data_elems),), dtype=torch.float32, device=file_dev.device)
    _check(_lib.bnn_tbin_load_raw(_ptr(file_dev), file_dev.numel(), C.byref(rec), _ptr(out),
                                  _stream(file_dev.device)), "bnn_tbin_load_raw")
    return out.view(*[int(rec.dims[d]) for d in range(rec.ndims)]) if rec.ndims else out


def bnn_ternary_pack(w: torch.Tensor, packed: torch.Tensor | None = None,
                     scale: torch.Tensor | None = None, delta: torch.Tensor | None = None):
    """float32 [n, k] -> (packed int16 [n, ceil(k/10)], scale float32 [n], delta float32 [1])."""
    _dev(w, "w", torch.float32)
    n, k = w.shape
    dev = w.device
    if packed is None:
        packed = torch.empty((n, trit_words_per_row(k)), dtype=torch.int16, device=dev)
    if scale is None:
        scale = torch.empty((n,), dtype=torch.float32, device=dev)
    if delta is None:
        delta = torch.empty((1,), dtype=torch.float32, device=dev)
    _dev(packed, "packed", torch.int16)
    _dev(scale, "scale", torch.float32, ndim=1)
    _dev(delta, "delta", torch.float32, ndim=1)
    _check(_lib.bnn_ternary_pack(_ptr(w), n, k, _ptr(packed), _ptr(scale), _ptr(delta), _stream(dev)),
           "bnn_ternary_pack")
    return packed, scale, delta


def bnn_ternary_pack_mode(w: torch.Tensor, mode: int, threshold: float = 0.0):
    """Ternarise with TERNARY_TWN / TERNARY_ABSMEAN / TERNARY_DELTA (threshold = F).
    Returns (packed int16 [n, ceil(k/10)], scale float32 [n], threshold used float32 [1])."""
    _dev(w, "w", torch.float32)
    n, k = w.shape
    dev = w.device
    packed = torch.empty((n, trit_words_per_row(k)), dtype=torch.int16, device=dev)
    scale = torch.empty((n,), dtype=torch.float32, device=dev)
    thresh = torch.empty((1,), dtype=torch.float32, device=dev)
    _check(_lib.bnn_ternary_pack_mode(_ptr(w), n, k, int(mode), float(threshold), _ptr(packed), _ptr(scale),
                                      _ptr(thresh), _stream(dev)), "bnn_ternary_pack_mode")
    return packed, scale, thresh


def bnn_ternary_gemm(x: torch.Tensor, packed: torch.Tensor, scale: torch.Tensor, k: int | None = None,
                     out: torch.Tensor | None = None, algo: int = TALGO_AUTO) -> torch.Tensor:
    """bf16 [m, k] x base-3 packed [n, ceil(k/10)] -> float32 [m, n] (scale applied).
    `algo` selects the kernel family (TALGO_AUTO, TALGO_CUDA_CORES, TALGO_MMA, TALGO_TC)."""
    _dev(x, "x", torch.bfloat16)
    _dev(packed, "packed", torch.int16)
    _dev(scale, "scale", torch.float32, ndim=1)
    m, kk = x.shape
    k = kk if k is None else k
    if k != kk or packed.shape[1] != trit_words_per_row(k):
        raise ValueError("packed rows must hold ceil(k/10) words")
    n = packed.shape[0]
    if out is None:
        out = torch.empty((m, n), dtype=torch.float32, device=x.device)
    _dev(out, "out", torch.float32)
    if algo == TALGO_AUTO:
        st = _lib.bnn_ternary_gemm(_ptr(x), _ptr(packed), _ptr(scale), m, n, k, _ptr(out), _stream(x.device))
    else:
        st = _lib.bnn_ternary_gemm_algo(_ptr(x), _ptr(packed), _ptr(scale), m, n, k, _ptr(out), int(algo),
                                        _stream(x.device))
    _check(st, "bnn_ternary_gemm")
    return out


def bnn_ternary_linear(x: torch.Tensor, packed: torch.Tensor, scale: torch.Tensor, bias: torch.Tensor | None,
                       out: torch.Tensor | None = None) -> torch.Tensor:
    """bnn_ternary_gemm plus the per-channel bias: float32 [m, n]."""
    _dev(x, "x", torch.bfloat16)
    _dev(packed, "packed", torch.int16)
    _dev(scale, "scale", torch.float32, ndim=1)
    m, k = x.shape
    if packed.shape[1] != trit_words_per_row(k):
        raise ValueError("packed rows must hold ceil(k/10) words")
    n = packed.shape[0]
    if bias is not None:
        _dev(bias, "bias", torch.float32, ndim=1)
    if out is None:
        out = torch.empty((m, n), dtype=torch.float32, device=x.device)
    _dev(out, "out", torch.float32)
    _check(_lib.bnn_ternary_linear(_ptr(x), _ptr(packed), _ptr(scale), _ptr(bias), m, n, k, _ptr(out),
                                   _stream(x.device)), "bnn_ternary_linear")
    return out
