"""The C-ABI library loads and exports every symbol include/bnn.h declares,
and its host-side argument checks reject bad calls before any CUDA work (these
calls never reach a kernel, so they run without a GPU)."""
import ctypes as C
import os
import re

import pytest

from conftest import ROOT

HEADER = os.path.join(ROOT, "include", "bnn.h")
HEADERS = [HEADER, os.path.join(ROOT, "include", "bnn_probe.h")]


def declared_symbols(paths=(HEADER,)):
    names = set()
    for path in paths:
        text = re.sub(r"/\*.*?\*/", "", open(path).read(), flags=re.S)
        names |= set(re.findall(r"\b(bnn_[a-z0-9_]+)\s*\(", text))
    return sorted(names)


@pytest.fixture(scope="module")
def bnn():
    from ternary_neural_net_b200 import bnn as mod
    return mod


def test_header_declares_the_four_calls():
    syms = declared_symbols()
    for name in ("bnn_pack_signs", "bnn_binary_gemm", "bnn_ternary_pack", "bnn_ternary_gemm",
                 "bnn_status_string", "bnn_last_cuda_error"):
        assert name in syms


def test_library_exports_every_declared_symbol(bnn):
    lib = C.CDLL(bnn.LIB_PATH)
    for name in declared_symbols(HEADERS):
        assert hasattr(lib, name), name
    assert set(bnn.ABI_SYMBOLS) <= set(declared_symbols())


def test_status_strings(bnn):
    lib = bnn.lib()
    for st in range(5):
        assert lib.bnn_status_string(st)
    assert b"INVALID" in lib.bnn_status_string(1)
    assert b"UNKNOWN" in lib.bnn_status_string(99)


def test_host_argument_checks(bnn):
    lib = bnn.lib()
    P = C.c_void_p
    good8 = P(0x1000)
    good2 = P(0x1002)
    # negative sizes
    assert lib.bnn_pack_signs(good8, -1, 5, good8, None) == bnn.BNN_ERR_INVALID_ARG
    assert lib.bnn_binary_gemm(good8, good8, good8, 1, 1, -3, good8, good8, None) == bnn.BNN_ERR_INVALID_ARG
    assert lib.bnn_ternary_pack(good8, -1, 3, good8, good8, good8, None) == bnn.BNN_ERR_INVALID_ARG
    assert lib.bnn_ternary_gemm(good8, good8, good8, 1, -1, 3, good8, None) == bnn.BNN_ERR_INVALID_ARG
    # k beyond the exact-float32 bound
    assert lib.bnn_binary_gemm(good8, good8, good8, 1, 1, (1 << 24) + 1, good8, None, None) == bnn.BNN_ERR_INVALID_ARG
    # no output at all / out without alpha
    assert lib.bnn_binary_gemm(good8, good8, good8, 1, 1, 64, None, None, None) == bnn.BNN_ERR_INVALID_ARG
    assert lib.bnn_binary_gemm(good8, good8, None, 1, 1, 64, None, good8, None) == bnn.BNN_ERR_INVALID_ARG
    # null required pointers
    assert lib.bnn_pack_signs(None, 2, 5, good8, None) == bnn.BNN_ERR_INVALID_ARG
    assert lib.bnn_ternary_gemm(None, good8, good8, 1, 1, 3, good8, None) == bnn.BNN_ERR_INVALID_ARG
    assert lib.bnn_ternary_pack(good8, 2, 3, good8, good8, None, None) == bnn.BNN_ERR_INVALID_ARG
    # misaligned pointers
    assert lib.bnn_pack_signs(P(0x1001), 2, 5, good8, None) == bnn.BNN_ERR_MISALIGNED
    assert lib.bnn_pack_signs(good8, 2, 5, P(0x1004), None) == bnn.BNN_ERR_MISALIGNED
    assert lib.bnn_binary_gemm(P(0x1004), good8, good8, 1, 1, 64, good8, None, None) == bnn.BNN_ERR_MISALIGNED
    assert lib.bnn_ternary_gemm(P(0x1001), good2, good8, 1, 1, 3, good8, None) == bnn.BNN_ERR_MISALIGNED
    assert lib.bnn_ternary_pack(good8, 1, 3, P(0x1001), good8, good8, None) == bnn.BNN_ERR_MISALIGNED
    # empty problems are valid and launch nothing
    assert lib.bnn_pack_signs(None, 0, 5, None, None) == bnn.BNN_OK
    assert lib.bnn_pack_signs(good8, 3, 0, good8, None) == bnn.BNN_OK
    assert lib.bnn_binary_gemm(None, None, None, 0, 5, 64, good8, None, None) == bnn.BNN_OK
    assert lib.bnn_ternary_gemm(None, None, None, 4, 0, 10, good8, None) == bnn.BNN_OK


def test_binding_rejects_host_tensors(bnn):
    import torch
    with pytest.raises(ValueError):
        bnn.bnn_pack_signs(torch.zeros(2, 3))


def test_binary_linear_host_checks(bnn):
    lib = bnn.lib()
    P = C.c_void_p
    g = P(0x1000)
    # no output at all; out or next without alpha
    assert lib.bnn_binary_linear(g, g, g, None, 1, 1, 64, None, None, None, None) == bnn.BNN_ERR_INVALID_ARG
    assert lib.bnn_binary_linear(g, g, None, None, 1, 1, 64, None, g, None, None) == bnn.BNN_ERR_INVALID_ARG
    assert lib.bnn_binary_linear(g, g, None, None, 1, 1, 64, None, None, g, None) == bnn.BNN_ERR_INVALID_ARG
    # dots alone need no alpha; sizes and k bound as for the GEMM
    assert lib.bnn_binary_linear(g, g, None, None, 1, -1, 64, g, None, None, None) == bnn.BNN_ERR_INVALID_ARG
    assert lib.bnn_binary_linear(g, g, g, None, 1, 1, (1 << 24) + 1, g, None, None, None) == bnn.BNN_ERR_INVALID_ARG
    # misaligned next (8 bytes) and bias (4 bytes)
    assert lib.bnn_binary_linear(g, g, g, None, 1, 1, 64, None, None, P(0x1004), None) == bnn.BNN_ERR_MISALIGNED
    assert lib.bnn_binary_linear(g, g, g, P(0x1002), 1, 1, 64, None, g, None, None) == bnn.BNN_ERR_MISALIGNED
    # empty problems launch nothing
    assert lib.bnn_binary_linear(None, None, None, None, 0, 7, 64, g, None, None, None) == bnn.BNN_OK
    assert lib.bnn_binary_linear(None, None, g, None, 3, 0, 64, None, None, g, None) == bnn.BNN_OK


def test_ternary_linear_host_checks(bnn):
    lib = bnn.lib()
    P = C.c_void_p
    g = P(0x1000)
    assert lib.bnn_ternary_linear(g, g, g, g, 1, -1, 3, g, None) == bnn.BNN_ERR_INVALID_ARG
    assert lib.bnn_ternary_linear(g, g, None, g, 1, 1, 3, g, None) == bnn.BNN_ERR_INVALID_ARG
    assert lib.bnn_ternary_linear(g, g, g, P(0x1002), 1, 1, 3, g, None) == bnn.BNN_ERR_MISALIGNED
    assert lib.bnn_ternary_linear(None, None, None, None, 0, 3, 3, g, None) == bnn.BNN_OK


def test_sparse_host_checks(bnn):
    lib = bnn.lib()
    P = C.c_void_p
    g = P(0x1000)
    assert lib.bnn_ternary_sparse_count(g, 2, (1 << 15) + 1, g, None) == bnn.BNN_ERR_INVALID_ARG
    assert lib.bnn_ternary_sparse_count(g, 2, 10, None, None) == bnn.BNN_ERR_INVALID_ARG
    assert lib.bnn_ternary_sparse_count(g, 2, 10, P(0x1004), None) == bnn.BNN_ERR_MISALIGNED
    assert lib.bnn_ternary_sparse_encode(g, 2, 10, g, None, None) == bnn.BNN_ERR_INVALID_ARG
    assert lib.bnn_ternary_sparse_encode(g, 2, 10, g, P(0x1001), None) == bnn.BNN_ERR_MISALIGNED
    assert lib.bnn_ternary_sparse_encode(None, 0, 10, g, None, None) == bnn.BNN_OK
    assert lib.bnn_ternary_sparse_gemm(g, g, g, g, None, 1, 1, -1, g, None) == bnn.BNN_ERR_INVALID_ARG
    assert lib.bnn_ternary_sparse_gemm(g, g, g, None, None, 1, 1, 10, g, None) == bnn.BNN_ERR_INVALID_ARG
    assert lib.bnn_ternary_sparse_gemm(g, g, g, g, P(0x1002), 1, 1, 10, g, None) == bnn.BNN_ERR_MISALIGNED
    assert lib.bnn_ternary_sparse_gemm(None, None, None, None, None, 0, 4, 10, None, None) == bnn.BNN_OK


def _plan(lib, n, k, active):
    f = lib.bnn_probe_ternary_plan
    f.argtypes = [C.c_int64, C.c_int64, C.POINTER(C.c_int), C.POINTER(C.c_int), C.POINTER(C.c_int)]
    f.restype = C.c_int
    act = (C.c_int * 4)(*active)
    rows, ks = C.c_int(0), C.c_int(0)
    st = f(n, k, act, C.byref(rows), C.byref(ks))
    return st, rows.value, ks.value


# clusters of 1..4 CTAs of the tensor-memory kernel that fit a 148-SM B200 at
# once (cudaOccupancyMaxActiveClusters on that GPU)
B200_ACTIVE = (148, 74, 45, 33)


def test_ternary_plan_cases(bnn):
    """The plan of the decode-into-tensor-memory ternary kernel: 115 CTAs of
    96 rows in one wave for the 11008 x 4096 layer (3-CTA clusters would need
    two waves); small layers split K over clusters; no split without clusters
    or without enough stages."""
    lib = bnn.lib()
    assert _plan(lib, 11008, 4096, B200_ACTIVE) == (bnn.BNN_OK, 96, 1)
    assert _plan(lib, 300, 4096, B200_ACTIVE) == (bnn.BNN_OK, 64, 4)
    assert _plan(lib, 385, 1288, B200_ACTIVE) == (bnn.BNN_OK, 64, 3)
    assert _plan(lib, 300, 4096, (148, 0, 0, 0)) == (bnn.BNN_OK, 64, 1)
    assert _plan(lib, 129, 8, B200_ACTIVE) == (bnn.BNN_OK, 64, 1)  # one stage: no split
    assert _plan(lib, 0, 4096, B200_ACTIVE)[0] == bnn.BNN_ERR_INVALID_ARG
    assert _plan(lib, 10, 0, B200_ACTIVE)[0] == bnn.BNN_ERR_INVALID_ARG


@pytest.mark.parametrize("n", [1, 31, 32, 97, 1000, 4096, 11008, 28672, 100000])
@pytest.mark.parametrize("k", [8, 640, 4096, 16384])
def test_ternary_plan_is_valid(bnn, n, k):
    lib = bnn.lib()
    st, rows, ks = _plan(lib, n, k, B200_ACTIVE)
    assert st == bnn.BNN_OK
    assert rows in (32, 64, 96, 128) and 1 <= ks <= 4
    stages = -(-k // 256)  # 256-trit stages up to trit k
    assert ks == 1 or stages >= 2 * ks  # every CTA of a split keeps at least two stages
