"""bnn_ternary_pack_noalloc: the TWN pack for callers that cannot allocate
device memory (a runtime that owns all device memory through its own
allocator, a setup without stream-ordered memory pools, a loop that cannot
risk an allocator call).  It keeps its partial sums in a fixed array inside
libbnn.so; this test calls it through the C ABI and checks it against the
allocating entry point bnn_ternary_pack on two calls in a row with different
inputs.  Both entry points run the same kernels in the same reduction order,
so words, scales and the threshold must be bitwise equal.  The file sorts last so that a run
stopping at the first failure has already run every other test."""
import ctypes as C

import numpy as np
import pytest
import torch

from ternary_neural_net_b200 import synth

pytestmark = pytest.mark.gpu

MAX_WEIGHTS = 1 << 29


def _entry(bnn):
    f = bnn.lib().bnn_ternary_pack_noalloc
    f.argtypes = [C.c_void_p, C.c_int64, C.c_int64, C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p]
    f.restype = C.c_int
    return f


def _ulps(a: torch.Tensor, b: torch.Tensor) -> int:
    ia = a.cpu().numpy().view(np.int32).astype(np.int64)
    ib = b.cpu().numpy().view(np.int32).astype(np.int64)
    return int(np.abs(ia - ib).max()) if ia.size else 0


def test_noalloc_matches_allocating_pack_twice(cuda_device):
    from ternary_neural_net_b200 import bnn
    f = _entry(bnn)
    stream = C.c_void_p(torch.cuda.current_stream().cuda_stream)
    # two calls in a row; the second is smaller, so slots left by the first
    # call must not leak into it
    for seed, (n, k) in ((1, (513, 4096 + 7)), (2, (37, 1000))):
        w = torch.from_numpy(synth.normal_f32(seed, 61, (n, k))).cuda()
        want_p, want_s, want_d = bnn.bnn_ternary_pack(w)
        p = torch.full_like(want_p, -1)
        s = torch.full_like(want_s, float("nan"))
        d = torch.full_like(want_d, float("nan"))
        st = f(C.c_void_p(w.data_ptr()), n, k, C.c_void_p(p.data_ptr()), C.c_void_p(s.data_ptr()),
               C.c_void_p(d.data_ptr()), stream)
        assert st == bnn.BNN_OK, bnn.lib().bnn_status_string(st)
        torch.cuda.synchronize()
        assert torch.equal(p, want_p)
        assert torch.equal(d, want_d)
        assert torch.equal(s, want_s), f"scales differ by up to {_ulps(s, want_s)} ulp"


def test_noalloc_rejects_sizes_beyond_its_array(cuda_device):
    from ternary_neural_net_b200 import bnn
    f = _entry(bnn)
    dummy = torch.zeros(4, dtype=torch.float32, device="cuda")
    n, k = 8193, 65536  # one partial sum more than the array holds
    assert n * k > MAX_WEIGHTS
    st = f(C.c_void_p(dummy.data_ptr()), n, k, C.c_void_p(dummy.data_ptr()), C.c_void_p(dummy.data_ptr()),
           C.c_void_p(dummy.data_ptr()), None)
    assert st == bnn.BNN_ERR_INVALID_ARG
