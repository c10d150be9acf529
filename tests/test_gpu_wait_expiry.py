"""Failure detection on the GPU without a fault: the tensor-core binary GEMMs
(the one-SM tile kernel and the persistent CTA-pair kernel) bound every
mbarrier wait.  With the main waits cut to a few polls
(bnn_probe_wait_limit), they run out before the first copies land.  The
kernel must then count the run-out (bnn_device_error_count, read on the
host), skip every store (the outputs keep their sentinel values), wait for
its own copies and MMAs, free its tensor memory and return normally, so the
call still reports BNN_OK and the context stays usable: the next normal call
on the same process is bit-exact against the oracle."""
import ctypes as C

import numpy as np
import pytest
import torch

import oracle
from gpu_util import to_dev_f32, to_dev_u64
from ternary_neural_net_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bnn(cuda_device):
    from ternary_neural_net_b200 import bnn as mod
    return mod


def _limit(bnn, polls):
    f = bnn.lib().bnn_probe_wait_limit
    f.argtypes = [C.c_uint32]
    f.restype = C.c_int
    assert f(polls) == bnn.BNN_OK


def test_main_waits_run_out_then_a_normal_call_is_exact(bnn):
    # one 128 x 64 tile, 4 stages, no split K (the single-CTA path), TMA-fed
    m, n, k = 64, 128, 512
    xp = synth.fair_coin_words(3, 1, m, k)
    wp = synth.fair_coin_words(3, 2, n, k)
    alpha = synth.uniform_f32(3, 3, (n,), 0.5, 1.5)
    xd, wd, ad = to_dev_u64(xp), to_dev_u64(wp), to_dev_f32(alpha)
    torch.cuda.synchronize()
    bnn.device_error_count(reset=True)
    dots = torch.full((m, n), -7, dtype=torch.int32, device="cuda")
    out = torch.full((m, n), float("nan"), dtype=torch.float32, device="cuda")
    _limit(bnn, 4)
    try:
        bnn.bnn_binary_gemm(xd, wd, ad, k, dots=dots, out=out, algo=bnn.ALGO_TC)
        torch.cuda.synchronize()
    finally:
        _limit(bnn, 0)
    ran_out = bnn.device_error_count(reset=True)
    assert ran_out > 0, "no wait ran out"
    assert torch.all(dots == -7), "an aborted CTA stored dots"
    assert torch.all(torch.isnan(out)), "an aborted CTA stored outputs"

    want_d, want_o = oracle.binary_gemm(xp, wp, alpha, m, n, k)
    d2, o2 = bnn.bnn_binary_gemm(xd, wd, ad, k, algo=bnn.ALGO_TC)
    assert np.array_equal(d2.cpu().numpy(), want_d)
    assert np.array_equal(o2.cpu().numpy().view(np.uint32), want_o.view(np.uint32))
    assert bnn.device_error_count() == 0


def test_pair_kernel_waits_run_out_then_a_normal_call_is_exact(bnn):
    # the persistent CTA-pair kernel (two waves of 256 x 224 pair tiles: m = 256, n = 148 x 256);
    # its epilogue warps wait for a tile that never comes, up to their one-second bound
    m, n, k = 256, 148 * 256, 128
    xp = synth.fair_coin_words(4, 1, m, k)
    wp = synth.fair_coin_words(4, 2, n, k)
    alpha = synth.uniform_f32(4, 3, (n,), 0.5, 1.5)
    xd, wd, ad = to_dev_u64(xp), to_dev_u64(wp), to_dev_f32(alpha)
    torch.cuda.synchronize()
    bnn.device_error_count(reset=True)
    dots = torch.full((m, n), -7, dtype=torch.int32, device="cuda")
    out = torch.full((m, n), float("nan"), dtype=torch.float32, device="cuda")
    _limit(bnn, 4)
    try:
        bnn.bnn_binary_gemm(xd, wd, ad, k, dots=dots, out=out, algo=bnn.ALGO_TC)
        torch.cuda.synchronize()
    finally:
        _limit(bnn, 0)
    ran_out = bnn.device_error_count(reset=True)
    assert ran_out > 0, "no wait ran out"
    assert torch.all(dots == -7), "an aborted pair stored dots"
    assert torch.all(torch.isnan(out)), "an aborted pair stored outputs"

    rows = np.arange(0, m, 37)
    want_d, want_o = oracle.binary_gemm(xp[rows], wp, alpha, len(rows), n, k)
    d2, o2 = bnn.bnn_binary_gemm(xd, wd, ad, k, algo=bnn.ALGO_TC)
    assert np.array_equal(d2.cpu().numpy()[rows], want_d)
    assert np.array_equal(o2.cpu().numpy()[rows].view(np.uint32), want_o.view(np.uint32))
    assert bnn.device_error_count() == 0
