"""GPU parity of the fused layer epilogue (bnn_binary_linear): int32 dots,
y = fl32(fl32(alpha*dot) + bias) bitwise, and the next layer's packed input
bit-exact, against the oracle, on every tensor-core configuration and on a
chained two-layer stack at the headline size.  Every call goes through the C ABI
via the binding."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import assert_bits_equal, host_u64, to_dev_f32, to_dev_u64
from ternary_neural_net_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bnn(cuda_device):
    from ternary_neural_net_b200 import bnn as mod
    return mod


def _case(seed, m, n, k):
    xp = synth.fair_coin_words(seed, 1, m, k)
    wp = synth.fair_coin_words(seed, 2, n, k)
    alpha = synth.uniform_f32(seed, 3, (n,), -1.0, 2.0)
    bias = (synth.normal_f32(seed, 4, (n,)) * np.float32(8.0)).astype(np.float32)
    return xp, wp, alpha, bias


# every tensor-core configuration (64-row tiles with 1/2/4-CTA split K, 256-row
# tiles, TMA and plain loads), small m, and n off the 64- and 32-bit boundaries
@pytest.mark.parametrize("m,n,k", [(1, 100, 640), (5, 64, 64), (40, 300, 2048 + 37), (64, 1000, 1000),
                                   (100, 500, 4096), (128, 129, 1100), (70, 9600, 512), (257, 383, 4160),
                                   (600, 9000, 760), (2304, 4219, 130), (33, 31, 3000), (2304, 4219, 128)])
@pytest.mark.parametrize("with_bias", [True, False])
def test_linear_matches_oracle(bnn, m, n, k, with_bias):
    xp, wp, alpha, bias = _case(m + 3 * n + k, m, n, k)
    b = bias if with_bias else None
    want_d, want_y, want_next = oracle.binary_linear(xp, wp, alpha, b, m, n, k)
    d, y, nxt = bnn.bnn_binary_linear(to_dev_u64(xp), to_dev_u64(wp), to_dev_f32(alpha),
                                      to_dev_f32(b) if with_bias else None, k, want_dots=True)
    torch.cuda.synchronize()
    assert_bits_equal(d.cpu().numpy(), want_d, f"dots {m}x{n}x{k}")
    assert_bits_equal(y.cpu().numpy(), want_y, f"y {m}x{n}x{k}")
    assert_bits_equal(host_u64(nxt), want_next, f"next {m}x{n}x{k}")
    assert oracle.count_pad_bits(host_u64(nxt), n) == 0


def test_linear_outputs_are_independent(bnn):
    """next alone, out alone and dots alone give the same values as all three."""
    m, n, k = 70, 257, 700
    xp, wp, alpha, bias = _case(7, m, n, k)
    want_d, want_y, want_next = oracle.binary_linear(xp, wp, alpha, bias, m, n, k)
    args = (to_dev_u64(xp), to_dev_u64(wp), to_dev_f32(alpha), to_dev_f32(bias), k)
    _, _, nxt = bnn.bnn_binary_linear(*args, want_dots=False, want_out=False, want_next=True)
    assert_bits_equal(host_u64(nxt), want_next, "next only")
    _, y, _ = bnn.bnn_binary_linear(*args, want_dots=False, want_out=True, want_next=False)
    assert_bits_equal(y.cpu().numpy(), want_y, "out only")
    d, _, _ = bnn.bnn_binary_linear(to_dev_u64(xp), to_dev_u64(wp), None, None, k, want_dots=True,
                                    want_out=False, want_next=False)
    assert_bits_equal(d.cpu().numpy(), want_d, "dots only")


def test_linear_zero_crossings_pack_as_minus_one(bnn):
    """A bias that cancels y exactly gives +0, which packs to bit 1 (0 is not > 0)."""
    m, n, k = 9, 130, 256
    xp, wp, alpha, _ = _case(8, m, n, k)
    _, y0, _ = oracle.binary_linear(xp, wp, alpha, None, m, n, k)
    bias = -y0[3].copy()
    want_d, want_y, want_next = oracle.binary_linear(xp, wp, alpha, bias, m, n, k)
    _, y, nxt = bnn.bnn_binary_linear(to_dev_u64(xp), to_dev_u64(wp), to_dev_f32(alpha), to_dev_f32(bias), k)
    assert_bits_equal(y.cpu().numpy(), want_y, "y")
    assert_bits_equal(host_u64(nxt), want_next, "next")
    assert np.all(y.cpu().numpy()[3] == 0.0)


def test_linear_k_zero(bnn):
    m, n = 3, 70
    alpha = synth.uniform_f32(9, 3, (n,), 0.5, 1.5)
    bias = synth.normal_f32(9, 4, (n,))
    xp = torch.empty((m, 0), dtype=torch.int64, device="cuda")
    wp = torch.empty((n, 0), dtype=torch.int64, device="cuda")
    want_d, want_y, want_next = oracle.binary_linear(np.zeros((m, 0), np.uint64), np.zeros((n, 0), np.uint64),
                                                     alpha, bias, m, n, 0)
    d, y, nxt = bnn.bnn_binary_linear(xp, wp, to_dev_f32(alpha), to_dev_f32(bias), 0, want_dots=True)
    assert_bits_equal(d.cpu().numpy(), want_d, "dots")
    assert_bits_equal(y.cpu().numpy(), want_y, "y")
    assert_bits_equal(host_u64(nxt), want_next, "next")


def test_two_layer_stack_headline_size(bnn):
    """Layer 1 (256 x 4096 x 4096, bias) packs its output as layer 2's input;
    layer 2 (4096 -> 4096) consumes it.  Checked on sampled outputs plus the
    whole packed intermediate against the oracle's pack of layer 1's y."""
    m, n, k = 256, 4096, 4096
    c = synth.gemm_fused_pack(1)
    w1 = bnn.bnn_pack_signs(to_dev_f32(c["w"]))
    torch.cuda.synchronize()  # weights are complete before a matmul reads them
    x = bnn.bnn_pack_signs(to_dev_f32(c["x"]))
    w2p = synth.fair_coin_words(11, 2, n, n)
    b1 = synth.normal_f32(11, 5, (n,))
    a2 = synth.uniform_f32(11, 6, (n,), 0.5, 1.5)
    _, y1, h = bnn.bnn_binary_linear(x, w1, to_dev_f32(c["alpha"]), to_dev_f32(b1), k)
    d2, y2, _ = bnn.bnn_binary_linear(h, to_dev_u64(w2p), to_dev_f32(a2), None, n, want_dots=True,
                                      want_next=False)
    torch.cuda.synchronize()
    hx, hw = host_u64(x), host_u64(w1)
    # layer 1 on sampled rows, in full along n, then its pack
    rows = np.array([0, 1, 77, 255])
    _, y1r, nr = oracle.binary_linear(hx[rows], hw, c["alpha"], b1, len(rows), n, k)
    assert_bits_equal(y1.cpu().numpy()[rows], y1r, "layer 1 y")
    hh = host_u64(h)
    assert_bits_equal(hh[rows], nr, "packed intermediate")
    assert np.array_equal(hh, oracle.pack_signs(y1.cpu().numpy())), "intermediate = pack of layer 1 output"
    # layer 2 on sampled outputs
    rng = np.random.default_rng(3)
    r2, c2 = rng.integers(0, m, 2048), rng.integers(0, n, 2048)
    sd, so = oracle.binary_gemm_sampled(hh, w2p, a2, m, n, n, r2, c2)
    assert_bits_equal(d2.cpu().numpy()[r2, c2], sd, "layer 2 dots")
    assert_bits_equal(y2.cpu().numpy()[r2, c2], so, "layer 2 y")
    assert bnn.device_error_count() == 0


# ---------------------------------------------------------------------------
# Ternary layer with bias (bnn_ternary_linear): every AUTO kernel family
# (pair-table GEMV at m = 1, CUDA-core GEMV at m <= 8, bf16 MMA above)
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("m,n,k", [(1, 300, 4096), (1, 70, 33), (3, 140, 700), (8, 65, 161), (64, 200, 4096),
                                   (100, 130, 1001)])
def test_ternary_linear_matches_oracle(bnn, m, n, k):
    from gpu_util import assert_ternary_close, to_dev_bf16, to_dev_u16
    seed = m * 7 + n + k
    w = synth.normal_f32(seed, 1, (n, k))
    trits, scale, _ = oracle.twn_ternarize(w)
    packed = oracle.base3_pack(trits)
    xb = synth.bf16_bits_from_f32(synth.normal_f32(seed, 2, (m, k)))
    bias = synth.normal_f32(seed, 3, (n,))
    want, mag = oracle.ternary_linear(xb, packed, scale, bias, m, n, k)
    got = bnn.bnn_ternary_linear(to_dev_bf16(xb), to_dev_u16(packed), to_dev_f32(scale), to_dev_f32(bias))
    assert_ternary_close(got.cpu().numpy(), want, mag, f"ternary linear {m}x{n}x{k}")
    # without a bias it is bnn_ternary_gemm
    got0 = bnn.bnn_ternary_linear(to_dev_bf16(xb), to_dev_u16(packed), to_dev_f32(scale), None)
    ref0 = bnn.bnn_ternary_gemm(to_dev_bf16(xb), to_dev_u16(packed), to_dev_f32(scale), k)
    assert torch.equal(got0, ref0)
