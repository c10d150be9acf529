"""GPU parity of the index + sign sparse ternary path: row_ptr and entries
bit-exact against the oracle's encoding of the same trits (from base-3 words
made by the GPU pack), and the sparse layer within the ternary tolerance of the
float64 oracle, at small ragged shapes and at the 11008 x 4096 layer with a
high-sparsity threshold."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import assert_bits_equal, assert_ternary_close, to_dev_bf16, to_dev_f32, to_dev_u16
from ternary_neural_net_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bnn(cuda_device):
    from ternary_neural_net_b200 import bnn as mod
    return mod


def _encode(bnn, trits, k):
    packed = oracle.base3_pack(trits)
    row_ptr, ent = bnn.bnn_ternary_sparse_encode(to_dev_u16(packed), k)
    torch.cuda.synchronize()
    return packed, row_ptr, ent


@pytest.mark.parametrize("n,k,density", [(1, 1, 1.0), (5, 9, 0.5), (37, 130, 0.1), (64, 4096, 0.58),
                                         (3, 32768, 0.05), (9, 1000, 0.0), (20, 311, 1.0)])
def test_encode_matches_oracle(bnn, n, k, density):
    rng = np.random.default_rng(n * 13 + k)
    trits = ((rng.integers(0, 2, (n, k)) * 2 - 1) * (rng.random((n, k)) < density)).astype(np.int8)
    _, row_ptr, ent = _encode(bnn, trits, k)
    want_rp, want_ent = oracle.sparse_encode(trits)
    assert_bits_equal(row_ptr.cpu().numpy(), want_rp, "row_ptr")
    assert_bits_equal(ent.cpu().numpy().view(np.uint16), want_ent, "entries")


@pytest.mark.parametrize("m,n,k", [(1, 70, 33), (1, 300, 4096), (3, 140, 700), (8, 65, 161), (13, 40, 999)])
@pytest.mark.parametrize("with_bias", [True, False])
def test_sparse_gemm_matches_oracle(bnn, m, n, k, with_bias):
    rng = np.random.default_rng(m * 100 + n + k)
    trits = (rng.integers(-1, 2, (n, k)) * (rng.random((n, k)) < 0.2)).astype(np.int8)
    scale = (rng.random(n) + 0.5).astype(np.float32)
    bias = rng.standard_normal(n).astype(np.float32) if with_bias else None
    xb = synth.bf16_bits_from_f32(synth.normal_f32(m + k, 1, (m, k)))
    _, row_ptr, ent = _encode(bnn, trits, k)
    got = bnn.bnn_ternary_sparse_gemm(to_dev_bf16(xb), row_ptr, ent, to_dev_f32(scale),
                                      to_dev_f32(bias) if with_bias else None)
    rp, en = oracle.sparse_encode(trits)
    want, mag = oracle.sparse_gemm(xb, rp, en, scale, bias, m, n, k)
    assert_ternary_close(got.cpu().numpy(), want, mag, f"sparse {m}x{n}x{k}")


def test_sparse_layer_full_size(bnn):
    """The 11008 x 4096 layer ternarised with the fixed-threshold (delta) mode at
    a threshold leaving ~10% non-zero trits: GPU pack -> GPU sparse encode ->
    sparse GEMV; the encoding is checked in full, the outputs against the
    float64 oracle at every row, and against the dense layer on the same words."""
    c = synth.ternary(1, m=1)
    n, k = c["n"], c["k"]
    w = torch.from_numpy(c["w"]).cuda()
    packed, scale, _ = bnn.bnn_ternary_pack_mode(w, bnn.TERNARY_DELTA, 1.6449)
    row_ptr, ent = bnn.bnn_ternary_sparse_encode(packed, k)
    hp = packed.cpu().numpy().view(np.uint16)
    trits, bad = oracle.base3_unpack(hp, k)
    assert bad == 0
    rp, en = oracle.sparse_encode(trits)
    assert_bits_equal(row_ptr.cpu().numpy(), rp, "row_ptr")
    assert_bits_equal(ent.cpu().numpy().view(np.uint16), en, "entries")
    density = len(en) / (n * k)
    assert 0.08 < density < 0.12, density
    xb = c["x_bf16"]
    got = bnn.bnn_ternary_sparse_gemm(to_dev_bf16(xb), row_ptr, ent, scale)
    hs = scale.cpu().numpy()
    want, mag = oracle.sparse_gemm(xb, rp, en, hs, None, 1, n, k)
    assert_ternary_close(got.cpu().numpy(), want, mag, "sparse full")
    dense = bnn.bnn_ternary_gemm(to_dev_bf16(xb), packed, scale, k)
    assert_ternary_close(dense.cpu().numpy(), want, mag, "dense on the same words")
    assert bnn.device_error_count() == 0


def test_sparse_gemm_right_after_encode_with_device_x(bnn):
    """The natural call sequence with everything already on the device and no
    copy in between: pack -> encode -> sparse matmul.  The matmul starts early
    (programmatic dependent launch) and reads row_ptr and entries before its
    wait, so the binding's encode must return complete weights."""
    n, k, m = 3000, 4096, 2
    w = torch.from_numpy(synth.normal_f32(77, 3, (n, k))).cuda()
    xd = to_dev_bf16(synth.bf16_bits_from_f32(synth.normal_f32(77, 4, (m, k))))
    torch.cuda.synchronize()
    packed, scale, _ = bnn.bnn_ternary_pack_mode(w, bnn.TERNARY_DELTA, 1.2)
    torch.cuda.synchronize()
    for _ in range(3):
        row_ptr, ent = bnn.bnn_ternary_sparse_encode(packed, k)
        got = bnn.bnn_ternary_sparse_gemm(xd, row_ptr, ent, scale)
        trits, _ = oracle.base3_unpack(packed.cpu().numpy().view(np.uint16), k)
        rp, en = oracle.sparse_encode(trits)
        want, mag = oracle.sparse_gemm(xd.view(torch.int16).cpu().numpy().view(np.uint16), rp, en,
                                       scale.cpu().numpy(), None, m, n, k)
        assert_ternary_close(got.cpu().numpy(), want, mag, "sparse right after encode")
        del row_ptr, ent


@pytest.mark.parametrize("n,k,density", [(150, 32768, 0.1), (300, 1000, 0.0), (1000, 777, 0.7), (5, 3, 1.0),
                                         (1000, 32768, 0.9), (700000, 20, 0.5), (11008, 4096, 0.1)])
def test_sparse_gemv_m1_shapes(bnn, n, k, density):
    """m = 1 (x staged in shared memory): the longest rows k allows (several
    passes of 512 entries per row), empty rows, dense rows and tiny k, with
    every other row emptied; long dense rows at the largest k, thousands of
    rows per CTA, and the full 11008 x 4096 layer at 10% density."""
    rng = np.random.default_rng(n + k)
    trits = ((rng.integers(0, 2, (n, k)) * 2 - 1) * (rng.random((n, k)) < density)).astype(np.int8)
    trits[::2] = 0
    scale = (rng.random(n) + 0.5).astype(np.float32)
    bias = rng.standard_normal(n).astype(np.float32)
    xb = synth.bf16_bits_from_f32(synth.normal_f32(n + k, 1, (1, k)))
    _, row_ptr, ent = _encode(bnn, trits, k)
    rp, en = oracle.sparse_encode(trits)
    for b in (None, bias):
        got = bnn.bnn_ternary_sparse_gemm(to_dev_bf16(xb), row_ptr, ent, to_dev_f32(scale),
                                          None if b is None else to_dev_f32(b))
        want, mag = oracle.sparse_gemm(xb, rp, en, scale, b, 1, n, k)
        lim = mag + (0 if b is None else np.abs(b.astype(np.float64)))
        assert_ternary_close(got.cpu().numpy(), want, lim, f"sparse m=1 {n}x{k}")


@pytest.mark.parametrize("n,k,density", [(11008, 4096, 0.1), (300, 5000, 0.6)])
def test_sparse_gemv_m1_entries_two_bytes_off(bnn, n, k, density):
    """m = 1 with the entries 2 bytes off a 4-byte boundary (16-bit loads of
    each pair instead of one 32-bit load): the same sums in the same order, so
    bit-identical outputs, and both match the oracle."""
    rng = np.random.default_rng(3 * n + k)
    trits = ((rng.integers(0, 2, (n, k)) * 2 - 1) * (rng.random((n, k)) < density)).astype(np.int8)
    scale = (rng.random(n) + 0.5).astype(np.float32)
    xb = synth.bf16_bits_from_f32(synth.normal_f32(n + k, 2, (1, k)))
    _, row_ptr, ent = _encode(bnn, trits, k)
    buf = torch.empty(ent.numel() + 1, dtype=ent.dtype, device="cuda")
    buf[1:] = ent
    ent_off = buf[1:]
    assert ent.data_ptr() % 4 == 0 and ent_off.data_ptr() % 4 == 2
    xd, sd = to_dev_bf16(xb), to_dev_f32(scale)
    got = bnn.bnn_ternary_sparse_gemm(xd, row_ptr, ent, sd)
    got_off = bnn.bnn_ternary_sparse_gemm(xd, row_ptr, ent_off, sd)
    assert torch.equal(got.view(torch.int32), got_off.view(torch.int32))
    rp, en = oracle.sparse_encode(trits)
    want, mag = oracle.sparse_gemm(xb, rp, en, scale, None, 1, n, k)
    assert_ternary_close(got.cpu().numpy(), want, mag, f"sparse m=1 {n}x{k} entries +2")
