"""GPU parity of the binary path (sign-pack, XOR+popcount matmul, alpha
epilogue) against the CPU oracle: bit-exact packing and int32 dots, bitwise
float32 outputs.  Every call goes through the C ABI (libbnn.so) via the
binding."""
import numpy as np
import pytest
import torch

import oracle
from conftest import golden_lines
from gpu_util import assert_bits_equal, host_u64, to_dev_f32, to_dev_u64
from ternary_neural_net_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bnn(cuda_device):
    from ternary_neural_net_b200 import bnn as mod
    return mod


def test_pack_special_values(bnn):
    bits = []
    vals = []
    for line in golden_lines("sign_pack_special.txt"):
        h, b = line.split()[:2]
        vals.append(int(h, 16))
        bits.append(int(b))
    x = np.array(vals, dtype=np.uint32).view(np.float32).reshape(1, -1)
    got = host_u64(bnn.bnn_pack_signs(to_dev_f32(x)))
    want = sum(b << i for i, b in enumerate(bits))
    assert int(got[0, 0]) == want


@pytest.mark.parametrize("rows,k", [(1, 1), (3, 63), (5, 64), (7, 65), (2, 1000), (33, 4096 + 17),
                                    (256, 4096), (1, 8192), (300, 129), (4, 2047)])
def test_pack_matches_oracle(bnn, rows, k):
    x = synth.normal_f32(rows * 7 + k, 1, (rows, k))
    x[:, ::13] = 0.0
    special = np.array([-0.0, np.nan, np.inf, -np.inf, 1e-45], np.float32)
    x[0, :min(5, k)] = special[:min(5, k)]
    got = host_u64(bnn.bnn_pack_signs(to_dev_f32(x)))
    assert_bits_equal(got, oracle.pack_signs(x), f"pack {rows}x{k}")


def test_pack_empty(bnn):
    out = bnn.bnn_pack_signs(torch.empty((0, 100), device="cuda"))
    assert out.shape == (0, 2)
    out = bnn.bnn_pack_signs(torch.empty((4, 0), device="cuda"))
    assert out.shape == (4, 0)


def _gemm_case(bnn, m, n, k, seed, offset_words=0, algos=(0, 1, 2, 3)):
    xp = synth.fair_coin_words(seed, 1, m, k)
    wp = synth.fair_coin_words(seed, 2, n, k)
    alpha = synth.uniform_f32(seed, 3, (n,), -1.0, 2.0)
    if n > 2:
        alpha[1] = 0.0
    if offset_words:
        # place the operands 8 bytes past a 16-byte boundary to exercise the 8-byte path
        kw = synth.words_per_row(k)
        bx = torch.zeros(m * kw + offset_words, dtype=torch.int64, device="cuda")
        bw = torch.zeros(n * kw + offset_words, dtype=torch.int64, device="cuda")
        bx[offset_words:] = to_dev_u64(xp).reshape(-1)
        bw[offset_words:] = to_dev_u64(wp).reshape(-1)
        dxp, dwp = bx[offset_words:].view(m, kw), bw[offset_words:].view(n, kw)
    else:
        dxp, dwp = to_dev_u64(xp), to_dev_u64(wp)
    want_d, want_o = oracle.binary_gemm(xp, wp, alpha, m, n, k)
    for algo in algos:
        dots, out = bnn.bnn_binary_gemm(dxp, dwp, to_dev_f32(alpha), k, algo=algo)
        torch.cuda.synchronize()
        assert_bits_equal(dots.cpu().numpy(), want_d, f"dots {m}x{n}x{k} algo {algo}")
        assert_bits_equal(out.cpu().numpy(), want_o, f"out {m}x{n}x{k} algo {algo}")


@pytest.mark.parametrize("m", [1, 2, 3, 4, 5, 8])
@pytest.mark.parametrize("n,k", [(1, 1), (17, 63), (130, 64), (129, 65), (1000, 1000), (64, 4096 + 64 * 3 + 5)])
def test_skinny_matches_oracle(bnn, m, n, k):
    _gemm_case(bnn, m, n, k, seed=m * 1000 + n + k)


# m = 1 GEMV shapes: long rows (several 16-byte passes per lane), short rows
# with many of them, ragged word counts, fewer rows than SMs.
@pytest.mark.parametrize("n,k", [(5000, 16384), (3000, 12000), (70000, 128), (100, 8192), (20000, 640), (7, 4096)])
def test_gemv_m1_shapes(bnn, n, k):
    _gemm_case(bnn, 1, n, k, seed=n + k, algos=(0,))


@pytest.mark.parametrize("m,n,k", [(9, 33, 64), (64, 64, 128), (130, 257, 1000), (300, 129, 4096 + 100),
                                   (129, 1000, 63), (512, 640, 512), (17, 3, 130), (16, 8, 32), (1000, 2500, 257),
                                   (2400, 2500, 640)])
def test_tiled_matches_oracle(bnn, m, n, k):
    _gemm_case(bnn, m, n, k, seed=m + 7 * n + k)


# Shapes that reach each tensor-core configuration: 64- and 128-row activation
# tiles with the stages split over 1, 2 or 4 CTAs of a cluster, with the deep
# ring (one CTA per SM) and without, 256-row tiles, TMA copies (even word
# count) and plain loads (odd), and ragged m, n and k.
@pytest.mark.parametrize("m,n,k", [(40, 300, 2048 + 37), (64, 1000, 1000), (100, 500, 4096), (128, 129, 1100),
                                   (70, 9600, 512), (65, 2, 64 * 20 + 1), (256, 4096 + 3, 4096 - 64),
                                   (257, 383, 2048 * 2 + 64), (2304, 4219, 130), (600, 9000, 760), (50, 700, 2000),
                                   (64, 1000, 300), (64, 2000, 500), (200, 1000, 2048), (300, 3000, 256),
                                   (384, 6400, 128), (250, 700, 2048 + 130),
                                   # two waves of 256 x 224 CTA-pair tiles (the two-SM kernel): ragged m and
                                   # n, one activation tile, a single stage and several, ragged K
                                   (2304, 4219, 128), (2000, 4800, 256), (200, 38000, 128), (300, 40000, 128),
                                   (2048, 4800, 1000), (4100, 2500, 4096)])
def test_tc_tile_configs(bnn, m, n, k):
    _gemm_case(bnn, m, n, k, seed=5 * m + n + 3 * k, algos=(3,))


@pytest.mark.parametrize("m,n,k", [(512, 2431, 8192), (1024, 4096, 1024), (256, 11008, 4096)])
def test_one_sm_plans_sampled(bnn, m, n, k):
    """Shapes where the one-SM plan model picks the split 256-row tiles (512 x
    2431 x 8192: 2-CTA clusters of 256-row activation tiles), one wave of
    256-row tiles, and 256-row tiles over an FFN-sized weight: every output
    against the popcount properties (|dot| <= k, dot = k mod 2), the rows at
    the tile and cluster boundaries bit-exact against the oracle."""
    xp = synth.fair_coin_words(m + 7, 1, m, k)
    wp = synth.fair_coin_words(m + 7, 2, n, k)
    alpha = synth.uniform_f32(m + 7, 3, (n,), 0.5, 1.5)
    dots, out = bnn.bnn_binary_gemm(to_dev_u64(xp), to_dev_u64(wp), to_dev_f32(alpha), k, algo=3)
    d = dots.cpu().numpy()
    assert np.all(np.abs(d) <= k) and np.all((d - k) % 2 == 0)
    rows = np.array(sorted(r for r in {0, 127, 128, 255, 256, m // 2, m - 1} if r < m), dtype=np.int64)
    rr = np.repeat(rows, n)
    cc = np.tile(np.arange(n, dtype=np.int64), rows.size)
    sd, so = oracle.binary_gemm_sampled(xp, wp, alpha, m, n, k, rr, cc)
    assert_bits_equal(d[rr, cc], sd, f"dots {m}x{n}x{k} sampled rows")
    assert_bits_equal(out.cpu().numpy()[rr, cc], so, f"out {m}x{n}x{k} sampled rows")


@pytest.mark.parametrize("m,n,k", [(1, 100, 200), (3, 50, 640), (40, 70, 128), (200, 300, 1024)])
def test_unaligned_operands_use_the_8_byte_path(bnn, m, n, k):
    _gemm_case(bnn, m, n, k, seed=99 + m, offset_words=1)


def test_k_zero_gives_zero_and_alpha_times_zero(bnn):
    for m in (1, 20):
        for algo in (0, 1, 2, 3):
            xp = torch.empty((m, 0), dtype=torch.int64, device="cuda")
            wp = torch.empty((5, 0), dtype=torch.int64, device="cuda")
            alpha = to_dev_f32(np.array([1.0, -2.0, 0.0, 3.5, 1e-3], np.float32))
            dots, out = bnn.bnn_binary_gemm(xp, wp, alpha, 0, algo=algo)
            assert torch.all(dots == 0) and torch.all(out == 0)


def test_dots_only_and_out_only(bnn):
    m, n, k = 6, 40, 300
    xp, wp = synth.fair_coin_words(5, 1, m, k), synth.fair_coin_words(5, 2, n, k)
    alpha = synth.uniform_f32(5, 3, (n,), 0.5, 1.5)
    want_d, want_o = oracle.binary_gemm(xp, wp, alpha, m, n, k)
    d, o = bnn.bnn_binary_gemm(to_dev_u64(xp), to_dev_u64(wp), None, k, want_out=False)
    assert o is None and np.array_equal(d.cpu().numpy(), want_d)
    d, o = bnn.bnn_binary_gemm(to_dev_u64(xp), to_dev_u64(wp), to_dev_f32(alpha), k, want_dots=False)
    assert d is None
    assert_bits_equal(o.cpu().numpy(), want_o, "out only")


def test_identity_special_rows(bnn):
    """x = w gives k, x = -w gives -k, for k across word boundaries."""
    for k in (1, 63, 64, 65, 127, 128, 129, 1000):
        w = synth.fair_coin_words(k, 1, 2, k)
        mask = synth.fair_coin_words(0, 0, 1, k)
        mask[:] = np.uint64(0xFFFFFFFFFFFFFFFF)
        kw = synth.words_per_row(k)
        if k % 64:
            mask[0, kw - 1] = np.uint64((1 << (k % 64)) - 1)
        x = np.stack([w[0], w[0] ^ mask[0]])
        dots, _ = bnn.bnn_binary_gemm(to_dev_u64(x), to_dev_u64(w[:1]), None, k, want_out=False)
        d = dots.cpu().numpy()
        assert d[0, 0] == k and d[1, 0] == -k


# ---------------------------------------------------------------------------
# The five workloads at their full sizes, in the launch configuration the bench
# times; outputs the oracle can compute one by one are sampled.
# ---------------------------------------------------------------------------
def _samples(m, n, count, seed):
    rng = np.random.default_rng(seed)
    rows = np.concatenate([rng.integers(0, m, count), np.zeros(n, np.int64) if n <= 4096 else np.zeros(0, np.int64),
                           np.arange(min(m, 4096))])
    cols = np.concatenate([rng.integers(0, n, count), np.arange(n) if n <= 4096 else np.zeros(0, np.int64),
                           np.zeros(min(m, 4096), np.int64)])
    return rows.astype(np.int64), cols.astype(np.int64)


def test_workload_gemv_small_full(bnn):
    c = synth.gemv_small(1)
    dots, out = bnn.bnn_binary_gemm(to_dev_u64(c["xp"]), to_dev_u64(c["wp"]), to_dev_f32(c["alpha"]), c["k"])
    want_d, want_o = oracle.binary_gemm(c["xp"], c["wp"], c["alpha"], c["m"], c["n"], c["k"])
    assert_bits_equal(dots.cpu().numpy(), want_d, "cfg1 dots")
    assert_bits_equal(out.cpu().numpy(), want_o, "cfg1 out")


@pytest.mark.parametrize("algo", [0, 1, 2, 3])
def test_workload_gemm_fused_pack(bnn, algo):
    c = synth.gemm_fused_pack(1)
    wp = bnn.bnn_pack_signs(to_dev_f32(c["w"]))
    torch.cuda.synchronize()  # weights are complete before a matmul reads them (bnn.h, "Weights are static data")
    xp = bnn.bnn_pack_signs(to_dev_f32(c["x"]))
    dots, out = bnn.bnn_binary_gemm(xp, wp, to_dev_f32(c["alpha"]), c["k"], algo=algo)
    hx, hw = host_u64(xp), host_u64(wp)
    assert_bits_equal(hx, oracle.pack_signs(c["x"]), "cfg2 x pack")
    assert_bits_equal(hw, oracle.pack_signs(c["w"]), "cfg2 w pack")
    rows, cols = _samples(c["m"], c["n"], 4096, 2)
    sd, so = oracle.binary_gemm_sampled(hx, hw, c["alpha"], c["m"], c["n"], c["k"], rows, cols)
    assert_bits_equal(dots.cpu().numpy()[rows, cols], sd, "cfg2 dots")
    assert_bits_equal(out.cpu().numpy()[rows, cols], so, "cfg2 out")


def test_workload_gemv_ffn(bnn):
    c = synth.gemv_ffn(1)
    xp = bnn.bnn_pack_signs(to_dev_f32(c["x"]))
    _, out = bnn.bnn_binary_gemm(xp, to_dev_u64(c["wp"]), to_dev_f32(c["alpha"]), c["k"], want_dots=False)
    hx = host_u64(xp)
    assert_bits_equal(hx, oracle.pack_signs(c["x"]), "cfg3 x pack")
    _, want_o = oracle.binary_gemm(hx, c["wp"], c["alpha"], 1, c["n"], c["k"])  # 2.3e8 MAC: full
    assert_bits_equal(out.cpu().numpy(), want_o, "cfg3 out")


@pytest.mark.parametrize("algo", [0, 1, 3])
def test_workload_gemm_large(bnn, algo):
    c = synth.gemm_large(1)
    dots, out = bnn.bnn_binary_gemm(to_dev_u64(c["xp"]), to_dev_u64(c["wp"]), to_dev_f32(c["alpha"]), c["k"],
                                    algo=algo)
    torch.cuda.synchronize()
    rows, cols = _samples(c["m"], c["n"], 2048, 4)
    sd, so = oracle.binary_gemm_sampled(c["xp"], c["wp"], c["alpha"], c["m"], c["n"], c["k"], rows, cols)
    d = dots.cpu().numpy()
    assert_bits_equal(d[rows, cols], sd, "cfg4 dots")
    assert_bits_equal(out.cpu().numpy()[rows, cols], so, "cfg4 out")
    # properties at every output: parity of k, range, and out = alpha * dot
    k = c["k"]
    assert np.all((d - k) % 2 == 0) and np.abs(d).max() <= k
    o = out.cpu().numpy()
    assert_bits_equal(o, c["alpha"][None, :] * d.astype(np.float32), "cfg4 epilogue everywhere")
    if algo == 0:
        # every output against the CPU baseline restated from the pages' XOR + popcount
        # loop (itself checked bitwise against the oracle), on all host cores
        import os
        kd, _ = oracle.k1_binary_gemm(c["xp"], c["wp"], c["alpha"], c["m"], c["n"], k, os.cpu_count() or 1)
        assert np.array_equal(d, kd), "cfg4 dots differ from the CPU XOR + popcount baseline"


def test_algos_agree_bitwise_on_random_shapes(bnn):
    """Every kernel family gives the same bits on ragged shapes (m from 1 to 300)."""
    rng = np.random.default_rng(77)
    for _ in range(12):
        m, n, k = int(rng.integers(1, 300)), int(rng.integers(1, 300)), int(rng.integers(1, 700))
        xp = to_dev_u64(synth.fair_coin_words(int(m + n + k), 1, m, k))
        wp = to_dev_u64(synth.fair_coin_words(int(m + n + k), 2, n, k))
        alpha = to_dev_f32(synth.uniform_f32(3, 3, (n,), -2.0, 2.0))
        res = [bnn.bnn_binary_gemm(xp, wp, alpha, k, algo=a) for a in (0, 1, 2, 3)]
        for d, o in res[1:]:
            assert torch.equal(d, res[0][0]) and torch.equal(o.view(torch.int32), res[0][1].view(torch.int32))


def test_unknown_algo_rejected(bnn):
    xp = torch.zeros((2, 1), dtype=torch.int64, device="cuda")
    with pytest.raises(bnn.BnnError):
        bnn.bnn_binary_gemm(xp, xp, None, 64, want_out=False, algo=7)


def test_no_device_wait_ran_out(bnn):
    """Every bounded wait of the tensor-core kernels completed in this run."""
    torch.cuda.synchronize()
    assert bnn.device_error_count() == 0
