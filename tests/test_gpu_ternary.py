"""GPU parity of the ternary path (TWN ternarise + least-squares scale +
base-3 pack, and the ternary matmul) against the CPU oracle.  Trits/words are
bit-exact given the same threshold; scales within 1 ulp (float64 sums in a
different order, rounded once); matmul outputs within 1e-3 of scale*sum|x t|."""
import math

import numpy as np
import pytest
import torch

import oracle
from gpu_util import assert_bits_equal, assert_ternary_close, host_u16, to_dev_bf16, to_dev_f32, to_dev_u16
from ternary_neural_net_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bnn(cuda_device):
    from ternary_neural_net_b200 import bnn as mod
    return mod


def _ulp_diff(a: np.ndarray, b: np.ndarray) -> int:
    ia = a.astype(np.float32).view(np.int32).astype(np.int64)
    ib = b.astype(np.float32).view(np.int32).astype(np.int64)
    return int(np.abs(ia - ib).max()) if a.size else 0


def _check_pack(bnn, w: np.ndarray, what: str):
    n, k = w.shape
    packed, scale, delta = bnn.bnn_ternary_pack(to_dev_f32(w))
    torch.cuda.synchronize()
    gp, gs, gd = host_u16(packed), scale.cpu().numpy(), np.float32(delta.cpu().numpy()[0])
    od = oracle.twn_delta(w)
    if gd != od:
        # float64 sums in another order rounded to a different float32 Delta:
        # compare against the oracle run at the GPU's Delta, and say how many
        # weights lie between the two thresholds.
        lo, hi = min(gd, od), max(gd, od)
        between = int(((np.abs(w) > lo) & (np.abs(w) <= hi)).sum())
        print(f"{what}: Delta differs (gpu {gd!r}, oracle {od!r}); {between} weights in between")
        assert abs(float(gd) - float(od)) <= 2 * np.spacing(np.float32(od))
    trits, oscale = oracle.twn_apply(w, gd)
    assert_bits_equal(gp, oracle.base3_pack(trits), f"{what} words")
    assert _ulp_diff(gs, oscale) <= 1, f"{what} scales"
    return gp, gs, gd


@pytest.mark.parametrize("n,k", [(1, 1), (3, 10), (5, 23), (2, 9), (7, 4096), (64, 1000), (300, 4096 + 7)])
def test_pack_matches_oracle(bnn, n, k):
    w = synth.normal_f32(n + k, 5, (n, k))
    w[0, :3] = [0.0, -0.0, np.float32(1e-30)][: min(3, k)]
    _check_pack(bnn, w, f"pack {n}x{k}")


def test_pack_golden_tie_and_empty_rows(bnn):
    w = np.array([[-7, 13, -10, 10]], np.float32)  # Delta = 7 exactly, |-7| is not > Delta
    packed, scale, delta = bnn.bnn_ternary_pack(to_dev_f32(w))
    t, bad = oracle.base3_unpack(host_u16(packed), 4)
    assert bad == 0 and t.tolist() == [[0, 1, -1, 1]]
    assert float(delta.cpu()[0]) == 7.0 and float(scale.cpu()[0]) == 11.0
    w = np.array([[0.1, -0.1, 0.1, -0.1], [5, -5, 5, -5]], np.float32)
    packed, scale, _ = bnn.bnn_ternary_pack(to_dev_f32(w))
    t, _ = oracle.base3_unpack(host_u16(packed), 4)
    assert t.tolist() == [[0, 0, 0, 0], [1, -1, 1, -1]] and scale.cpu().tolist() == [0.0, 5.0]
    w = np.zeros((3, 11), np.float32)
    packed, scale, delta = bnn.bnn_ternary_pack(to_dev_f32(w))
    assert np.all(host_u16(packed)[:, 0] == 29524) and float(delta.cpu()[0]) == 0.0
    assert torch.all(scale == 0)


def test_pack_empty_shapes(bnn):
    packed, scale, delta = bnn.bnn_ternary_pack(torch.empty((0, 5), device="cuda"))
    torch.cuda.synchronize()
    assert packed.shape == (0, 1) and float(delta.cpu()[0]) == 0.0
    packed, scale, delta = bnn.bnn_ternary_pack(torch.empty((4, 0), device="cuda"))
    torch.cuda.synchronize()
    assert packed.shape == (4, 0) and torch.all(scale == 0) and float(delta.cpu()[0]) == 0.0


def test_pack_is_reproducible(bnn):
    w = to_dev_f32(synth.normal_f32(3, 3, (513, 777)))
    a = [t.clone() for t in bnn.bnn_ternary_pack(w)]
    b = bnn.bnn_ternary_pack(w)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def _gemm_case(bnn, m, n, k, seed, trits=None, algos=(0,)):
    rng = np.random.default_rng(seed)
    if trits is None:
        trits = rng.integers(-1, 2, (n, k)).astype(np.int8)
    packed = oracle.base3_pack(trits)
    scale = synth.uniform_f32(seed, 1, (n,), 0.25, 2.0)
    xb = synth.bf16_bits_from_f32(synth.normal_f32(seed, 2, (m, k)))
    ref, mag = oracle.ternary_gemm(xb, packed, scale, m, n, k)
    worst = 0.0
    for algo in algos:
        out = bnn.bnn_ternary_gemm(to_dev_bf16(xb), to_dev_u16(packed), to_dev_f32(scale), k, algo=algo)
        worst = max(worst, assert_ternary_close(out.cpu().numpy(), ref, mag, f"ternary {m}x{n}x{k} algo {algo}"))
    return worst


@pytest.mark.parametrize("m,n,k", [(1, 7, 10), (1, 100, 4096), (2, 33, 95), (4, 65, 161), (8, 64, 1000),
                                   (1, 5, 1), (3, 9, 9)])
def test_gemv_matches_oracle(bnn, m, n, k):
    _gemm_case(bnn, m, n, k, seed=m * 31 + n + k)


@pytest.mark.parametrize("m,n,k", [(9, 65, 161), (64, 64, 160), (64, 200, 4096), (100, 130, 1001),
                                   (130, 70, 33), (65, 1, 10), (64, 300, 640), (1, 129, 64), (3, 140, 700)])
def test_gemm_matches_oracle(bnn, m, n, k):
    _gemm_case(bnn, m, n, k, seed=m * 17 + n + k, algos=(0, 2, 3))


@pytest.mark.parametrize("m", [1, 64])
def test_every_base3_word_decodes(bnn, m):
    """One weight row holding all 3^10 words once (k = 590490): every code goes
    through the kernel's decoder."""
    words = np.arange(59049, dtype=np.uint16).reshape(1, -1)
    trits, bad = oracle.base3_unpack(words, 590490)
    assert bad == 0
    rows = np.concatenate([trits, -trits, np.zeros_like(trits)])
    _gemm_case(bnn, m, 3, 590490, seed=5 + m, trits=rows, algos=(0, 3) if m > 1 else (0,))


# Shapes for the warp-specialised tensor-core kernels (k a multiple of 8): the
# stages split over 4, 3, 2 and 1 CTAs, ragged m and n, word groups cut short,
# a single stage, and m = 1.  m <= 64 takes the kernel that decodes into
# tensor memory, larger m the one that decodes into shared memory.
@pytest.mark.parametrize("m,n,k", [(64, 300, 4096), (200, 1000, 640), (128, 9600, 160), (1, 129, 64),
                                   (70, 130, 4096 + 8), (33, 255, 2400), (50, 10000, 1600), (40, 385, 1288),
                                   (64, 129, 8)])
def test_tc_warp_specialised_configs(bnn, m, n, k):
    _gemm_case(bnn, m, n, k, seed=m * 5 + n + k, algos=(3,))


def test_every_base3_word_decodes_tma_path(bnn):
    """All 3^10 words in one row with k a multiple of 8 (the TMA kernel), then
    a zero-trit word: every code goes through the phase-specialised decoder."""
    k = 590496
    words = np.concatenate([np.arange(59049, dtype=np.uint16), np.array([29524], np.uint16)]).reshape(1, -1)
    trits, bad = oracle.base3_unpack(words, k)
    assert bad == 0
    rows = np.concatenate([trits, -trits, np.zeros_like(trits)])
    _gemm_case(bnn, 64, 3, k, seed=17, trits=rows, algos=(3,))


def test_every_base3_word_decodes_row_kernel(bnn):
    """All 3^10 words spread over 60 rows of 1000 words (k = 10000, the m = 1
    pair-table kernel), every code through its decoder, with a bias."""
    k = 10000
    words = (np.arange(60000) % 59049).astype(np.uint16).reshape(60, 1000)
    trits, bad = oracle.base3_unpack(words, k)
    assert bad == 0
    _gemm_case(bnn, 1, 60, k, seed=23, trits=trits, algos=(0, 1))


@pytest.mark.parametrize("k,kt", [(4100, 410), (4090, 409)])
def test_every_base3_word_decodes_table_kernel(bnn, k, kt):
    """All 3^10 words in 145 rows (k = 4100: 410 words a row, the m = 1
    kernel on 5 + 5-trit activation tables with 32-bit word pairs; k = 4090:
    409 words, the same kernel on 16-bit loads), every code through both
    tables of every lane position, with and without a bias."""
    rows = (59049 + kt - 1) // kt
    words = (np.arange(rows * kt) % 59049).astype(np.uint16).reshape(rows, kt)
    trits, bad = oracle.base3_unpack(words, k)
    assert bad == 0
    _gemm_case(bnn, 1, rows, k, seed=29, trits=trits, algos=(0,))
    scale = synth.uniform_f32(29, 1, (rows,), 0.25, 2.0)
    bias = synth.normal_f32(29, 3, (rows,))
    xb = synth.bf16_bits_from_f32(synth.normal_f32(29, 2, (1, k)))
    ref, mag = oracle.ternary_linear(xb, words, scale, bias, 1, rows, k)
    out = bnn.bnn_ternary_linear(to_dev_bf16(xb), to_dev_u16(words), to_dev_f32(scale), to_dev_f32(bias))
    assert_ternary_close(out.cpu().numpy(), ref, mag + np.abs(bias.astype(np.float64)), "table kernel with bias")


# m = 1 shapes around the table kernel's limits: word counts from 2 to its
# maximum 480 (k = 4800; 4801 takes the pair-table kernel), even (32-bit word
# pairs) and odd (16-bit loads), clusters with more rows than one chunk of
# 1024, fewer rows than a round of 128, one cluster, and pad trits in the last
# word.
@pytest.mark.parametrize("n,k", [(1, 11), (7, 20), (300, 640), (149, 4160), (1000, 4140), (40000, 100),
                                 (5000, 4096), (500, 1300), (33, 4161), (64, 1290), (150, 4170),
                                 (2000, 4800), (300, 4801), (129, 4791)])
def test_gemv_m1_table_shapes(bnn, n, k):
    _gemm_case(bnn, 1, n, k, seed=n + k)


def test_gemv_m1_packed_two_bytes_off(bnn):
    """Packed words 2 bytes off 4-byte alignment take the table kernel's
    16-bit loads, with the same results."""
    n, k = 300, 4096
    rng = np.random.default_rng(5)
    trits = rng.integers(-1, 2, (n, k)).astype(np.int8)
    packed = oracle.base3_pack(trits)
    scale = synth.uniform_f32(5, 1, (n,), 0.25, 2.0)
    xb = synth.bf16_bits_from_f32(synth.normal_f32(5, 2, (1, k)))
    ref, mag = oracle.ternary_gemm(xb, packed, scale, 1, n, k)
    pbuf = torch.empty(packed.size + 1, dtype=torch.int16, device="cuda")
    pbuf[1:] = to_dev_u16(packed).reshape(-1)
    p_off = pbuf[1:].view(packed.shape)
    assert p_off.data_ptr() % 4 == 2
    for pd in (to_dev_u16(packed), p_off):
        out = bnn.bnn_ternary_gemm(to_dev_bf16(xb), pd, to_dev_f32(scale), k)
        assert_ternary_close(out.cpu().numpy(), ref, mag, "m = 1, packed alignment")


def test_gemv_m1_is_deterministic(bnn):
    c = synth.ternary(2, m=1)
    trits = np.random.default_rng(3).integers(-1, 2, (2000, c["k"])).astype(np.int8)
    pd = to_dev_u16(oracle.base3_pack(trits))
    xd, sd = to_dev_bf16(c["x_bf16"]), to_dev_f32(np.ones(2000, np.float32))
    a = bnn.bnn_ternary_gemm(xd, pd, sd, c["k"])
    b = bnn.bnn_ternary_gemm(xd, pd, sd, c["k"])
    assert torch.equal(a, b)


def test_zero_trits_give_exact_zero(bnn):
    k = 300
    packed = np.full((4, 30), 29524, np.uint16)
    xb = synth.bf16_bits_from_f32(synth.normal_f32(1, 1, (3, k)))
    for m in (1, 3):
        out = bnn.bnn_ternary_gemm(to_dev_bf16(xb[:m]), to_dev_u16(packed), to_dev_f32(np.ones(4, np.float32)), k)
        assert torch.all(out == 0)


@pytest.mark.parametrize("m", [1, 64])
def test_workload_ternary_full(bnn, m):
    c = synth.ternary(1, m=m)
    gp, gs, gd = _check_pack(bnn, c["w"], "cfg5 pack")
    zero_frac = float((oracle.base3_unpack(gp, c["k"])[0] == 0).mean())
    print(f"cfg5: Delta={gd} zero fraction={zero_frac:.4f}")
    assert 0.40 < zero_frac < 0.45
    ref, mag = oracle.ternary_gemm(c["x_bf16"], gp, gs, m, c["n"], c["k"])
    for algo in ((0,) if m == 1 else (0, 2, 3)):
        out = bnn.bnn_ternary_gemm(to_dev_bf16(c["x_bf16"]), to_dev_u16(gp), to_dev_f32(gs), c["k"], algo=algo)
        worst = assert_ternary_close(out.cpu().numpy(), ref, mag, f"cfg5 m={m} algo {algo}")
        print(f"cfg5 m={m} algo {algo}: worst |err|/mag = {worst:.3e}")
    assert bnn.device_error_count() == 0


def _check_absmean(bnn, w: np.ndarray, what: str):
    """GPU absmean pack against the oracle.  gamma is the float64 mean of |W|
    rounded once to float32; the GPU sums in another order, so its gamma may be
    a neighbouring float32.  Then the trits and scales are compared with the
    oracle's trit rule run at the GPU's gamma (the same float32 quotient and
    rounding on both sides), and the number of weights whose trit the two
    gammas would decide differently is reported."""
    packed, scale, gamma = bnn.bnn_ternary_pack_mode(to_dev_f32(w), bnn.TERNARY_ABSMEAN)
    torch.cuda.synchronize()
    gg = np.float32(gamma.cpu().numpy()[0])
    ot, os_, og = oracle.absmean_ternarize(w)
    if gg != og:
        assert abs(float(gg) - float(og)) <= 2 * np.spacing(np.float32(og)), (what, gg, og)
        ot, os_ = oracle.absmean_apply(w, gg)
        moved = int((oracle.absmean_apply(w, og)[0] != ot).sum())
        print(f"{what}: gamma differs (gpu {gg!r}, oracle {og!r}); {moved} trits decided differently")
    assert_bits_equal(host_u16(packed), oracle.base3_pack(ot), f"{what} words")
    assert _ulp_diff(scale.cpu().numpy(), os_) <= 1, f"{what} scales"
    return host_u16(packed), scale.cpu().numpy(), gg


@pytest.mark.parametrize("n,k", [(7, 4096), (64, 1000), (300, 4096 + 7), (1, 1), (1000, 777)])
def test_pack_mode_absmean_matches_oracle(bnn, n, k):
    w = synth.normal_f32(n * 3 + k, 7, (n, k))
    _check_absmean(bnn, w, f"absmean {n}x{k}")


def test_pack_modes_full_size(bnn):
    """absmean and delta (F = 0.5 and the 10%-density F = 1.6449) on the
    11008 x 4096 layer: words bit-exact, scales within 1 ulp."""
    w = synth.ternary(1, m=1)["w"]
    gp, _, gg = _check_absmean(bnn, w, "absmean 11008x4096")
    zero_frac = float((oracle.base3_unpack(gp, w.shape[1])[0] == 0).mean())
    print(f"absmean 11008x4096: gamma={gg} zero fraction={zero_frac:.4f}")
    # N(0,1): gamma -> sqrt(2/pi); |w / gamma| <= 0.5 with probability erf(gamma / (2 sqrt 2))
    assert abs(zero_frac - math.erf(float(gg) / (2 * math.sqrt(2)))) < 2e-3
    for F in (0.5, 1.6449):
        packed, scale, thr = bnn.bnn_ternary_pack_mode(to_dev_f32(w), bnn.TERNARY_DELTA, F)
        torch.cuda.synchronize()
        ot, os_ = oracle.delta_ternarize(w, np.float32(F))
        assert float(thr.cpu()[0]) == np.float32(F)
        assert_bits_equal(host_u16(packed), oracle.base3_pack(ot), f"delta F={F} 11008x4096 words")
        assert _ulp_diff(scale.cpu().numpy(), os_) <= 1, f"delta F={F} scales"


def test_ternary_m256_full_size_sampled(bnn):
    """The AUTO route for m > 64 (the tensor-core kernel that decodes into
    shared memory) at 256 x 11008 x 4096: 4096 sampled outputs plus all of
    row 0, row 255 and columns 0 and 11007 against the oracle, and a
    property at every output: |y| <= |scale| * sum |x| (the largest value a
    row of trits can give)."""
    c = synth.ternary(1, m=256)
    n, k = c["n"], c["k"]
    gp, gs, _ = _check_pack(bnn, c["w"], "cfg5 pack (m=256)")
    xd = to_dev_bf16(c["x_bf16"])
    out = bnn.bnn_ternary_gemm(xd, to_dev_u16(gp), to_dev_f32(gs), k).cpu().numpy()
    assert bnn.device_error_count() == 0
    rng = np.random.default_rng(256)
    rows = np.concatenate([rng.integers(0, 256, 4096), np.zeros(n, np.int64), np.full(n, 255),
                           np.arange(256), np.arange(256)])
    cols = np.concatenate([rng.integers(0, n, 4096), np.arange(n), np.arange(n), np.zeros(256, np.int64),
                           np.full(256, n - 1)])
    ref, mag = oracle.ternary_gemm_sampled(c["x_bf16"], gp, gs, 256, n, k, rows, cols)
    assert_ternary_close(out[rows, cols], ref, mag, "cfg5 m=256 sampled")
    xabs = np.abs((c["x_bf16"].astype(np.uint32) << 16).view(np.float32).astype(np.float64))
    bound = np.abs(gs.astype(np.float64))[None, :] * xabs.sum(axis=1)[:, None]
    assert np.all(np.isfinite(out)) and np.all(np.abs(out) <= bound * (1 + 1e-3) + 1e-30)


@pytest.mark.parametrize("F", [0.0, 0.5, 1.3])
def test_pack_mode_delta_matches_oracle(bnn, F):
    w = synth.normal_f32(5, 8, (33, 777))
    w[0, :3] = [0.5, -0.5, 1.3]  # ties at the thresholds
    packed, scale, thr = bnn.bnn_ternary_pack_mode(to_dev_f32(w), bnn.TERNARY_DELTA, F)
    torch.cuda.synchronize()
    ot, os_ = oracle.delta_ternarize(w, np.float32(F))
    assert float(thr.cpu()[0]) == np.float32(F)
    assert_bits_equal(host_u16(packed), oracle.base3_pack(ot), f"delta F={F}")
    assert _ulp_diff(scale.cpu().numpy(), os_) <= 1


def test_pack_mode_twn_is_bnn_ternary_pack(bnn):
    w = to_dev_f32(synth.normal_f32(6, 9, (40, 500)))
    a = bnn.bnn_ternary_pack(w)
    b = bnn.bnn_ternary_pack_mode(w, bnn.TERNARY_TWN)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_pack_mode_golden_absmean_ties(bnn):
    w = np.array([[1, -1, 3, -3]], np.float32)   # gamma = 2: +-0.5 ties round to 0, +-1.5 clip to +-1
    packed, scale, gamma = bnn.bnn_ternary_pack_mode(to_dev_f32(w), bnn.TERNARY_ABSMEAN)
    t, _ = oracle.base3_unpack(host_u16(packed), 4)
    assert t.tolist() == [[0, 0, 1, -1]] and float(gamma.cpu()[0]) == 2.0 and float(scale.cpu()[0]) == 3.0
    with pytest.raises(bnn.BnnError):
        bnn.bnn_ternary_pack_mode(to_dev_f32(w), 7)
    with pytest.raises(bnn.BnnError):
        bnn.bnn_ternary_pack_mode(to_dev_f32(w), bnn.TERNARY_DELTA, -1.0)


def test_auto_one_tile_edge_cases(bnn):
    """AUTO for 9 <= m <= 64 takes the tensor-memory kernel only when k % 8 == 0,
    x is 16-byte and the packed words 4-byte aligned: an empty K gives
    scale * 0, packed words 2 bytes off take the shared-memory tcgen05 kernel
    and activations 2 bytes off the mma.sync kernel, with the same results."""
    n = 70
    x0 = torch.empty((20, 0), dtype=torch.bfloat16, device="cuda")
    p0 = torch.empty((n, 0), dtype=torch.int16, device="cuda")
    out = bnn.bnn_ternary_gemm(x0, p0, to_dev_f32(np.ones(n, np.float32)), 0)
    assert torch.all(out == 0)

    m, k = 24, 640
    rng = np.random.default_rng(41)
    trits = rng.integers(-1, 2, (n, k)).astype(np.int8)
    packed = oracle.base3_pack(trits)
    scale = synth.uniform_f32(41, 1, (n,), 0.25, 2.0)
    xb = synth.bf16_bits_from_f32(synth.normal_f32(41, 2, (m, k)))
    ref, mag = oracle.ternary_gemm(xb, packed, scale, m, n, k)
    # 2-byte offsets: a view one element into a larger buffer
    pbuf = torch.empty(packed.size + 1, dtype=torch.int16, device="cuda")
    pbuf[1:] = to_dev_u16(packed).reshape(-1)
    p_off = pbuf[1:].view(packed.shape)
    xbuf = torch.empty(xb.size + 1, dtype=torch.int16, device="cuda")
    xbuf[1:] = to_dev_u16(xb).reshape(-1)
    x_off = xbuf[1:].view(torch.bfloat16).view(m, k)
    assert p_off.data_ptr() % 4 == 2 and x_off.data_ptr() % 16 == 2
    sc = to_dev_f32(scale)
    for xd, pd, what in ((to_dev_bf16(xb), to_dev_u16(packed), "aligned"), (to_dev_bf16(xb), p_off, "packed +2"),
                         (x_off, to_dev_u16(packed), "x +2")):
        out = bnn.bnn_ternary_gemm(xd, pd, sc, k)
        assert_ternary_close(out.cpu().numpy(), ref, mag, f"AUTO one tile, {what}")


# The tensor-memory kernel (9 <= m <= 64, k % 8 == 0): tiles whose rows fit
# shared memory whole (one bulk copy of the tile's words, the matrix end not on
# a 16-byte boundary, odd word counts), long rows that take the word-group
# loads, and split-K plans.
@pytest.mark.parametrize("m,n,k", [(64, 999, 4100), (48, 5000, 1288), (64, 300, 32000), (17, 2000, 4096),
                                   (64, 150, 8000)])
def test_tmem_word_sources(bnn, m, n, k):
    _gemm_case(bnn, m, n, k, seed=3 * m + n + k)
