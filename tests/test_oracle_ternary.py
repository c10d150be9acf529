"""Pins for the oracle's ternary path: exhaustive base-3 round trip over all
3^10 codes, closed-form words, hand-worked TWN cases, least-squares
optimality, N(0,1) statistics with known closed forms, and the ternary matmul
against numpy float64 matmul and special cases.

Page: "BalancedTernaryEngine" README, sections "Features" (TWN threshold,
least-squares per-channel scale, 10 trits per 16-bit word in base 3),
".tbin Format" and Layer.forward in "Module Overview"."""
import math

import numpy as np
import pytest
import torch

import oracle
from conftest import golden_lines
from ternary_neural_net_b200 import synth


def all_trit_vectors():
    """All 3^10 trit vectors, as an independent enumeration (itertools order)."""
    import itertools
    return np.array(list(itertools.product((-1, 0, 1), repeat=10)), dtype=np.int8)


def test_base3_exhaustive_bijection():
    t = all_trit_vectors()                        # 59049 x 10
    words = oracle.base3_pack(t).reshape(-1)       # one word per vector
    assert words.dtype == np.uint16
    assert words.max() == 59048 and words.min() == 0
    assert np.unique(words).size == 59049          # injective onto 0..59048
    back, bad = oracle.base3_unpack(words.reshape(-1, 1), 10)
    assert bad == 0 and np.array_equal(back, t)
    all_words = np.arange(59049, dtype=np.uint16).reshape(-1, 1)
    t2, bad2 = oracle.base3_unpack(all_words, 10)
    assert bad2 == 0
    assert np.array_equal(oracle.base3_pack(t2).reshape(-1), all_words.reshape(-1))


def test_base3_words_above_range_are_flagged():
    w = np.array([[59049], [65535], [59048]], dtype=np.uint16)
    _, bad = oracle.base3_unpack(w, 10)
    assert bad == 2


def test_base3_golden_words():
    for line in golden_lines("base3_words.txt"):
        f = line.split()
        word, t = int(f[0]), np.array([[int(v) for v in f[1:]]], dtype=np.int8)
        assert int(oracle.base3_pack(t)[0, 0]) == word
        back, bad = oracle.base3_unpack(np.array([[word]], np.uint16), 10)
        assert bad == 0 and np.array_equal(back, t)


@pytest.mark.parametrize("k", [1, 9, 10, 11, 19, 20, 21, 4096])
def test_base3_row_padding(k):
    """Rows are packed independently; trits past k are 0 (digit 1)."""
    rng = np.random.default_rng(k)
    t = rng.integers(-1, 2, (3, k)).astype(np.int8)
    p = oracle.base3_pack(t)
    assert p.shape == (3, (k + 9) // 10)
    back, bad = oracle.base3_unpack(p, k)
    assert bad == 0 and np.array_equal(back, t)
    padded = np.zeros((3, 10 * p.shape[1]), np.int8)
    padded[:, :k] = t
    back_full, _ = oracle.base3_unpack(p, 10 * p.shape[1])
    assert np.array_equal(back_full, padded)
    # word j depends only on trits 10j..10j+9: one word per 10-trit slice
    for j in range(p.shape[1]):
        assert np.array_equal(oracle.base3_pack(padded[:, 10 * j: 10 * j + 10])[:, 0], p[:, j])


def _twn_cases():
    lines = list(golden_lines("twn_small.txt"))
    i = 0
    while i < len(lines):
        _, name, rows, cols = lines[i].split()
        rows, cols = int(rows), int(cols)
        w = np.array([[float(v) for v in lines[i + 1 + r].split()] for r in range(rows)], np.float32)
        d = lines[i + 1 + rows].split()[1]
        tr, sc = [], []
        for r in range(rows):
            a, b = lines[i + 2 + rows + r].split("|")
            tr.append([int(v) for v in a.split()])
            sc.append(float(b))
        yield name, w, (None if d == "-" else int(d, 16)), np.array(tr, np.int8), np.array(sc, np.float32)
        i += 2 + 2 * rows


@pytest.mark.parametrize("case", list(_twn_cases()), ids=lambda c: c[0])
def test_twn_golden(case):
    _, w, delta_bits, trits, scales = case
    t, s, d = oracle.twn_ternarize(w)
    if delta_bits is not None:
        assert int(np.array([d], np.float32).view(np.uint32)[0]) == delta_bits
    assert np.array_equal(t, trits)
    assert np.array_equal(s, scales)


def test_twn_constant_magnitude_rows_reconstruct_exactly():
    rng = np.random.default_rng(21)
    c = np.float32(rng.random() * 4 + 0.1)
    signs = np.where(rng.random((5, 33)) < 0.5, 1, -1).astype(np.float32)
    w = c * signs
    t, s, d = oracle.twn_ternarize(w)
    assert np.array_equal(t, signs.astype(np.int8))
    assert np.all(s == c)
    assert d == np.float32(0.7 * np.float64(c))


def test_twn_least_squares_optimal():
    """For the oracle's trits, its scale minimises sum (w - s t)^2 per row: a
    perturbation either way does not lower the error (textbook LS)."""
    w = synth.normal_f32(3, 1, (16, 300)).astype(np.float64)
    t, s, _ = oracle.twn_ternarize(w.astype(np.float32))
    t = t.astype(np.float64)
    for r in range(16):
        def err(sc):
            return float(((w[r] - sc * t[r]) ** 2).sum())
        s_ls = float((w[r] * t[r]).sum() / (t[r] * t[r]).sum())   # numpy normal equations
        assert abs(float(s[r]) - s_ls) <= 2e-7 * s_ls
        for eps in (1e-3, 1e-5):
            assert err(float(s[r])) <= err(float(s[r]) * (1 + eps))
            assert err(float(s[r])) <= err(float(s[r]) * (1 - eps))


def test_twn_gaussian_statistics():
    """For W ~ N(0,1): mean|W| -> sqrt(2/pi), Delta -> 0.7 sqrt(2/pi), the zero
    fraction -> erf(Delta/sqrt 2), and the mean scale -> E[|w| : |w| > Delta]
    = phi(Delta) / (1 - Phi(Delta))."""
    w = synth.normal_f32(4, 2, (512, 4096))
    t, s, d = oracle.twn_ternarize(w)
    delta_inf = 0.7 * math.sqrt(2 / math.pi)
    assert abs(float(d) - delta_inf) < 3e-3
    zero_frac = float((t == 0).mean())
    assert abs(zero_frac - math.erf(float(d) / math.sqrt(2))) < 3e-3
    phi = math.exp(-float(d) ** 2 / 2) / math.sqrt(2 * math.pi)
    tail = 0.5 * math.erfc(float(d) / math.sqrt(2))
    assert abs(float(s.mean()) - phi / tail) < 5e-3
    # trits agree with the sign of w wherever they are not zero, and |w| > Delta there
    nz = t != 0
    assert np.all(np.sign(w[nz]) == t[nz])
    assert np.all(np.abs(w[nz]) > d) and np.all(np.abs(w[~nz]) <= d)


def _bf16(x):
    return synth.bf16_bits_from_f32(np.asarray(x, np.float32))


def _bf16_to_f64_torch(bits):
    """Independent widening: torch's own bfloat16 -> float64 conversion."""
    t = torch.from_numpy(np.asarray(bits, np.uint16).astype(np.int16)).view(torch.bfloat16)
    return t.to(torch.float64).numpy()


def test_ternary_gemm_special_cases():
    k = 37
    xb = _bf16(synth.normal_f32(5, 1, (2, k)))
    xd = _bf16_to_f64_torch(xb)
    trits = np.zeros((4, k), np.int8)
    trits[0] = 1                 # all +1 -> s * sum x
    trits[2, 11] = 1             # one-hot +1 at 11 -> s * x_11
    trits[3, 30] = -1            # one-hot -1 at 30 -> -s * x_30
    scale = np.array([1.25, 3.0, 0.5, 2.0], np.float32)
    y, mag = oracle.ternary_gemm(xb, oracle.base3_pack(trits), scale, 2, 4, k)
    for i in range(2):
        assert y[i, 0] == pytest.approx(1.25 * xd[i].sum(), rel=1e-15, abs=1e-15)
        assert mag[i, 0] == pytest.approx(1.25 * np.abs(xd[i]).sum(), rel=1e-15)
        assert y[i, 1] == 0.0 and mag[i, 1] == 0.0
        assert y[i, 2] == 0.5 * xd[i, 11]
        assert y[i, 3] == -2.0 * xd[i, 30]


@pytest.mark.parametrize("m,n,k", [(1, 5, 10), (3, 7, 23), (4, 2, 95), (2, 3, 1)])
def test_ternary_gemm_against_numpy(m, n, k):
    rng = np.random.default_rng(m * 100 + n * 10 + k)
    trits = rng.integers(-1, 2, (n, k)).astype(np.int8)
    scale = (rng.random(n) + 0.5).astype(np.float32)
    xb = _bf16(rng.standard_normal((m, k)))
    y, mag = oracle.ternary_gemm(xb, oracle.base3_pack(trits), scale, m, n, k)
    xd = _bf16_to_f64_torch(xb)
    want = (xd @ trits.T.astype(np.float64)) * scale.astype(np.float64)[None, :]
    np.testing.assert_allclose(y, want, rtol=1e-12, atol=1e-12)
    want_mag = (np.abs(xd) @ np.abs(trits.T).astype(np.float64)) * scale.astype(np.float64)[None, :]
    np.testing.assert_allclose(mag, want_mag, rtol=1e-12, atol=1e-12)
    rows, cols = rng.integers(0, m, 9), rng.integers(0, n, 9)
    ys, ms = oracle.ternary_gemm_sampled(xb, oracle.base3_pack(trits), scale, m, n, k, rows, cols)
    assert np.array_equal(ys, y[rows, cols]) and np.array_equal(ms, mag[rows, cols])


def test_twn_steps_compose():
    w = synth.normal_f32(9, 3, (7, 45))
    t, s, d = oracle.twn_ternarize(w)
    assert oracle.twn_delta(w) == d
    t2, s2 = oracle.twn_apply(w, d)
    assert np.array_equal(t, t2) and np.array_equal(s, s2)
    # a larger threshold can only zero more trits
    t3, _ = oracle.twn_apply(w, np.float32(d * 2))
    assert np.all((t3 == 0) | (t3 == t)) and (t3 == 0).sum() >= (t == 0).sum()


def _mode_cases():
    lines = list(golden_lines("absmean_delta_small.txt"))
    i = 0
    while i < len(lines):
        _, name, rows, cols, param = lines[i].split()
        rows, cols = int(rows), int(cols)
        w = np.array([[float(v) for v in lines[i + 1 + r].split()] for r in range(rows)], np.float32)
        th = int(lines[i + 1 + rows].split()[1], 16)
        tr, sc = [], []
        for r in range(rows):
            a, b = lines[i + 2 + rows + r].split("|")
            tr.append([int(v) for v in a.split()])
            sc.append(float(b))
        yield name, w, (None if param == "-" else np.float32(param)), th, np.array(tr, np.int8), np.array(sc, np.float32)
        i += 2 + 2 * rows


@pytest.mark.parametrize("case", list(_mode_cases()), ids=lambda c: c[0])
def test_absmean_and_delta_golden(case):
    name, w, param, th_bits, trits, scales = case
    if param is None:
        t, s, g = oracle.absmean_ternarize(w)
        assert int(np.array([g], np.float32).view(np.uint32)[0]) == th_bits
    else:
        assert int(np.array([param], np.float32).view(np.uint32)[0]) == th_bits
        t, s = oracle.delta_ternarize(w, param)
    assert np.array_equal(t, trits)
    assert np.array_equal(s, scales)


@pytest.mark.parametrize("case", [c for c in _mode_cases() if c[2] is None], ids=lambda c: c[0])
def test_absmean_apply_golden(case):
    """The absmean trit rule at the golden gamma alone (the step the GPU
    parity test re-runs when the GPU's gamma is a neighbouring float32)."""
    name, w, _, th_bits, trits, scales = case
    g = np.array([th_bits], np.uint32).view(np.float32)[0]
    t, s = oracle.absmean_apply(w, g)
    assert np.array_equal(t, trits) and np.array_equal(s, scales)


@pytest.mark.parametrize("gamma", [0.3, 0.7978846, 1.0, 2.5])
def test_absmean_apply_is_roundclip_at_any_gamma(gamma):
    """At a gamma that is not the tensor's own mean, the trits are still
    numpy's RoundClip of the float32 quotient (np.round: half to even), and
    the scales the least-squares mean of |w| over the non-zero trits."""
    w = synth.normal_f32(21, 4, (48, 301))
    g = np.float32(gamma)
    w[0, :4] = [g * np.float32(0.5), -g * np.float32(0.5), g * np.float32(1.5), -g * np.float32(2.5)]
    t, s = oracle.absmean_apply(w, g)
    want = np.clip(np.round((w / g).astype(np.float32)), -1, 1).astype(np.int8)
    assert np.array_equal(t, want)
    kept = np.abs(w.astype(np.float64)) * (t != 0)
    cnt = (t != 0).sum(axis=1)
    want_s = np.where(cnt > 0, kept.sum(axis=1) / np.maximum(cnt, 1), 0).astype(np.float32)
    assert np.array_equal(s, want_s)
    # a larger gamma can only zero more trits
    t2, _ = oracle.absmean_apply(w, np.float32(gamma * 1.5))
    assert np.all((t2 == 0) | (t2 == t)) and (t2 == 0).sum() >= (t == 0).sum()


def test_absmean_apply_tells_neighbouring_gammas_apart():
    """Re-running the trit rule at the GPU's gamma matters: a weight at exactly
    half of the next float32 above gamma is a tie (trit 0) there and a
    non-zero trit at gamma itself."""
    g = np.float32(0.7978846)
    g_up = np.nextafter(g, np.float32(np.inf))
    w = np.array([[g_up * np.float32(0.5), -(g_up * np.float32(0.5)), 1.0]], np.float32)
    t_g, _ = oracle.absmean_apply(w, g)
    t_up, _ = oracle.absmean_apply(w, g_up)
    assert t_g.tolist() == [[1, -1, 1]] and t_up.tolist() == [[0, 0, 1]]


def test_absmean_ternarize_is_gamma_then_apply():
    w = synth.normal_f32(22, 4, (17, 555))
    t, s, g = oracle.absmean_ternarize(w)
    assert g == np.float32(np.abs(w.astype(np.float64)).mean())
    t2, s2 = oracle.absmean_apply(w, g)
    assert np.array_equal(t, t2) and np.array_equal(s, s2)
    t0, s0 = oracle.absmean_apply(w, np.float32(0))
    assert not t0.any() and not s0.any()


def test_absmean_is_roundclip_of_numpy():
    """The absmean trits equal numpy's own RoundClip (np.round is half-to-even)
    of the float32 quotient, with gamma the float64 mean rounded to float32."""
    w = synth.normal_f32(11, 4, (64, 777))
    t, s, g = oracle.absmean_ternarize(w)
    g_np = np.float32(np.abs(w.astype(np.float64)).mean())
    assert g == g_np
    q = (w / g_np).astype(np.float32)
    want = np.clip(np.round(q), -1, 1).astype(np.int8)
    assert np.array_equal(t, want)
    _, s_ls = oracle.twn_apply(w, np.float32(0))  # same LS rule, given the trits below
    kept = np.abs(w.astype(np.float64)) * (t != 0)
    cnt = (t != 0).sum(axis=1)
    want_s = np.where(cnt > 0, kept.sum(axis=1) / np.maximum(cnt, 1), 0).astype(np.float32)
    assert np.array_equal(s, want_s)


def test_absmean_gaussian_statistics():
    """For N(0,1): gamma -> sqrt(2/pi) and the zero fraction -> erf(gamma / (2 sqrt 2))."""
    w = synth.normal_f32(12, 5, (512, 4096))
    t, s, g = oracle.absmean_ternarize(w)
    assert abs(float(g) - math.sqrt(2 / math.pi)) < 3e-3
    assert abs(float((t == 0).mean()) - math.erf(float(g) / (2 * math.sqrt(2)))) < 3e-3


def test_delta_mode_equals_threshold_rule():
    w = synth.normal_f32(13, 6, (9, 100))
    F = np.float32(0.8)
    t, s = oracle.delta_ternarize(w, F)
    assert np.array_equal(t, (np.sign(w) * (np.abs(w) > F)).astype(np.int8))


def test_ternary_linear_adds_the_bias():
    k = 31
    xb = _bf16(synth.normal_f32(6, 1, (2, k)))
    trits = np.zeros((3, k), np.int8)
    trits[0] = 1
    trits[2, 5] = -1
    scale = np.array([1.5, 2.0, 0.25], np.float32)
    bias = np.array([0.5, -3.0, 8.0], np.float32)
    packed = oracle.base3_pack(trits)
    y0, m0 = oracle.ternary_gemm(xb, packed, scale, 2, 3, k)
    y, mag = oracle.ternary_linear(xb, packed, scale, bias, 2, 3, k)
    assert np.array_equal(y, y0 + bias.astype(np.float64)[None, :])
    assert np.array_equal(mag, m0 + np.abs(bias).astype(np.float64)[None, :])
    assert np.all(y[:, 1] == -3.0)          # all-zero trits: the bias alone
    yn, mn = oracle.ternary_linear(xb, packed, scale, None, 2, 3, k)
    assert np.array_equal(yn, y0) and np.array_equal(mn, m0)


# ---------------------------------------------------------------------------
# Index + sign sparse encoding ("Features": sparse encoding for high-sparsity
# layers; Packer.pack_sparse)
# ---------------------------------------------------------------------------
def test_sparse_encoding_by_hand():
    trits = np.zeros((3, 20), np.int8)
    trits[0, [0, 5, 19]] = [1, -1, 1]
    trits[2, 7] = -1               # row 1 empty
    row_ptr, ent = oracle.sparse_encode(trits)
    assert row_ptr.tolist() == [0, 3, 3, 4]
    assert ent.tolist() == [0, 5 | 0x8000, 19, 7 | 0x8000]


@pytest.mark.parametrize("n,k,density", [(5, 1, 0.5), (7, 33, 0.1), (4, 4096, 0.58), (3, 32768, 0.02),
                                         (6, 100, 1.0), (2, 50, 0.0)])
def test_sparse_round_trip_and_counts(n, k, density):
    rng = np.random.default_rng(n * k)
    trits = (rng.integers(0, 2, (n, k)) * 2 - 1).astype(np.int8) * (rng.random((n, k)) < density)
    row_ptr, ent = oracle.sparse_encode(trits)
    assert row_ptr[0] == 0 and np.all(np.diff(row_ptr) == (trits != 0).sum(axis=1))
    back, bad = oracle.sparse_decode(row_ptr, ent, n, k)
    assert bad == 0 and np.array_equal(back, trits)


def test_sparse_decode_flags_malformed_entries():
    row_ptr = np.array([0, 3], np.int64)
    ent = np.array([4, 4, 9], np.uint16)        # repeated position, position >= k
    _, bad = oracle.sparse_decode(row_ptr, ent, 1, 8)
    assert bad == 2


@pytest.mark.parametrize("m,n,k", [(1, 9, 130), (3, 5, 4096), (2, 4, 1)])
def test_sparse_gemm_equals_dense_ternary_layer(m, n, k):
    """The sparse layer over the entries of a trit matrix is the dense ternary
    layer over the same trits (the dense oracle is pinned above)."""
    rng = np.random.default_rng(m + n + k)
    trits = rng.integers(-1, 2, (n, k)).astype(np.int8) * (rng.random((n, k)) < 0.3)
    scale = (rng.random(n) + 0.5).astype(np.float32)
    bias = rng.standard_normal(n).astype(np.float32)
    xb = _bf16(rng.standard_normal((m, k)))
    row_ptr, ent = oracle.sparse_encode(trits)
    y, mag = oracle.sparse_gemm(xb, row_ptr, ent, scale, bias, m, n, k)
    yd, md = oracle.ternary_linear(xb, oracle.base3_pack(trits), scale, bias, m, n, k)
    np.testing.assert_allclose(y, yd, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(mag, md, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------------------
# .tbin files ("BalancedTernaryEngine" README, ".tbin Format")
# ---------------------------------------------------------------------------
def golden_tbin_files():
    files, cur = {}, None
    for line in golden_lines("tbin_small.txt"):
        if line.startswith("file "):
            cur = line.split()[1]
            files[cur] = bytearray()
        else:
            files[cur] += bytes.fromhex(line.split("#")[0])
    return {k: bytes(v) for k, v in files.items()}


def test_tbin_golden_files():
    from oracle import tbin
    f = golden_tbin_files()
    ver, meta, recs = tbin.read(f["v2"])
    assert ver == 2 and meta == b"{}" and len(recs) == 2
    t, r = recs
    assert (t["kind"], t["name"], t["out_feat"], t["in_feat"]) == ("ternary", "ab", 1, 3)
    assert t["delta"] == 0.5 and t["sparsity"] == 0.0 and t["biases"] is None
    assert t["scales"].tolist() == [1.0] and t["words"].tolist() == [5]
    assert oracle.base3_unpack(t["words"].reshape(1, 1), 3)[0].tolist() == [[1, 0, -1]]
    assert (r["kind"], r["name"], r["dims"], r["data"].tolist()) == ("raw", "n", [2], [1.0, -2.0])
    ver, meta, recs = tbin.read(f["v1"])
    (t,) = recs
    assert ver == 1 and meta == b"" and (t["name"], t["out_feat"], t["in_feat"]) == ("w", 2, 11)
    assert t["delta"] == np.float32(0.1) and t["sparsity"] == 0.25
    assert t["scales"].tolist() == [2.0, 0.5] and t["biases"].tolist() == [1.0, -1.0]
    trits, bad = oracle.base3_unpack(t["words"].reshape(2, 2), 11)
    assert bad == 0
    assert trits[0].tolist() == [1, 1, -1, -1, 0, 0, 0, 0, 0, 0, 1]
    assert trits[1].tolist() == [-1, -1, 1, 0, 1, -1, -1, -1, -1, -1, -1]
    # the writer reproduces both files byte for byte
    assert tbin.write([dict(kind="ternary", name="ab", out_feat=1, in_feat=3, delta=0.5, sparsity=0.0,
                            scales=[1.0], biases=None, words=[5]),
                       dict(kind="raw", name="n", dims=[2], data=[1.0, -2.0])]) == f["v2"]
    assert tbin.write([dict(kind="ternary", name="w", out_feat=2, in_feat=11, delta=np.float32(0.1), sparsity=0.25,
                            scales=[2.0, 0.5], biases=[1.0, -1.0], words=[29492, 29525, 207, 29523])],
                      metadata=b"", version=1) == f["v1"]


def test_tbin_rejects_malformed_files():
    from oracle import tbin
    f = golden_tbin_files()["v2"]
    for bad in (b"XBN\0" + f[4:], f[:-1], f[:20]):
        with pytest.raises((ValueError, IndexError, Exception)):
            tbin.read(bad)
