"""Pins for the oracle's binary path, against things other than itself:
numpy's own bit packing and popcount, numpy integer dot products, IEEE float32
multiplication, the printed edge-case rules and hand-written special values.

Pages: "Binary Math Effectiveness -- why / how / when", section 1 (encoding
table, identity <x,w> = n - 2d, XNOR form, "Edge cases"); "Architecture
Decision Record", "Decision" (binary_gemm_u64 over uint64 words)."""
import numpy as np
import pytest

import oracle
from conftest import golden_lines


def np_pack(pm1: np.ndarray) -> np.ndarray:
    """Independent packer for +-1 int arrays: numpy packbits (little bit order)
    of (value == -1), little-endian bytes grouped into uint64 words."""
    rows, k = pm1.shape
    kw = (k + 63) // 64
    bits = np.zeros((rows, 64 * kw), dtype=np.uint8)
    bits[:, :k] = (pm1 == -1)
    by = np.packbits(bits, axis=1, bitorder="little")
    return np.ascontiguousarray(by).view("<u8").reshape(rows, kw).astype(np.uint64)


def rand_pm1(rng, rows, k):
    return np.where(rng.random((rows, k)) < 0.5, 1, -1).astype(np.int64)


def test_pack_special_values_golden():
    for line in golden_lines("sign_pack_special.txt"):
        hexbits, bit, name = line.split()[:3]
        x = np.array([[int(hexbits, 16)]], dtype=np.uint32).view(np.float32)
        got = int(oracle.pack_signs(x)[0, 0])
        assert got == int(bit), name


@pytest.mark.parametrize("k", list(range(1, 65)) + [65, 127, 128, 129, 1000, 4096])
def test_pack_matches_numpy_packbits(k):
    rng = np.random.default_rng(1000 + k)
    x = rng.standard_normal((3, k)).astype(np.float32)
    x[0, :: max(1, k // 7)] = 0.0
    want = np_pack(np.where(x > 0, 1, -1))
    got = oracle.pack_signs(x)
    assert got.dtype == np.uint64 and got.shape == want.shape
    assert np.array_equal(got, want)
    assert oracle.count_pad_bits(got, k) == 0


def test_unpack_inverts_numpy_pack():
    rng = np.random.default_rng(7)
    for k in (1, 63, 64, 65, 200):
        v = rand_pm1(rng, 4, k)
        assert np.array_equal(oracle.unpack_signs(np_pack(v), k), v)


@pytest.mark.parametrize("n", range(0, 131))
def test_identity_against_bruteforce(n):
    """n - 2*popcount(x XOR w) (numpy bitwise_count on the packed words) and the
    brute-force +-1 dot (numpy int64) both equal the oracle's unpack-and-sum."""
    for seed in range(4):
        rng = np.random.default_rng(10_000 * seed + n)
        x = rand_pm1(rng, 1, n)
        w = rand_pm1(rng, 3, n)
        w[1] = x[0]
        w[2] = -x[0]
        xp, wp = np_pack(x), np_pack(w)
        alpha = np.ones(3, dtype=np.float32)
        dots, _ = oracle.binary_gemm(xp, wp, alpha, 1, 3, n)
        brute = (w @ x[0]).astype(np.int64)
        d = np.bitwise_count(xp[0][None, :] ^ wp).sum(axis=1).astype(np.int64) if n else np.zeros(3, np.int64)
        assert np.array_equal(dots[0], brute)
        assert np.array_equal(dots[0], n - 2 * d)
        assert dots[0, 1] == n and dots[0, 2] == -n


def test_xnor_form_equivalent():
    rng = np.random.default_rng(3)
    for n in (1, 64, 100, 128, 300):
        x, w = rand_pm1(rng, 1, n), rand_pm1(rng, 1, n)
        xp, wp = np_pack(x), np_pack(w)
        mask = np_pack(-np.ones((1, n), dtype=np.int64))  # ones on the n logical bits only
        agree = np.bitwise_count(~(xp ^ wp) & mask).sum()
        dots, _ = oracle.binary_gemm(xp, wp, np.ones(1, np.float32), 1, 1, n)
        assert dots[0, 0] == 2 * int(agree) - n


def test_n_zero_gives_zero():
    xp = np.zeros((2, 0), dtype=np.uint64)
    wp = np.zeros((3, 0), dtype=np.uint64)
    alpha = np.array([1.5, -2.0, 0.0], dtype=np.float32)
    dots, out = oracle.binary_gemm(xp, wp, alpha, 2, 3, 0)
    assert np.all(dots == 0) and np.all(out == 0)


def test_alpha_zero_gives_zero_and_identity_holds():
    rng = np.random.default_rng(5)
    x, w = rand_pm1(rng, 4, 77), rand_pm1(rng, 5, 77)
    alpha = np.zeros(5, dtype=np.float32)
    dots, out = oracle.binary_gemm(np_pack(x), np_pack(w), alpha, 4, 5, 77)
    assert np.all(out == 0.0)
    assert np.array_equal(dots, x @ w.T)


def test_padding_invariance():
    """Appending p entries equal to +1 to both vectors adds exactly p; pad bits
    (which encode +1) are never counted on their own."""
    rng = np.random.default_rng(11)
    for n in (1, 40, 63, 64, 65, 120):
        x, w = rand_pm1(rng, 1, n), rand_pm1(rng, 1, n)
        base = oracle.binary_gemm(np_pack(x), np_pack(w), np.ones(1, np.float32), 1, 1, n)[0][0, 0]
        for p in (1, 3, 64 - n % 64, 70):
            xe = np.concatenate([x, np.ones((1, p), np.int64)], axis=1)
            we = np.concatenate([w, np.ones((1, p), np.int64)], axis=1)
            ext = oracle.binary_gemm(np_pack(xe), np_pack(we), np.ones(1, np.float32), 1, 1, n + p)[0][0, 0]
            assert ext == base + p


@pytest.mark.parametrize("m,n,k", [(3, 7, 150), (7, 3, 129), (5, 5, 64)])
def test_rectangular_and_alpha_epilogue(m, n, k):
    """m != n either way catches a transposed operand or output; out equals the
    IEEE float32 product alpha_j * float32(dot) computed by numpy (bitwise)."""
    rng = np.random.default_rng(12 + m)
    x, w = rand_pm1(rng, m, k), rand_pm1(rng, n, k)
    alpha = (rng.random(n) * 3 - 1).astype(np.float32)
    alpha[2] = 0.0
    dots, out = oracle.binary_gemm(np_pack(x), np_pack(w), alpha, m, n, k)
    assert np.array_equal(dots, (x @ w.T).astype(np.int32))
    want = alpha[None, :] * dots.astype(np.float32)
    assert want.dtype == np.float32
    assert np.array_equal(out.view(np.uint32), want.view(np.uint32)) or np.array_equal(out, want)


def test_sampled_matches_full():
    rng = np.random.default_rng(13)
    m, n, k = 6, 9, 130
    xp, wp = np_pack(rand_pm1(rng, m, k)), np_pack(rand_pm1(rng, n, k))
    alpha = rng.random(n).astype(np.float32)
    dots, out = oracle.binary_gemm(xp, wp, alpha, m, n, k)
    rows = rng.integers(0, m, 40)
    cols = rng.integers(0, n, 40)
    sd, so = oracle.binary_gemm_sampled(xp, wp, alpha, m, n, k, rows, cols)
    assert np.array_equal(sd, dots[rows, cols]) and np.array_equal(so, out[rows, cols])


def test_pad_bit_counter_sees_planted_bit():
    xp = oracle.pack_signs(np.ones((1, 70), np.float32))
    assert oracle.count_pad_bits(xp, 70) == 0
    xp[0, 1] |= np.uint64(1) << np.uint64(9)
    assert oracle.count_pad_bits(xp, 70) == 1


# ---------------------------------------------------------------------------
# Fused layer epilogue: y = fl32(fl32(alpha * dot) + bias), next = sign pack of y
# ---------------------------------------------------------------------------
def test_linear_without_bias_is_the_gemm_and_its_pack():
    rng = np.random.default_rng(21)
    m, n, k = 5, 70, 200   # n past one word: pad bits in `next`
    xp, wp = np_pack(rand_pm1(rng, m, k)), np_pack(rand_pm1(rng, n, k))
    alpha = (rng.random(n) * 2 - 0.5).astype(np.float32)
    d, y, nxt = oracle.binary_linear(xp, wp, alpha, None, m, n, k)
    gd, go = oracle.binary_gemm(xp, wp, alpha, m, n, k)
    assert np.array_equal(d, gd) and np.array_equal(y.view(np.uint32), go.view(np.uint32))
    # the next layer's input, by an independent packer: bit j = !(y_j > 0)
    assert np.array_equal(nxt, np_pack(np.where(y > 0, 1, -1)))
    assert oracle.count_pad_bits(nxt, n) == 0


def test_linear_bias_special_cases():
    rng = np.random.default_rng(22)
    m, n, k = 3, 6, 129
    xp, wp = np_pack(rand_pm1(rng, m, k)), np_pack(rand_pm1(rng, n, k))
    alpha = (rng.random(n) + 0.5).astype(np.float32)
    _, y0, _ = oracle.binary_linear(xp, wp, alpha, None, m, n, k)
    # bias cancelling row 0 exactly: y = +0 there, which packs as -1 (0 is not > 0)
    bias = -y0[0].copy()
    _, y, nxt = oracle.binary_linear(xp, wp, alpha, bias, m, n, k)
    assert np.all(y[0] == 0.0) and not np.any(np.signbit(y[0]))
    assert int(nxt[0, 0]) == (1 << n) - 1
    # huge positive / negative bias forces every sign
    _, y, nxt = oracle.binary_linear(xp, wp, alpha, np.full(n, 1e30, np.float32), m, n, k)
    assert np.all(nxt == 0) and np.all(y == np.float32(1e30))
    _, _, nxt = oracle.binary_linear(xp, wp, alpha, np.full(n, -np.inf, np.float32), m, n, k)
    assert np.all(nxt[:, 0] == (1 << n) - 1)
    # one float32 addition after the rounded product: a bias below half an ulp of
    # y leaves y unchanged (no fused multiply-add)
    tiny = np.full(n, 1e-30, np.float32)
    _, yt, _ = oracle.binary_linear(xp, wp, alpha, tiny, m, n, k)
    assert np.array_equal(yt[y0 != 0], y0[y0 != 0])


def test_linear_bias_is_one_float32_addition():
    rng = np.random.default_rng(23)
    m, n, k = 4, 33, 300
    xp, wp = np_pack(rand_pm1(rng, m, k)), np_pack(rand_pm1(rng, n, k))
    alpha = (rng.random(n) * 3 - 1).astype(np.float32)
    bias = rng.standard_normal(n).astype(np.float32) * 20
    d, y, nxt = oracle.binary_linear(xp, wp, alpha, bias, m, n, k)
    want = (alpha[None, :] * d.astype(np.float32)) + bias[None, :]
    assert want.dtype == np.float32
    assert np.array_equal(y.view(np.uint32), want.view(np.uint32))
    assert np.array_equal(nxt, np_pack(np.where(want > 0, 1, -1)))
