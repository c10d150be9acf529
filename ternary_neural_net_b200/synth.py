"""Seeded synthetic inputs for the packed 1-bit / balanced-ternary matmul.

This module only draws random numbers and lays them out; it holds none of the
method's arithmetic (no sign packing, no dot products, no ternarisation, no
base-3 coding).  Both the CUDA path (tests, bench) and the CPU oracle are fed
from here, so the two sides always see the same bytes.

Generator: SplitMix64 (Steele, Lea & Flood, "Fast splittable pseudorandom
number generators", OOPSLA 2014), used in counter mode: draw i of a stream is
mix(key + (i + 1) * 0x9E3779B97F4A7C15).  Streams are told apart by a 64-bit
stream id folded into the key, so every tensor of a workload has its own
independent sequence and any tensor can be regenerated alone.

Distributions (the recipe is stated once here and nowhere else):
  * fair coins: raw 64-bit draws used as packed sign words, with the bits past
    the logical length of each row cleared (pad bits are 0, i.e. +1);
  * U(0,1]: ((u >> 11) + 1) * 2**-53;
  * N(0,1): Box-Muller cosine branch on two U(0,1] draws, computed in float64,
    rounded once to float32;
  * U(a,b) float32: a + (b - a) * U(0,1] in float64, rounded once to float32;
  * bf16: round-to-nearest-even of the float32 value (the float32 draws here are
    finite, so no NaN handling is needed).
"""
from __future__ import annotations

import numpy as np

_GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)


def _mix(z: np.ndarray) -> np.ndarray:
    """SplitMix64 output function on a uint64 array (wrapping arithmetic)."""
    z = np.asarray(z, dtype=np.uint64).copy()
    with np.errstate(over="ignore"):
        z ^= z >> np.uint64(30)
        z *= _M1
        z ^= z >> np.uint64(27)
        z *= _M2
        z ^= z >> np.uint64(31)
    return z


def _key(seed: int, stream: int) -> np.uint64:
    s = _mix(np.array([np.uint64(seed & 0xFFFFFFFFFFFFFFFF)]))[0]
    t = _mix(np.array([np.uint64(stream & 0xFFFFFFFFFFFFFFFF) ^ np.uint64(0xD1B54A32D192ED03)]))[0]
    return np.uint64(s ^ t)


def u64(seed: int, stream: int, count: int) -> np.ndarray:
    """`count` raw 64-bit draws of stream `stream` under `seed`."""
    key = _key(seed, stream)
    with np.errstate(over="ignore"):
        ctr = (np.arange(1, count + 1, dtype=np.uint64) * _GOLDEN) + key
    return _mix(ctr)


def uniform01(seed: int, stream: int, count: int) -> np.ndarray:
    """U(0,1] in float64 (53-bit grid, never 0)."""
    u = u64(seed, stream, count)
    return ((u >> np.uint64(11)).astype(np.float64) + 1.0) * (2.0 ** -53)


def normal_f32(seed: int, stream: int, shape) -> np.ndarray:
    """N(0,1) float32 of the given shape (Box-Muller, cosine branch, float64)."""
    count = int(np.prod(shape, dtype=np.int64))
    u1 = uniform01(seed, (1 << 32) + 2 * stream, count)
    u2 = uniform01(seed, (1 << 32) + 2 * stream + 1, count)
    z = np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * np.pi * u2)
    return z.astype(np.float32).reshape(shape)


def uniform_f32(seed: int, stream: int, shape, lo: float, hi: float) -> np.ndarray:
    count = int(np.prod(shape, dtype=np.int64))
    u = uniform01(seed, stream, count)
    return (lo + (hi - lo) * u).astype(np.float32).reshape(shape)


def words_per_row(k: int) -> int:
    """Number of 64-bit words that hold k sign bits (ceil(k/64))."""
    return (k + 63) // 64


def trit_words_per_row(k: int) -> int:
    """Number of 16-bit words that hold k trits at 10 per word (ceil(k/10))."""
    return (k + 9) // 10


def fair_coin_words(seed: int, stream: int, rows: int, k: int) -> np.ndarray:
    """[rows, ceil(k/64)] uint64 of iid fair-coin bits, pad bits (>= k) cleared."""
    kw = words_per_row(k)
    w = u64(seed, stream, rows * kw).reshape(rows, kw)
    tail = k - 64 * (kw - 1) if kw else 0
    if kw and tail < 64:
        w[:, kw - 1] &= np.uint64((1 << tail) - 1)
    return w


def bf16_bits_from_f32(x: np.ndarray) -> np.ndarray:
    """Round-to-nearest-even float32 -> bfloat16, returned as uint16 bit patterns."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    rounded = (b + np.uint64(0x7FFF) + ((b >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    return rounded.astype(np.uint16).reshape(np.shape(x))


def bf16_bits_to_f32(h: np.ndarray) -> np.ndarray:
    """Exact widening of bfloat16 bit patterns to float32."""
    return (np.asarray(h, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def mean_abs_rows_f32(w: np.ndarray) -> np.ndarray:
    """Per-row mean of |w| in float64, rounded once to float32.

    This is the per-output-channel alpha the workloads below are defined with
    (harness-side input preparation, not a step of the kernel path)."""
    return np.abs(np.asarray(w, dtype=np.float64)).mean(axis=1).astype(np.float32)


# ----------------------------------------------------------------------------
# The five workloads.  Each returns a dict of host numpy arrays.  Stream ids are
# fixed per tensor so that any tensor can be regenerated alone.
# ----------------------------------------------------------------------------

def gemv_small(seed: int = 1):
    """M=1, K=1000 (16 words, 24 pad bits), N=1024; fair-coin x and W; alpha from
    an independent N(0,1) float32 latent (alpha_n = mean |latent[n,:1000]|)."""
    m, n, k = 1, 1024, 1000
    latent = normal_f32(seed, 13, (n, k))
    return dict(m=m, n=n, k=k,
                xp=fair_coin_words(seed, 11, m, k),
                wp=fair_coin_words(seed, 12, n, k),
                alpha=mean_abs_rows_f32(latent))


def gemm_fused_pack(seed: int = 1, m: int = 256, n: int = 4096, k: int = 4096):
    """fp32 N(0,1) activations [m,k] (packed on device per call) and fp32 N(0,1)
    latent weights [n,k] (packed offline); alpha_n = mean |W[n,:]|."""
    x = normal_f32(seed, 21, (m, k))
    w = normal_f32(seed, 22, (n, k))
    return dict(m=m, n=n, k=k, x=x, w=w, alpha=mean_abs_rows_f32(w))


def gemv_ffn(seed: int = 1, n: int = 28672, k: int = 8192):
    """M=1, K=8192, N=28672: fair-coin packed weights, fp32 N(0,1) activations
    (packed on device), alpha ~ U(0.5,1.5)."""
    return dict(m=1, n=n, k=k,
                x=normal_f32(seed, 31, (1, k)),
                wp=fair_coin_words(seed, 32, n, k),
                alpha=uniform_f32(seed, 33, (n,), 0.5, 1.5))


def gemm_large(seed: int = 1, m: int = 8192, n: int = 8192, k: int = 8192):
    """M=N=K=8192 fair-coin activations and weights, pre-packed; alpha ~ U(0.5,1.5)."""
    return dict(m=m, n=n, k=k,
                xp=fair_coin_words(seed, 41, m, k),
                wp=fair_coin_words(seed, 42, n, k),
                alpha=uniform_f32(seed, 43, (n,), 0.5, 1.5))


def ternary(seed: int = 1, m: int = 1, n: int = 11008, k: int = 4096):
    """fp32 N(0,1) weights [n,k] (ternarised on device) and bf16 N(0,1)
    activations [m,k] as uint16 bit patterns."""
    return dict(m=m, n=n, k=k,
                w=normal_f32(seed, 51, (n, k)),
                x_bf16=bf16_bits_from_f32(normal_f32(seed, 52, (m, k))))
