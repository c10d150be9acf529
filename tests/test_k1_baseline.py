"""The CPU baseline restated from the pages' binary_gemm_u64 ("Architecture
Decision Record", "Decision": row-by-row XOR + 64-bit popcount) against the
oracle, which never counts bits: dots and alpha-scaled outputs bitwise equal,
on one thread and on several, across word boundaries and ragged sizes."""
import numpy as np
import pytest

import oracle
from ternary_neural_net_b200 import synth


@pytest.mark.parametrize("m,n,k", [(1, 1, 1), (3, 5, 63), (4, 7, 64), (5, 3, 65), (9, 17, 1000), (2, 3, 0),
                                   (16, 16, 4096 + 1)])
@pytest.mark.parametrize("threads", [1, 4])
def test_k1_matches_oracle(m, n, k, threads):
    xp = synth.fair_coin_words(m * 7 + k, 1, m, k)
    wp = synth.fair_coin_words(m * 7 + k, 2, n, k)
    alpha = synth.uniform_f32(k, 3, (n,), 0.5, 1.5)
    alpha[0] = 0.0
    d, o = oracle.k1_binary_gemm(xp, wp, alpha, m, n, k, threads)
    wd, wo = oracle.binary_gemm(xp, wp, alpha, m, n, k)
    assert np.array_equal(d, wd)
    assert np.array_equal(o.view(np.uint32) & np.uint32(0x7FFFFFFF), wo.view(np.uint32) & np.uint32(0x7FFFFFFF))
    assert np.array_equal(o, wo)


def test_k1_threads_used():
    assert oracle.k1_threads_used(1) == 1
    assert oracle.k1_threads_used(3) == 3
