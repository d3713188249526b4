"""The chunked (WY/UT) form reaches the stepwise oracle's result.

The leaderboard commentary (section 二.1) names two paths of one recurrence:
chunked prefill (chunk 64) and stepwise decode. Agreement of the numpy
chunked form with the C++ stepwise oracle to ~1e-12, for several chunk sizes,
ragged tails and carried states, pins both (they share no code), and checks
the chunk formulas the CUDA prefill kernel implements.
"""
import numpy as np
import pytest

import oracle
from oracle import chunked


def case(T, d=16, H_k=1, H_v=3, seed=0, long_memory=False):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((T, H_k, d))
    k = rng.standard_normal((T, H_k, d))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    q /= np.linalg.norm(q, axis=-1, keepdims=True)
    v = rng.standard_normal((T, H_v, d))
    g = np.exp(-np.logaddexp(0, rng.standard_normal((T, H_v))))
    b = 1 / (1 + np.exp(-rng.standard_normal((T, H_v))))
    if long_memory:
        g = g ** 0.01
        b = np.ones_like(b)
    return q, k, v, g, b


@pytest.mark.parametrize("C", [1, 7, 64])
@pytest.mark.parametrize("long_memory", [False, True])
def test_chunked_equals_stepwise(C, long_memory):
    cu = np.array([0, 150, 151, 278])
    q, k, v, g, b = case(cu[-1], long_memory=long_memory)
    S0 = np.random.default_rng(1).standard_normal((3, 3, 16, 16)) * 0.1
    o_ref, S_ref = oracle.recurrence(q, k, v, g, b, S0, cu_seqlens=cu, scale=0.5)
    o, S = chunked.chunked(q, k, v, g, b, S0, cu_seqlens=cu, scale=0.5, chunk=C)
    np.testing.assert_allclose(o, o_ref, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(S, S_ref, rtol=1e-10, atol=1e-12)


def test_extreme_decay_no_overflow():
    """g ~ 1e-6 per token: cumulative log-decay inside a chunk reaches ~-880;
    only non-positive differences are exponentiated, so nothing overflows."""
    q, k, v, g, b = case(64)
    g = np.full_like(g, 1e-6)
    o_ref, S_ref = oracle.recurrence(q, k, v, g, b)
    with np.errstate(over="raise", invalid="raise"):
        o, S = chunked.chunked(q, k, v, g, b)
    np.testing.assert_allclose(o, o_ref, rtol=1e-10, atol=1e-14)
    np.testing.assert_allclose(S, S_ref, rtol=1e-10, atol=1e-14)


def test_rounding_helpers():
    assert chunked.round_bf16(1.0 + 2 ** -9) == 1.0            # tie -> even
    assert chunked.round_bf16(1.0 + 3 * 2 ** -9) == 1.0 + 2 ** -7
    assert chunked.round_fp16(1.0 + 2 ** -12) == 1.0
    assert chunked.round_fp16(65504.0) == 65504.0
    assert chunked.round_tf32(1.0 + 2 ** -11) == 1.0
    assert chunked.round_tf32(1.0 + 3 * 2 ** -11) == 1.0 + 2 ** -9
