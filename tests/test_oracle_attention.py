"""Pins for the oracle's global-attention layer (fp64).

The layer (Agnes-3.0-Flash Preview model card, section 架构, rows 全局注意力
and 位置编码; leaderboard commentary, section 二.1): RMS-norm on q and k,
three-axis rotary on the first 64 dims of each head (base 1e7, axes
interleaved 11 : 11 : 10), causal GQA softmax attention, sigmoid output gate.

Each pin fixes the oracle to something outside its own code:

* a two-token case worked by hand (``tests/golden/attention_hand_two_tokens.txt``,
  a closed form in cos 1);
* the rotary of a basis vector is cos / sin of the textbook angle at the
  coupled dims (pairing, frequency ladder, direction), and only pairs on the
  axis that moved turn;
* a single key gives its value times the gate; keys that normalise to zero
  give the running mean of the values (the causal mask, to the token);
* rotary depends on position differences only; q and k are scale-free through
  their norms; a common factor on the norm weights equals that factor squared
  on the softmax scale;
* GQA equals multi-head attention on key/value heads repeated per group;
* an independent numpy formulation (complex rotation, masked softmax matrix)
  on ragged packed sequences with explicit three-axis positions.
"""
import os

import numpy as np
import pytest

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))


def rnd(seed, *shape):
    return np.random.default_rng(seed).standard_normal(shape)


def golden(name):
    vals = {}
    for line in open(os.path.join(HERE, "golden", name)):
        if line.startswith("#") or not line.strip():
            continue
        key, rest = line.split(":")
        vals[key.strip()] = np.array([float(x) for x in rest.split()])
    return vals


def test_two_tokens_worked_by_hand():
    g = golden("attention_hand_two_tokens.txt")
    e0 = np.array([1.0, 0.0])
    q = np.stack([e0, e0])[:, None, :]
    k = q.copy()
    v = np.array([[1.0, 0.0], [0.0, 1.0]])[:, None, :]
    out, _, _ = oracle.attention(q, k, v, np.zeros_like(q), np.ones(2), np.ones(2), eps=0.0,
                                 rope_dims=2, rope_base=10.0, scale=1.0)
    np.testing.assert_allclose(out[0, 0], g["out0"], atol=1e-10)
    np.testing.assert_allclose(out[1, 0], g["out1"], atol=1e-10)


@pytest.mark.parametrize("i", [0, 1, 5, 31])
def test_rotary_of_a_basis_vector(i):
    """x = e_i (dims 64 x 256 head): after the norm x = sqrt(D) e_i; the pair
    (i, i + 32) turns by theta = p * base^(-2i/64) counter-clockwise: dim i
    holds sqrt(D) cos theta and dim i + 32 holds sqrt(D) sin theta."""
    D, R, base, p = 256, 64, 1e7, 37
    x = np.zeros((p + 1, 1, D))
    x[:, 0, i] = 1.0
    _, qr, kr = oracle.attention(x, x, x, x, np.ones(D), np.ones(D), eps=0.0, rope_dims=R,
                                 rope_base=base)
    theta = p * base ** (-2.0 * i / R)
    want = np.zeros(D)
    want[i] = np.sqrt(D) * np.cos(theta)
    want[i + R // 2] = np.sqrt(D) * np.sin(theta)
    np.testing.assert_allclose(qr[p, 0], want, atol=1e-12)
    np.testing.assert_allclose(kr[p, 0], want, atol=1e-12)


def test_only_pairs_on_the_moved_axis_turn():
    """Positions (0, p, 0): pair i turns iff i % 3 == 1 (height); dims past 64
    never turn."""
    D, R, T = 256, 64, 1
    x = rnd(1, T, 1, D)
    pos = np.array([[0], [50], [0]])
    _, qr, _ = oracle.attention(x, x, x, x, np.ones(D), np.ones(D), positions=pos, eps=0.0)
    normed = x[0, 0] / np.sqrt(np.mean(x[0, 0] ** 2))
    for i in range(R // 2):
        same = np.allclose(qr[0, 0, [i, i + R // 2]], normed[[i, i + R // 2]], rtol=0,
                           atol=1e-14)
        assert same == (i % 3 != 1), i
    np.testing.assert_allclose(qr[0, 0, R:], normed[R:], atol=1e-12)


def test_first_token_is_its_value_times_the_gate():
    T, Hq, Hkv, D = 5, 6, 2, 32
    q, k, v, gate = rnd(2, T, Hq, D), rnd(3, T, Hkv, D), rnd(4, T, Hkv, D), rnd(5, T, Hq, D)
    cu = [0, 1, 1, 5]
    out, _, _ = oracle.attention(q, k, v, gate, np.ones(D), np.ones(D), cu_seqlens=cu,
                                 rope_dims=16)
    for t in (0, 1):   # each the first token of its sequence
        for h in range(Hq):
            np.testing.assert_allclose(out[t, h], v[t, h // 3] / (1 + np.exp(-gate[t, h])),
                                       rtol=1e-12)


def test_zero_keys_give_the_running_mean_of_the_values():
    """k = 0 normalises to 0 (eps > 0), so every score is 0 and token t
    averages the values of its own sequence's tokens 0..t."""
    T, Hq, Hkv, D = 9, 4, 2, 16
    q, v, gate = rnd(6, T, Hq, D), rnd(7, T, Hkv, D), rnd(8, T, Hq, D)
    cu = [0, 4, 9]
    out, _, _ = oracle.attention(q, np.zeros((T, Hkv, D)), v, gate, np.ones(D), np.ones(D),
                                 cu_seqlens=cu, rope_dims=8)
    for a, b in zip(cu[:-1], cu[1:]):
        for t in range(a, b):
            mean = v[a:t + 1].mean(axis=0)
            for h in range(Hq):
                np.testing.assert_allclose(out[t, h], mean[h // 2] / (1 + np.exp(-gate[t, h])),
                                           rtol=1e-12, atol=1e-14)


def test_rotary_is_relative():
    T, D = 12, 64
    q, k, v, gate = rnd(9, T, 2, D), rnd(10, T, 1, D), rnd(11, T, 1, D), rnd(12, T, 2, D)
    w = 1 + 0.3 * rnd(13, D)
    base, _, _ = oracle.attention(q, k, v, gate, w, w, rope_dims=32, rope_base=100.0)
    shifted, qr, _ = oracle.attention(q, k, v, gate, w, w, pos0=[1000], rope_dims=32,
                                      rope_base=100.0)
    np.testing.assert_allclose(shifted, base, rtol=1e-9, atol=1e-12)
    _, qr0, _ = oracle.attention(q, k, v, gate, w, w, rope_dims=32, rope_base=100.0)
    assert not np.allclose(qr, qr0)


def test_norms_make_q_and_k_scale_free_and_weights_act_as_scale():
    T, D = 10, 32
    q, k, v, gate = rnd(14, T, 3, D), rnd(15, T, 1, D), rnd(16, T, 1, D), rnd(17, T, 3, D)
    one = np.ones(D)
    a, _, _ = oracle.attention(q, k, v, gate, one, one, eps=0.0, rope_dims=16)
    b, _, _ = oracle.attention(7.5 * q, 0.2 * k, v, gate, one, one, eps=0.0, rope_dims=16)
    np.testing.assert_allclose(b, a, rtol=1e-10, atol=1e-13)
    c = 1.7
    w_scaled, _, _ = oracle.attention(q, k, v, gate, c * one, c * one, eps=0.0, rope_dims=16)
    s_scaled, _, _ = oracle.attention(q, k, v, gate, one, one, eps=0.0, rope_dims=16,
                                      scale=c * c * D ** -0.5)
    np.testing.assert_allclose(w_scaled, s_scaled, rtol=1e-10, atol=1e-13)
    plain, _, _ = oracle.attention(q, k, v, gate, one, one, eps=0.0, rope_dims=16)
    assert not np.allclose(w_scaled, plain)


def test_gqa_equals_mha_on_repeated_heads():
    T, Hq, Hkv, D = 11, 6, 2, 16
    q, k, v, gate = rnd(18, T, Hq, D), rnd(19, T, Hkv, D), rnd(20, T, Hkv, D), rnd(21, T, Hq, D)
    w = 1 + 0.2 * rnd(22, D)
    gqa, _, _ = oracle.attention(q, k, v, gate, w, w, rope_dims=8)
    rep = lambda a: np.repeat(a, Hq // Hkv, axis=1)
    mha, _, _ = oracle.attention(q, rep(k), rep(v), gate, w, w, rope_dims=8)
    np.testing.assert_allclose(gqa, mha, rtol=1e-12, atol=1e-14)


def numpy_attention(q, k, v, gate, wq, wk, cu, pos3, eps, R, base):
    """Separate formulation: rotary as multiplication of z = x_i + j x_{i+R/2}
    by exp(j theta); attention as one masked score matrix per sequence and head."""
    D = q.shape[-1]

    def norm_rope(x, w):
        y = x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps) * w
        freqs = base ** (-np.arange(R // 2) * 2.0 / R)
        theta = pos3[np.arange(R // 2) % 3].T * freqs             # [T, R/2]
        z = (y[..., :R // 2] + 1j * y[..., R // 2:R]) * np.exp(1j * theta)[:, None, :]
        return np.concatenate([z.real, z.imag, y[..., R:]], axis=-1)

    qr, kr = norm_rope(q, wq), norm_rope(k, wk)
    group = q.shape[1] // k.shape[1]
    out = np.zeros_like(q)
    for a, b in zip(cu[:-1], cu[1:]):
        L = b - a
        if L == 0:
            continue
        mask = np.tril(np.ones((L, L), dtype=bool))
        for h in range(q.shape[1]):
            s = qr[a:b, h] @ kr[a:b, h // group].T * D ** -0.5
            s = np.where(mask, s, -np.inf)
            p = np.exp(s - s.max(axis=1, keepdims=True))
            p /= p.sum(axis=1, keepdims=True)
            out[a:b, h] = (p @ v[a:b, h // group]) / (1 + np.exp(-gate[a:b, h]))
    return out, qr, kr


def test_against_a_separate_numpy_formulation():
    lens = [7, 0, 1, 13, 5]
    cu = np.concatenate([[0], np.cumsum(lens)])
    T, Hq, Hkv, D, R = int(cu[-1]), 6, 2, 48, 24
    q, k, v, gate = rnd(23, T, Hq, D), rnd(24, T, Hkv, D), rnd(25, T, Hkv, D), rnd(26, T, Hq, D)
    wq, wk = 1 + 0.3 * rnd(27, D), 1 + 0.3 * rnd(28, D)
    pos3 = np.random.default_rng(29).integers(0, 500, size=(3, T))
    got, qr, kr = oracle.attention(q, k, v, gate, wq, wk, cu_seqlens=cu, positions=pos3,
                                   eps=1e-6, rope_dims=R, rope_base=1e4)
    want, wqr, wkr = numpy_attention(q, k, v, gate, wq, wk, cu, pos3, 1e-6, R, 1e4)
    np.testing.assert_allclose(qr, wqr, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(kr, wkr, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(got, want, rtol=1e-10, atol=1e-12)


def test_selected_rows_equal_the_full_computation():
    T = 20
    q, k, v, gate = rnd(30, T, 2, 16), rnd(31, T, 1, 16), rnd(32, T, 1, 16), rnd(33, T, 2, 16)
    full, _, _ = oracle.attention(q, k, v, gate, np.ones(16), np.ones(16), rope_dims=8)
    part, _, _ = oracle.attention(q, k, v, gate, np.ones(16), np.ones(16), rope_dims=8,
                                  rows=[0, 7, 19])
    np.testing.assert_array_equal(part[[0, 7, 19]], full[[0, 7, 19]])
    assert not part[[1, 8, 18]].any()
