"""Pins of the fp64 recurrence oracle against things other than itself.

The oracle steps S_t = g_t S_{t-1}(I - b_t k_t k_t^T) + b_t v_t k_t^T and
reads o_t = scale S_t q_t (gated delta rule, "Agnes-3.0-Flash Preview"
leaderboard commentary section 二.1 and model card 架构 table). These tests
check it against: a hand-derived worked example, the expanded product form
on tiny inputs, closed forms for special gates/keys, and split/packing
invariants. Each is chosen so that a dropped term, a wrong sign, a wrong time
index or a transposed state fails at least one of them.
"""
import numpy as np
import pytest

import oracle

RTOL = 1e-12


def rand_case(rng, T, d, H_k=1, H_v=1, unit_keys=False):
    q = rng.standard_normal((T, H_k, d))
    k = rng.standard_normal((T, H_k, d))
    if unit_keys:
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((T, H_v, d))
    g = rng.uniform(0.2, 1.0, (T, H_v))
    b = rng.uniform(0.0, 1.5, (T, H_v))
    return q, k, v, g, b


def product_form(S0, q, k, v, g, b, scale):
    """Expanded solution of the recurrence for one head:
    S_T = S0 P_1...P_T + sum_t b_t v_t k_t^T P_{t+1}...P_T,
    P_t = g_t (I - b_t k_t k_t^T); o_t from the prefix solution."""
    T, d = k.shape
    P = [g[t] * (np.eye(d) - b[t] * np.outer(k[t], k[t])) for t in range(T)]

    def solve(Tn):
        S = S0.copy()
        for t in range(Tn):
            S = S @ P[t]
        for t in range(Tn):
            term = b[t] * np.outer(v[t], k[t])
            for s in range(t + 1, Tn):
                term = term @ P[s]
            S = S + term
        return S

    o = np.stack([scale * solve(t + 1) @ q[t] for t in range(T)])
    return o, solve(T)


def test_hand_worked_example(golden):
    f = golden("recurrence_hand_d2.txt")
    S0 = np.array(f["S0"]).reshape(1, 1, 2, 2)
    q = np.array(f["q"]).reshape(2, 1, 2)
    k = np.array(f["k"]).reshape(2, 1, 2)
    v = np.array(f["v"]).reshape(2, 1, 2)
    g = np.array(f["g"]).reshape(2, 1)
    b = np.array(f["beta"]).reshape(2, 1)
    o, S = oracle.recurrence(q, k, v, g, b, S0)
    np.testing.assert_allclose(o.reshape(-1), f["o"], rtol=0, atol=1e-13)
    np.testing.assert_allclose(S.reshape(-1), f["S_final"], rtol=0, atol=1e-13)


@pytest.mark.parametrize("d", [1, 2, 4])
@pytest.mark.parametrize("T", [1, 3, 6])
def test_bruteforce_product_form(d, T):
    rng = np.random.default_rng(100 * d + T)
    q, k, v, g, b = rand_case(rng, T, d)
    S0 = rng.standard_normal((d, d))          # non-symmetric on purpose
    scale = 0.7
    o, S = oracle.recurrence(q, k, v, g, b, S0[None, None], scale=scale)
    o_ref, S_ref = product_form(S0, q[:, 0], k[:, 0], v[:, 0], g[:, 0],
                                b[:, 0], scale)
    np.testing.assert_allclose(S[0, 0], S_ref, rtol=RTOL, atol=1e-12)
    np.testing.assert_allclose(o[:, 0], o_ref, rtol=RTOL, atol=1e-12)


def test_beta_zero_pure_decay():
    rng = np.random.default_rng(1)
    T, d = 9, 5
    q, k, v, g, _ = rand_case(rng, T, d)
    S0 = rng.standard_normal((d, d))
    o, S = oracle.recurrence(q, k, v, g, np.zeros((T, 1)), S0[None, None])
    cum = np.cumprod(g[:, 0])
    np.testing.assert_allclose(S[0, 0], cum[-1] * S0, rtol=RTOL)
    for t in range(T):
        np.testing.assert_allclose(o[t, 0], cum[t] * S0 @ q[t, 0], rtol=1e-11,
                                   atol=1e-14)


def test_beta_zero_gate_one_is_identity():
    rng = np.random.default_rng(2)
    T, d = 7, 4
    q, k, v, _, _ = rand_case(rng, T, d)
    S0 = rng.standard_normal((d, d))
    o, S = oracle.recurrence(q, k, v, np.ones((T, 1)), np.zeros((T, 1)),
                             S0[None, None])
    np.testing.assert_array_equal(S[0, 0], S0)
    np.testing.assert_allclose(o[:, 0], q[:, 0] @ S0.T, rtol=1e-13)


def test_beta_one_unit_key_writes_value():
    """beta=1, |k|=1: S_t k_t = v_t whatever g_t and S_{t-1} are; reading
    with q_t = k_t returns v_t."""
    rng = np.random.default_rng(3)
    T, d = 12, 8
    _, k, v, g, _ = rand_case(rng, T, d, unit_keys=True)
    S0 = rng.standard_normal((1, 1, d, d))
    o, _ = oracle.recurrence(k, k, v, g, np.ones((T, 1)), S0)
    np.testing.assert_allclose(o, v, rtol=0, atol=1e-12)


def test_orthonormal_keys_associative_memory():
    """g=1, beta=1, orthonormal keys e_1..e_T: S_T = S0 (I - sum e e^T) +
    sum v_t e_t^T, so querying e_t after all writes returns v_t."""
    rng = np.random.default_rng(4)
    d, T = 8, 5
    E, _ = np.linalg.qr(rng.standard_normal((d, d)))
    keys = E.T[:T]                               # orthonormal rows
    v = rng.standard_normal((T, 1, d))
    S0 = rng.standard_normal((d, d))
    q = np.repeat(keys[-1:], T, axis=0)[:, None]
    _, S = oracle.recurrence(q, keys[:, None], v, np.ones((T, 1)),
                             np.ones((T, 1)), S0[None, None])
    expect = S0 @ (np.eye(d) - keys.T @ keys) + v[:, 0].T @ keys
    np.testing.assert_allclose(S[0, 0], expect, rtol=0, atol=1e-12)
    for t in range(T):
        np.testing.assert_allclose(S[0, 0] @ keys[t], v[t, 0], atol=1e-12)


def test_scalar_d1_matches_closed_form_sum():
    """d=1: s_T = s0 prod_t a_t + sum_t b_t v_t k_t prod_{s>t} a_s with
    a_t = g_t (1 - b_t k_t^2)."""
    rng = np.random.default_rng(5)
    T = 20
    q, k, v, g, b = rand_case(rng, T, 1)
    s0 = 0.3
    _, S = oracle.recurrence(q, k, v, g, b, np.full((1, 1, 1, 1), s0))
    a = g[:, 0] * (1 - b[:, 0] * k[:, 0, 0] ** 2)
    expect = s0 * np.prod(a) + sum(
        b[t, 0] * v[t, 0, 0] * k[t, 0, 0] * np.prod(a[t + 1:]) for t in range(T))
    assert abs(S[0, 0, 0, 0] - expect) < 1e-12


@pytest.mark.parametrize("split", [1, 17, 39])
def test_split_carry_invariance(split):
    rng = np.random.default_rng(6)
    T, d = 40, 6
    q, k, v, g, b = rand_case(rng, T, d, H_k=1, H_v=3)
    S0 = rng.standard_normal((1, 3, d, d))
    o, S = oracle.recurrence(q, k, v, g, b, S0)
    o1, S1 = oracle.recurrence(q[:split], k[:split], v[:split], g[:split],
                               b[:split], S0)
    o2, S2 = oracle.recurrence(q[split:], k[split:], v[split:], g[split:],
                               b[split:], S1)
    np.testing.assert_allclose(np.concatenate([o1, o2]), o, rtol=1e-13,
                               atol=1e-13)
    np.testing.assert_allclose(S2, S, rtol=1e-13, atol=1e-13)


def test_packed_varlen_equals_separate_runs():
    rng = np.random.default_rng(7)
    lens = [1, 5, 0, 13]
    cu = np.concatenate([[0], np.cumsum(lens)])
    T, d = cu[-1], 4
    q, k, v, g, b = rand_case(rng, T, d, H_k=2, H_v=6)
    S0 = rng.standard_normal((len(lens), 6, d, d))
    o, S = oracle.recurrence(q, k, v, g, b, S0, cu_seqlens=cu)
    for n in range(len(lens)):
        a, e = cu[n], cu[n + 1]
        on, Sn = oracle.recurrence(q[a:e], k[a:e], v[a:e], g[a:e], b[a:e],
                                   S0[n:n + 1])
        np.testing.assert_array_equal(o[a:e], on)
        np.testing.assert_array_equal(S[n], Sn[0])
    # an empty sequence passes its state through unchanged
    np.testing.assert_array_equal(S[2], S0[2])


def test_gqa_group_mapping():
    """Value head h reads key/query head h // (H_v / H_k) (contiguous
    groups of 3 for 16 key / 48 value heads)."""
    rng = np.random.default_rng(8)
    T, d, H_k, H_v = 6, 3, 2, 6
    q, k, v, g, b = rand_case(rng, T, d, H_k=H_k, H_v=H_v)
    o, S = oracle.recurrence(q, k, v, g, b)
    for h in range(H_v):
        kh = h // 3
        o_ref, S_ref = product_form(np.zeros((d, d)), q[:, kh], k[:, kh],
                                    v[:, h], g[:, h], b[:, h], 1.0)
        np.testing.assert_allclose(o[:, h], o_ref, rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(S[0, h], S_ref, rtol=1e-12, atol=1e-13)


def test_scale_only_scales_output():
    rng = np.random.default_rng(9)
    q, k, v, g, b = rand_case(rng, 10, 4)
    o1, S1 = oracle.recurrence(q, k, v, g, b, scale=1.0)
    o2, S2 = oracle.recurrence(q, k, v, g, b, scale=128 ** -0.5)
    np.testing.assert_array_equal(S1, S2)
    np.testing.assert_allclose(o2, o1 * 128 ** -0.5, rtol=1e-14)


def test_thread_count_does_not_change_result():
    rng = np.random.default_rng(10)
    q, k, v, g, b = rand_case(rng, 30, 8, H_k=2, H_v=6)
    r1 = oracle.recurrence(q, k, v, g, b, threads=1)
    r4 = oracle.recurrence(q, k, v, g, b, threads=4)
    for a, c in zip(r1, r4):
        np.testing.assert_array_equal(a, c)
