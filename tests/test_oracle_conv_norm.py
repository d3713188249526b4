"""Pins of the oracle's causal conv (+SiLU, L2) and gated RMS-norm.

Sources: Agnes-3.0-Flash Preview model card, 架构 table (causal conv kernel 4
in front of the delta rule; gated RMS-norm on its output) and the leaderboard
commentary section 二.1 (kernel=4 causal conv). Pins: hand-worked examples,
numpy's own 1-D convolution as the brute-force reference, the identity-tap
special case, unit-norm and scale-invariance properties, history carry.
"""
import math

import numpy as np
import pytest

import oracle


def silu(a):
    return a / (1.0 + np.exp(-a))


def test_conv_hand_example_zero_history(golden):
    f = golden("conv_hand_c1.txt")
    x = np.array(f["x"])[:, None]
    y, st = oracle.conv1d_silu_l2(x, np.array(f["w"])[None])
    np.testing.assert_allclose(y[:, 0], silu(np.array(f["acc_A"])), rtol=1e-15)
    np.testing.assert_array_equal(st.reshape(-1), f["state_out"])


def test_conv_hand_example_carried_history(golden):
    f = golden("conv_hand_c1.txt")
    x = np.array(f["x"])[:, None]
    hist = np.array(f["history_B"]).reshape(1, 3, 1)
    y, _ = oracle.conv1d_silu_l2(x, np.array(f["w"])[None], conv_state_in=hist)
    np.testing.assert_allclose(y[:, 0], silu(np.array(f["acc_B"])), rtol=1e-15)


def test_conv_matches_numpy_convolve():
    """Causal depthwise conv == numpy.convolve of each channel with its
    reversed taps (full mode, first T outputs), with a bias."""
    rng = np.random.default_rng(0)
    T, C = 11, 5
    x = rng.standard_normal((T, C))
    w = rng.standard_normal((C, 4))
    bias = rng.standard_normal(C)
    y, _ = oracle.conv1d_silu_l2(x, w, bias=bias)
    for c in range(C):
        acc = np.convolve(x[:, c], w[c, ::-1], mode="full")[:T] + bias[c]
        np.testing.assert_allclose(y[:, c], silu(acc), rtol=1e-13, atol=1e-15)


def test_conv_identity_tap_is_silu():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((9, 3)) * 4
    w = np.tile([0.0, 0.0, 0.0, 1.0], (3, 1))
    y, _ = oracle.conv1d_silu_l2(x, w)
    np.testing.assert_allclose(y, silu(x), rtol=1e-15)
    assert silu(0.0) == 0.0 and abs(silu(50.0) - 50.0) < 1e-15


def test_l2_norm_of_qk_heads_and_passthrough_of_v():
    rng = np.random.default_rng(2)
    T, C = 6, 384          # two normalised heads, one raw head
    x = rng.standard_normal((T, C))
    w = rng.standard_normal((C, 4)) * 0.5
    y_raw, _ = oracle.conv1d_silu_l2(x, w, l2_channels=0)
    y, _ = oracle.conv1d_silu_l2(x, w, l2_channels=256, l2_eps=0.0)
    for h in range(2):
        sl = slice(128 * h, 128 * h + 128)
        np.testing.assert_allclose(np.linalg.norm(y[:, sl], axis=1), 1.0,
                                   rtol=1e-14)
        # direction is unchanged
        np.testing.assert_allclose(
            y[:, sl] * np.linalg.norm(y_raw[:, sl], axis=1, keepdims=True),
            y_raw[:, sl], rtol=1e-13, atol=1e-15)
    np.testing.assert_array_equal(y[:, 256:], y_raw[:, 256:])


@pytest.mark.parametrize("split", [1, 2, 3, 5])
def test_conv_history_carry_split(split):
    rng = np.random.default_rng(3)
    T, C = 8, 4
    x = rng.standard_normal((T, C))
    w = rng.standard_normal((C, 4))
    h0 = rng.standard_normal((1, 3, C))
    y, st = oracle.conv1d_silu_l2(x, w, conv_state_in=h0)
    y1, st1 = oracle.conv1d_silu_l2(x[:split], w, conv_state_in=h0)
    y2, st2 = oracle.conv1d_silu_l2(x[split:], w, conv_state_in=st1)
    np.testing.assert_array_equal(np.concatenate([y1, y2]), y)
    np.testing.assert_array_equal(st2, st)
    np.testing.assert_array_equal(st[0], x[-3:])


def test_conv_short_sequence_state_shift():
    """A 1-token sequence shifts the history by one: state_out =
    (h1, h2, x0)."""
    h = np.array([[[1.0], [2.0], [3.0]]])
    x = np.array([[7.0]])
    _, st = oracle.conv1d_silu_l2(x, np.ones((1, 4)), conv_state_in=h)
    np.testing.assert_array_equal(st.reshape(-1), [2.0, 3.0, 7.0])


def test_conv_varlen_sequences_do_not_mix():
    rng = np.random.default_rng(4)
    lens = [3, 1, 6]
    cu = np.concatenate([[0], np.cumsum(lens)])
    x = rng.standard_normal((cu[-1], 2))
    w = rng.standard_normal((2, 4))
    y, st = oracle.conv1d_silu_l2(x, w, cu_seqlens=cu)
    for n in range(3):
        yn, sn = oracle.conv1d_silu_l2(x[cu[n]:cu[n + 1]], w)
        np.testing.assert_array_equal(y[cu[n]:cu[n + 1]], yn)
        np.testing.assert_array_equal(st[n], sn[0])


def test_rmsnorm_hand_example(golden):
    f = golden("rmsnorm_hand.txt")
    x = np.array([f["x"]])
    z = np.array([[math.log(3.0), 0.0]])
    y = oracle.gated_rmsnorm(x, z, np.array(f["w"]), eps=0.0)
    assert abs(y[0, 0] - f["y0_over_sqrt2_ln3"][0] * math.sqrt(2) *
               math.log(3.0)) < 1e-15
    assert y[0, 1] == f["y1"][0]


def test_rmsnorm_unit_rms_and_scale_invariance():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((7, 128))
    z = rng.standard_normal((7, 128))
    w = rng.standard_normal(128)
    y = oracle.gated_rmsnorm(x, z, w, eps=0.0)
    core = y / (w * silu(z))
    np.testing.assert_allclose(np.sqrt(np.mean(core ** 2, axis=1)), 1.0,
                               rtol=1e-13)
    y3 = oracle.gated_rmsnorm(3.5 * x, z, w, eps=0.0)
    np.testing.assert_allclose(y3, y, rtol=1e-13, atol=1e-15)


def test_rmsnorm_eps_enters_under_the_root():
    x = np.full((1, 4), 1e-3)
    y = oracle.gated_rmsnorm(x, np.full((1, 4), 40.0), np.ones(4), eps=1e-6)
    # mean(x^2) = 1e-6, so the norm divides by sqrt(2e-6); SiLU(40) ~ 40
    np.testing.assert_allclose(y, 1e-3 / math.sqrt(2e-6) * silu(40.0),
                               rtol=1e-13)
