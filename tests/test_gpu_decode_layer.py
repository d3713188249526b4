"""GPU parity: gdn_decode_layer_step, the fused decode step of the layer.

One launch per token does the conv-cache roll with the kernel-4 conv, SiLU and
the q/k L2 norm, the stepwise recurrence on a pooled fp32 state, and the gated
RMS-norm. The oracle replays every sequence from its initial conv cache and
state in fp64 (conv -> recurrence -> gated RMS-norm) on the same bf16 inputs;
the fused kernel keeps q, k, v in fp32 between the stages, so nothing is
rounded in between on either side.

Bars (written here): the normed output is stored in bf16, so each element may
differ by half a bf16 ulp of its value (2^-9 relative, taken as 2^-8) plus
1e-3 of the output's rms for the fp32 arithmetic; final states within 1e-3
relative Frobenius per sequence (the bf16-input bar). Pool slots that no
sequence uses, and padding entries, must stay bit for bit as they were; the
rolled conv cache is byte work and must be exact.
"""
import numpy as np
import pytest
import torch

import gdn_inputs as gi
import oracle
import gated_delta_rule_106_b200 as gdn
from _parity import S_TOL, f64, state_err

pytestmark = pytest.mark.gpu
DEV = "cuda"


def pack_steps(per_step, N):
    """[steps][N, ...] -> [N*steps, ...] with sequence n's tokens contiguous."""
    a = np.stack([f64(x) for x in per_step], axis=1)
    return a.reshape(N * len(per_step), *a.shape[2:])


def oracle_layer(xs, gs, bs, zs, conv_w, norm_w, cache0, S0, steps):
    """fp64 chain over whole sequences: returns (out [N*steps, 48, 128], S, cache)."""
    ns = cache0.shape[0]
    cu = np.arange(ns + 1) * steps
    y, cache = oracle.conv1d_silu_l2(pack_steps(xs, ns), f64(conv_w), None, cu, f64(cache0),
                                     gi.L2_CHANNELS, 1e-6)
    T = y.shape[0]
    o, S = oracle.recurrence(y[:, :2048].reshape(T, 16, 128), y[:, 2048:4096].reshape(T, 16, 128),
                             y[:, 4096:].reshape(T, 48, 128), pack_steps(gs, ns),
                             pack_steps(bs, ns), f64(S0), cu)
    out = oracle.gated_rmsnorm(o, pack_steps(zs, ns), f64(norm_w), 1e-6)
    return out, S, cache


def test_fused_decode_256_sequences_128_steps_pooled():
    """The decode workload (256 sequences x 128 steps, bf16 per-step inputs,
    fp32 state ~N(0, 0.02), 3-row conv cache) on pools of 300 slots with a
    seeded permutation as state_idx; every sequence and head is checked."""
    N, steps, P, seed = 256, 128, 300, 0
    rng = np.random.default_rng(7)
    idx = rng.permutation(P)[:N].astype(np.int32)
    unused = np.setdiff1d(np.arange(P), idx)
    pool_S0 = gi.initial_states(seed, P, tag="pool")
    pool_c0 = gi.to_bf16(gi.normal(seed, "pconv", (P, 3, gi.CONV_CHANNELS)))
    conv_w = gi.conv_weight(seed)
    norm_w = torch.from_numpy(gi.normal(seed, "nw", (128,), std=0.5) + 1.0)
    state, cache = pool_S0.to(DEV), pool_c0.to(DEV)
    wd, nwd, idd = conv_w.to(DEV), norm_w.to(DEV), torch.from_numpy(idx).to(DEV)
    xs, gs, bs, zs, outs = [], [], [], [], []
    for s in range(steps):
        st = gi.decode_step_inputs(s, N, seed)
        out = gdn.gdn_decode_layer_step(st["x_pre"].to(DEV), wd, cache, st["g"].to(DEV),
                                        st["beta"].to(DEV), state, idd, st["z"].to(DEV), nwd,
                                        y_dtype=torch.bfloat16)
        xs.append(st["x_pre"]); gs.append(st["g"]); bs.append(st["beta"]); zs.append(st["z"])
        outs.append(out.cpu())
    torch.cuda.synchronize()
    state_h, cache_h = state.cpu(), cache.cpu()
    assert torch.equal(state_h[unused], pool_S0[unused])
    assert torch.equal(cache_h[unused], pool_c0[unused])
    worst_o, worst_s = 0.0, 0.0
    for g0 in range(0, N, 64):                       # bounded host memory
        sel = slice(g0, g0 + 64)
        ref, S_ref, c_ref = oracle_layer([x[sel] for x in xs], [x[sel] for x in gs],
                                         [x[sel] for x in bs], [x[sel] for x in zs], conv_w,
                                         norm_w, pool_c0[idx[sel]], pool_S0[idx[sel]], steps)
        got = pack_steps([o[sel] for o in outs], 64)
        rms = np.sqrt(np.mean(ref ** 2))
        bad = np.abs(got - ref) > 2.0 ** -8 * np.abs(ref) + 1e-3 * rms
        worst_o = max(worst_o, float(np.max(np.abs(got - ref)) / rms))
        assert not bad.any(), (g0, int(bad.sum()), worst_o)
        np.testing.assert_array_equal(f64(cache_h[idx[sel]]), c_ref)
        es = state_err(state_h[idx[sel]], S_ref)
        worst_s = max(worst_s, es)
        assert es <= S_TOL[torch.bfloat16], es
    print(f"fused decode: max|d out|/rms {worst_o:.3e}, state error {worst_s:.3e}")


def test_fused_decode_padding_and_fp32_paths():
    """Padding slots (negative or >= P) produce zero rows and touch nothing;
    fp32 inputs, fp32 gates and fp32 outputs take the same path; one step of
    8 sequences is checked against the oracle."""
    N, P, seed = 8, 12, 3
    idx = np.array([5, -1, 0, 11, 40, 7, 2, -7], dtype=np.int32)
    live = np.nonzero((idx >= 0) & (idx < P))[0]
    S0 = gi.initial_states(seed, P, tag="padS")
    c0 = torch.from_numpy(gi.normal(seed, "padc", (P, 3, gi.CONV_CHANNELS)))
    conv_w = gi.conv_weight(seed)
    norm_w = torch.ones(128)
    x = torch.from_numpy(gi.normal(seed, "padx", (N, gi.CONV_CHANNELS)))
    g, b = gi.gates(seed, N, dtype=torch.float32, tag="padg")
    z = torch.from_numpy(gi.normal(seed, "padz", (N, 48, 128)))
    state, cache = S0.to(DEV), c0.to(DEV)
    out = gdn.gdn_decode_layer_step(x.to(DEV), conv_w.to(DEV), cache, g.to(DEV), b.to(DEV),
                                    state, torch.from_numpy(idx).to(DEV), z.to(DEV),
                                    norm_w.to(DEV), y_dtype=torch.float32, scale=0.5)
    torch.cuda.synchronize()
    out = out.cpu()
    dead = np.setdiff1d(np.arange(N), live)
    assert torch.all(out[dead] == 0)
    untouched = np.setdiff1d(np.arange(P), idx[live])
    assert torch.equal(state.cpu()[untouched], S0[untouched])
    assert torch.equal(cache.cpu()[untouched], c0[untouched])
    ns = len(live)
    cu = np.arange(ns + 1)
    y, c_ref = oracle.conv1d_silu_l2(f64(x[live]), f64(conv_w), None, cu, f64(c0[idx[live]]),
                                     gi.L2_CHANNELS, 1e-6)
    o, S_ref = oracle.recurrence(y[:, :2048].reshape(ns, 16, 128), y[:, 2048:4096].reshape(ns, 16, 128),
                                 y[:, 4096:].reshape(ns, 48, 128), f64(g[live]), f64(b[live]),
                                 f64(S0[idx[live]]), cu, scale=0.5)
    ref = oracle.gated_rmsnorm(o, f64(z[live]), f64(norm_w), 1e-6)
    rms = np.sqrt(np.mean(ref ** 2))
    assert np.max(np.abs(f64(out[live]) - ref)) <= 1e-4 * rms + 1e-5 * np.abs(ref).max()
    assert state_err(state.cpu()[idx[live]], S_ref) <= 1e-5
    np.testing.assert_array_equal(f64(cache.cpu()[idx[live]]), c_ref)
