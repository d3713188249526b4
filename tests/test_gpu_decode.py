"""GPU parity: gdn_decode_step (stepwise decode) against the fp64 oracle.

A run of decode steps on N sequences equals the oracle's recurrence over N
packed sequences of `steps` tokens each. Bars: the gated delta rule
tolerances (output max/rms 1e-2 and state 1e-3 for bf16 inputs, 1e-4 for
fp32), plus a tighter 1e-4 / 1e-5 check because the kernel's arithmetic is
fp32 on exactly the values it consumed.
"""
import numpy as np
import pytest
import torch

import gdn_inputs as gi
import oracle
import gated_delta_rule_106_b200 as gdn
from _parity import O_TOL, S_TOL, bf16_out_bound, f64, o_err, state_err

pytestmark = pytest.mark.gpu
DEV = "cuda"


def step_inputs(seed, s, N, qkv_dtype, gate_dtype, H_k=16, H_v=48):
    q = torch.from_numpy(gi.unit_heads(seed, f"q{s}", N, H_k)).to(qkv_dtype)
    k = torch.from_numpy(gi.unit_heads(seed, f"k{s}", N, H_k)).to(qkv_dtype)
    v = torch.from_numpy(gi.normal(seed, f"v{s}", (N, H_v, 128))).to(qkv_dtype)
    g, b = gi.gates(seed, N, H_v, dtype=gate_dtype, tag=f"g{s}")
    return q, k, v, g, b


def pack_steps(per_step, N):
    """[steps][N, ...] -> [N*steps, ...] with sequence n's tokens contiguous."""
    a = np.stack([f64(x) for x in per_step], axis=1)      # [N, steps, ...]
    return a.reshape(N * len(per_step), *a.shape[2:])


@pytest.mark.parametrize("qkv_dtype,gate_dtype,o_dtype", [
    (torch.bfloat16, torch.bfloat16, torch.float32),
    (torch.bfloat16, torch.float32, torch.bfloat16),
    (torch.float32, torch.float32, torch.float32),
])
def test_decode_steps_match_oracle(qkv_dtype, gate_dtype, o_dtype):
    N, steps, seed = 7, 4, 3
    S0 = gi.initial_states(seed, N)
    Sd = S0.to(DEV)
    ins, outs = [], []
    for s in range(steps):
        q, k, v, g, b = step_inputs(seed, s, N, qkv_dtype, gate_dtype)
        o = gdn.gdn_decode_step(q.to(DEV), k.to(DEV), v.to(DEV), g.to(DEV),
                                b.to(DEV), Sd, o_dtype=o_dtype, scale=0.5)
        ins.append((q, k, v, g, b))
        outs.append(o.cpu())
    torch.cuda.synchronize()
    packed = [pack_steps([x[i] for x in ins], N) for i in range(5)]
    cu = np.arange(N + 1) * steps
    o_ref, S_ref = oracle.recurrence(*packed, state_in=f64(S0), cu_seqlens=cu,
                                     scale=0.5)
    o_got = pack_steps(outs, N)
    eo, es = o_err(o_got, o_ref), state_err(Sd, S_ref)
    bound = O_TOL[qkv_dtype] + (bf16_out_bound(o_ref) if o_dtype == torch.bfloat16 else 0)
    assert eo <= bound and es <= S_TOL[qkv_dtype], (eo, es)
    if o_dtype == torch.float32:
        assert eo <= 1e-4, eo
    assert es <= 1e-5, es


def test_decode_reads_strided_conv_output():
    """q/k/v as column views of one packed [N, 10240] buffer."""
    N, seed = 9, 4
    buf = torch.from_numpy(gi.normal(seed, "buf", (N, 10240), std=0.1)).to(torch.bfloat16)
    q = buf[:, :2048].view(N, 16, 128)
    k = buf[:, 2048:4096].view(N, 16, 128)
    v = buf[:, 4096:].view(N, 48, 128)
    g, b = gi.gates(seed, N, dtype=torch.bfloat16)
    S0 = gi.initial_states(seed, N)
    Sd = S0.to(DEV)
    bd = buf.to(DEV)
    o = gdn.gdn_decode_step(bd[:, :2048].view(N, 16, 128),
                            bd[:, 2048:4096].view(N, 16, 128),
                            bd[:, 4096:].view(N, 48, 128), g.to(DEV), b.to(DEV),
                            Sd, o_dtype=torch.float32)
    torch.cuda.synchronize()
    o_ref, S_ref = oracle.recurrence(f64(q), f64(k), f64(v), f64(g), f64(b),
                                     f64(S0), np.arange(N + 1))
    assert o_err(o, o_ref) <= 1e-4 and state_err(Sd, S_ref) <= 1e-5


def test_decode_layer_256_sequences_128_steps():
    """Decode workload: 256 sequences x 128 steps, fp32 state [256,48,128,128]
    ~ N(0, 0.02), conv cache of 3 prior tokens, bf16 per-step inputs. Each
    step: conv (in-place cache roll) -> decode step -> gated RMS-norm. The
    oracle replays sampled sequences on the exact values each kernel read."""
    N, steps, seed = 256, 128, 0
    init = gi.decode_initial(N, seed)
    conv_w = gi.conv_weight(seed)
    norm_w = torch.ones(128)
    sample = [0, 17, 128, 255]
    state = init["state"].to(DEV)
    cache = init["conv_state"].to(DEV)
    wd, nwd = conv_w.to(DEV), norm_w.to(DEV)
    cu = torch.arange(N + 1, dtype=torch.int32, device=DEV)
    xs, ys, gs, bs, zs, os_, yn = [], [], [], [], [], [], []
    for s in range(steps):
        st = gi.decode_step_inputs(s, N, seed)
        y = gdn.gdn_conv1d_silu(st["x_pre"].to(DEV), wd, cu, conv_state_in=cache,
                                conv_state_out=cache)
        g, b = st["g"].to(DEV), st["beta"].to(DEV)
        o = gdn.gdn_decode_step(y[:, :2048].view(N, 16, 128),
                                y[:, 2048:4096].view(N, 16, 128),
                                y[:, 4096:].view(N, 48, 128), g, b, state,
                                o_dtype=torch.float32)
        out = gdn.gdn_gated_rmsnorm(o, st["z"].to(DEV), nwd, eps=1e-6,
                                    y_dtype=torch.bfloat16)
        xs.append(st["x_pre"][sample])
        ys.append(y[sample].cpu())
        gs.append(st["g"][sample]); bs.append(st["beta"][sample])
        zs.append(st["z"][sample]); os_.append(o[sample].cpu()); yn.append(out[sample].cpu())
    torch.cuda.synchronize()
    ns = len(sample)
    cu_s = np.arange(ns + 1) * steps
    # conv: replay each sampled sequence's 128 tokens from its initial cache
    x_p = pack_steps(xs, ns)
    y_ref, cache_ref = oracle.conv1d_silu_l2(x_p, f64(conv_w), None, cu_s,
                                             f64(init["conv_state"][sample]),
                                             gi.L2_CHANNELS, 1e-6)
    y_p = pack_steps(ys, ns)
    assert np.all(np.abs(y_p - y_ref) <= 2.0 ** -8 * np.abs(y_ref) + 1e-6)
    np.testing.assert_array_equal(f64(cache[sample]), cache_ref)
    # recurrence on the consumed q/k/v
    q = y_p[:, :2048].reshape(-1, 16, 128)
    k = y_p[:, 2048:4096].reshape(-1, 16, 128)
    v = y_p[:, 4096:].reshape(-1, 48, 128)
    o_ref, S_ref = oracle.recurrence(q, k, v, pack_steps(gs, ns), pack_steps(bs, ns),
                                     f64(init["state"][sample]), cu_s)
    eo, es = o_err(pack_steps(os_, ns), o_ref), state_err(state[sample], S_ref)
    assert eo <= O_TOL[torch.bfloat16] and es <= S_TOL[torch.bfloat16], (eo, es)
    assert eo <= 1e-4 and es <= 1e-5, (eo, es)
    # gated RMS-norm on the consumed o
    yn_ref = oracle.gated_rmsnorm(pack_steps(os_, ns), pack_steps(zs, ns),
                                  f64(norm_w), 1e-6)
    yn_p = pack_steps(yn, ns)
    assert np.all(np.abs(yn_p - yn_ref) <= 2.0 ** -8 * np.abs(yn_ref) + 1e-6)
