"""GPU: the whole layer chain against the fp64 oracle chain from the pre-conv input.

Every other GPU test feeds the oracle the exact values the kernel under test
read (the previous GPU stage's bf16 output), so that it measures that kernel.
This test measures the chain as a user runs it: conv k=4 + SiLU + L2 ->
chunked prefill -> gated RMS-norm on the prefill workload (T=8192, bf16
activations, fp32 gates, bf16 outputs, as the benchmark runs it), against the
oracle's conv -> recurrence -> gated RMS-norm computed in fp64 from the same
x_pre, with no GPU intermediate.

What the bound is. The chain stores the conv output y, the layer output o
and the normed output in bf16. A max-over-rms bar cannot hold for any chain
that does so on this data: o peaks at ~37x its rms, and rounding y alone moves
o by ~0.13 of rms at those peaks. So the test measures both chains with the
relative Frobenius error, and bounds the GPU's by the triangle inequality:
    ||gpu - fp64|| <= ||R - fp64|| + ||gpu - R||,
where R is the oracle chain that rounds y, o and the normed output to bf16 at
the same points (what bf16 storage alone costs, computed here), and
||gpu - R|| / ||ref|| is at most the prefill kernel's own bar (1e-2 of rms on
its output, which bounds its relative Frobenius error) carried through the
norm. The measured values are recorded in the report (properties) and printed.
"""
import numpy as np
import pytest
import torch

import gdn_inputs as gi
import oracle
import gated_delta_rule_106_b200 as gdn
from _parity import O_TOL, f64

pytestmark = pytest.mark.gpu
DEV = "cuda"


def bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(torch.bfloat16).double().numpy()


def rel_frob(a, ref):
    return float(np.linalg.norm(a - ref) / np.linalg.norm(ref))


def max_rms(a, ref):
    return float(np.max(np.abs(a - ref)) / np.sqrt(np.mean(ref ** 2)))


def oracle_chain(y, p, cu, T, round_bf16):
    r = bf16 if round_bf16 else (lambda a: a)
    y = r(y)
    o, _ = oracle.recurrence(y[:, :2048].reshape(T, 16, 128), y[:, 2048:4096].reshape(T, 16, 128),
                             y[:, 4096:].reshape(T, 48, 128), f64(p["g"]), f64(p["beta"]), None,
                             cu.numpy())
    o = r(o)
    return o, r(oracle.gated_rmsnorm(o, f64(p["z"]), f64(p["norm_w"]), 1e-6))


def test_prefill_chain_from_pre_conv_input(record_property):
    T = 8192
    p = gi.prefill_inputs(T=T, seed=0)
    cu = p["cu_seqlens"]
    x = p["x_pre"].to(DEV)
    y = gdn.gdn_conv1d_silu(x, p["conv_w"].to(DEV), cu.to(DEV))
    o = gdn.gdn_chunked_prefill(y[:, :2048].view(T, 16, 128), y[:, 2048:4096].view(T, 16, 128),
                                y[:, 4096:].view(T, 48, 128), p["g"].to(DEV), p["beta"].to(DEV),
                                cu.to(DEV), o_dtype=torch.bfloat16)
    out = gdn.gdn_gated_rmsnorm(o, p["z"].to(DEV), p["norm_w"].to(DEV), eps=1e-6)
    torch.cuda.synchronize()
    o_gpu, out_gpu = f64(o), f64(out)
    del o, out, y

    y_ref, _ = oracle.conv1d_silu_l2(f64(p["x_pre"]), f64(p["conv_w"]), None, cu.numpy(),
                                     None, gi.L2_CHANNELS, 1e-6)
    o_ref, out_ref = oracle_chain(y_ref, p, cu, T, False)
    o_r, out_r = oracle_chain(y_ref, p, cu, T, True)

    m = {"o_rel_frob": rel_frob(o_gpu, o_ref), "out_rel_frob": rel_frob(out_gpu, out_ref),
         "o_max_over_rms": max_rms(o_gpu, o_ref), "out_max_over_rms": max_rms(out_gpu, out_ref),
         "storage_only_o_rel_frob": rel_frob(o_r, o_ref),
         "storage_only_out_rel_frob": rel_frob(out_r, out_ref),
         "storage_only_o_max_over_rms": max_rms(o_r, o_ref)}
    for k, v in m.items():
        record_property(f"chain_{k}", v)
    print("chain errors vs the fp64 oracle chain: " +
          ", ".join(f"{k} {v:.3e}" for k, v in m.items()))
    bar = O_TOL[torch.bfloat16]
    assert m["o_rel_frob"] <= m["storage_only_o_rel_frob"] + bar, m
    assert m["out_rel_frob"] <= m["storage_only_out_rel_frob"] + bar, m
