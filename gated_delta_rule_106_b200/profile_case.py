"""Small, fixed launches of one library kernel, for profiler captures.

    python -m gated_delta_rule_106_b200.profile_case decode  [--n 64]   [--launches 4]
    python -m gated_delta_rule_106_b200.profile_case prefill [--t 8192] [--launches 4]
    python -m gated_delta_rule_106_b200.profile_case conv    [--t 8192] [--launches 4]
    python -m gated_delta_rule_106_b200.profile_case norm    [--t 8192] [--launches 4]
    python -m gated_delta_rule_106_b200.profile_case dconv   [--n 64]   [--launches 4]

Each case allocates its inputs (synthetic, seeded; larger than the 126 MB L2
at the defaults so DRAM counters are meaningful, and a few GB at most), runs
the kernel `--launches` times on the current stream and exits. It prints the
mean CUDA-event time per launch, for reference only.
"""
from __future__ import annotations

import argparse
import os
import sys

import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import gdn_inputs as gi  # noqa: E402
import gated_delta_rule_106_b200 as gdn  # noqa: E402

DEV = "cuda"


def case_decode(a):
    N = a.n
    st = gi.decode_step_inputs(0, N, seed=0)
    state = gi.initial_states(0, N, tag="pstate").to(DEV)
    q = gi.to_bf16(gi.unit_heads(0, "pq", N, 16)).to(DEV)
    k = gi.to_bf16(gi.unit_heads(0, "pk", N, 16)).to(DEV)
    v = gi.to_bf16(gi.normal(0, "pv", (N, 48, 128))).to(DEV)
    g, b = st["g"].to(DEV), st["beta"].to(DEV)
    o = torch.empty((N, 48, 128), dtype=torch.bfloat16, device=DEV)
    return lambda: gdn.gdn_decode_step(q, k, v, g, b, state, o=o, scale=0.05)


def case_prefill(a):
    p = gi.prefill_inputs(T=a.t, seed=0)
    y = gdn.gdn_conv1d_silu(p["x_pre"].to(DEV), p["conv_w"].to(DEV),
                            p["cu_seqlens"].to(DEV))
    q = y[:, :2048].view(a.t, 16, 128)
    k = y[:, 2048:4096].view(a.t, 16, 128)
    v = y[:, 4096:].view(a.t, 48, 128)
    g, b, cu = p["g"].to(DEV), p["beta"].to(DEV), p["cu_seqlens"].to(DEV)
    o = torch.empty((a.t, 48, 128), dtype=torch.bfloat16, device=DEV)
    S = torch.empty((1, 48, 128, 128), device=DEV)
    return lambda: gdn.gdn_chunked_prefill(q, k, v, g, b, cu, state_out=S, o=o)


def case_conv(a):
    p = gi.prefill_inputs(T=a.t, seed=0)
    x, w, cu = p["x_pre"].to(DEV), p["conv_w"].to(DEV), p["cu_seqlens"].to(DEV)
    y = torch.empty_like(x)
    return lambda: gdn.gdn_conv1d_silu(x, w, cu, y=y)


def case_norm(a):
    x = gi.gate_z(1, a.t, tag="px").to(DEV)
    z = gi.gate_z(0, a.t).to(DEV)
    w = torch.ones(128, device=DEV)
    y = torch.empty_like(x)
    return lambda: gdn.gdn_gated_rmsnorm(x, z, w, eps=1e-6, y=y)


def case_dconv(a):
    """The decode step's conv: --n one-token sequences, 3-row cache rolled in place."""
    N = a.n
    cache = gi.to_bf16(gi.normal(0, "dconv", (N, 3, gi.CONV_CHANNELS))).to(DEV)
    x = gi.decode_step_inputs(0, N, 0)["x_pre"].to(DEV)
    w = gi.conv_weight(0).to(DEV)
    cu = torch.arange(N + 1, dtype=torch.int32, device=DEV)
    y = torch.empty((N, gi.CONV_CHANNELS), dtype=torch.bfloat16, device=DEV)
    return lambda: gdn.gdn_conv1d_silu(x, w, cu, conv_state_in=cache, conv_state_out=cache, y=y)


CASES = {"decode": case_decode, "prefill": case_prefill, "conv": case_conv,
         "norm": case_norm, "dconv": case_dconv}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("case", choices=sorted(CASES))
    ap.add_argument("--n", type=int, default=64)
    ap.add_argument("--t", type=int, default=8192)
    ap.add_argument("--launches", type=int, default=4)
    a = ap.parse_args()
    gdn.load()
    run = CASES[a.case](a)
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(a.launches):
        run()
    e.record()
    torch.cuda.synchronize()
    print(f"{a.case}: {s.elapsed_time(e) / a.launches:.4f} ms per launch")


if __name__ == "__main__":
    main()
