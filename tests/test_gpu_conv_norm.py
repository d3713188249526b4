"""GPU parity: gdn_conv1d_silu and gdn_gated_rmsnorm against the fp64 oracle.

Element-wise bars: fp32 outputs within 2e-6 relative + 1e-6 absolute (fp32
arithmetic with hardware exp); bf16 outputs within 2^-8 relative (half a bf16
ulp at worst) + 1e-6. Conv states are byte copies and must match exactly.
"""
import numpy as np
import pytest
import torch

import gdn_inputs as gi
import oracle
import gated_delta_rule_106_b200 as gdn
from _parity import close_elementwise, f64

pytestmark = pytest.mark.gpu
DEV = "cuda"
TOL = {torch.float32: (2e-6, 1e-6), torch.bfloat16: (2.0 ** -8, 1e-6)}


def conv_case(lens, x_dtype=torch.bfloat16, y_dtype=torch.bfloat16, hist=True,
              bias=False, C=gi.CONV_CHANNELS, l2c=gi.L2_CHANNELS, seed=0,
              in_place=False, x_pad=0):
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32)
    T, N = int(cu[-1]), len(lens)
    x = torch.from_numpy(gi.normal(seed, "cx", (T, C))).to(x_dtype)
    w = torch.from_numpy(gi.normal(seed, "cw", (C, 4), std=0.5))
    b = torch.from_numpy(gi.normal(seed, "cb", (C,), std=0.1)) if bias else None
    h = torch.from_numpy(gi.normal(seed, "ch", (N, 3, C))).to(x_dtype) if hist else None

    xd = torch.zeros((T, C + x_pad), dtype=x_dtype, device=DEV)
    xd[:, :C] = x.to(DEV)
    xv = xd[:, :C]                      # strided view when x_pad > 0
    hd = h.to(DEV) if hist else None
    cso = hd if (in_place and hist) else torch.full((N, 3, C), 7, dtype=x_dtype, device=DEV)
    y = gdn.gdn_conv1d_silu(xv, w.to(DEV), cu.to(DEV),
                            bias=None if b is None else b.to(DEV),
                            conv_state_in=hd, conv_state_out=cso,
                            l2norm_channels=l2c, y_dtype=y_dtype)
    torch.cuda.synchronize()
    y_ref, st_ref = oracle.conv1d_silu_l2(f64(x), f64(w), None if b is None else f64(b),
                                          cu.numpy(), None if h is None else f64(h),
                                          l2_channels=l2c, l2_eps=1e-6)
    rtol, atol = TOL[y_dtype]
    nbad, worst = close_elementwise(y, y_ref, rtol, atol)
    assert nbad == 0, f"{nbad} conv outputs off, worst |d|={worst}"
    np.testing.assert_array_equal(f64(cso), st_ref)


def test_conv_prefill_one_sequence_with_tail():
    conv_case([200])


def test_conv_varlen_ragged_with_history():
    conv_case([1, 2, 3, 63, 64, 65, 130], hist=True, bias=True)


def test_conv_varlen_no_history_fp32():
    conv_case([5, 0, 17, 1, 40], x_dtype=torch.float32, y_dtype=torch.float32,
              hist=False)


def test_conv_bf16_in_fp32_out_strided_input():
    conv_case([33, 70], y_dtype=torch.float32, x_pad=64)


def test_conv_decode_in_place_roll():
    """Decode: one token per sequence, history rolled in place."""
    conv_case([1] * 64, in_place=True)


def test_conv_short_sequences_cache_out():
    """Sequences of 0-3 tokens take the decode-shaped tiling: the conv kernel
    writes the caches of sequences held whole by one 2-token batch, the roll
    kernel the others (here some 2-token sequences straddle two batches)."""
    conv_case([1, 2, 1, 0, 2, 3, 1, 1, 2, 1], hist=True)


def test_conv_short_sequences_in_place():
    conv_case([1, 2, 1, 2, 2, 1, 1, 3, 0, 1], in_place=True)


def test_conv_short_sequences_fp32_no_history():
    conv_case([2, 1, 1, 3, 0, 1, 2], x_dtype=torch.float32, y_dtype=torch.float32,
              hist=False)


def test_conv_zero_tokens_only_copies_state():
    C = 256
    h = torch.randn(3, 3, C, dtype=torch.bfloat16, device=DEV)
    out = torch.zeros_like(h)
    cu = torch.zeros(4, dtype=torch.int32, device=DEV)
    x = torch.empty((0, C), dtype=torch.bfloat16, device=DEV)
    gdn.gdn_conv1d_silu(x, torch.ones(C, 4, device=DEV), cu, conv_state_in=h,
                        conv_state_out=out, l2norm_channels=0)
    torch.cuda.synchronize()
    assert torch.equal(out, h)


def test_conv_prefill_8192_full_width():
    """Prefill layer size: T=8192, 10240 channels (q|k|v), L2 on q|k."""
    p = gi.prefill_inputs(T=8192, seed=0)
    cu = p["cu_seqlens"]
    y = gdn.gdn_conv1d_silu(p["x_pre"].to(DEV), p["conv_w"].to(DEV), cu.to(DEV))
    torch.cuda.synchronize()
    y_ref, _ = oracle.conv1d_silu_l2(f64(p["x_pre"]), f64(p["conv_w"]), None,
                                     cu.numpy(), None, gi.L2_CHANNELS, 1e-6)
    nbad, worst = close_elementwise(y, y_ref, *TOL[torch.bfloat16])
    assert nbad == 0, (nbad, worst)


@pytest.mark.parametrize("x_dtype,z_dtype,w_dtype,y_dtype", [
    (torch.float32, torch.bfloat16, torch.float32, torch.float32),
    (torch.bfloat16, torch.bfloat16, torch.float32, torch.bfloat16),
    (torch.float32, torch.float32, torch.bfloat16, torch.bfloat16),
])
def test_gated_rmsnorm(x_dtype, z_dtype, w_dtype, y_dtype):
    rows = 300 * 48 + 5        # not a multiple of the rows per CTA
    x = torch.from_numpy(gi.normal(1, "nx", (rows, 128), std=0.3)).to(x_dtype)
    z = torch.from_numpy(gi.normal(1, "nz", (rows, 128))).to(z_dtype)
    w = torch.from_numpy(gi.normal(1, "nw", (128,))).to(w_dtype)
    y = gdn.gdn_gated_rmsnorm(x.to(DEV), z.to(DEV), w.to(DEV), eps=1e-6,
                              y_dtype=y_dtype)
    torch.cuda.synchronize()
    y_ref = oracle.gated_rmsnorm(f64(x), f64(z), f64(w), eps=1e-6)
    nbad, worst = close_elementwise(y, y_ref, *TOL[y_dtype])
    assert nbad == 0, (nbad, worst)


def test_gated_rmsnorm_in_place_prefill_size():
    T = 8192
    x = torch.from_numpy(gi.normal(2, "nx", (T, 48, 128), std=0.05)).to(torch.bfloat16)
    z = gi.gate_z(2, T)
    w = torch.ones(128)
    xd = x.to(DEV)
    gdn.gdn_gated_rmsnorm(xd, z.to(DEV), w.to(DEV), eps=1e-6, y=xd)
    torch.cuda.synchronize()
    y_ref = oracle.gated_rmsnorm(f64(x), f64(z), f64(w), eps=1e-6)
    nbad, worst = close_elementwise(xd, y_ref, *TOL[torch.bfloat16])
    assert nbad == 0, (nbad, worst)
