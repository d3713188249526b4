"""GPU: a bounded wait inside the chunked prefill kernel that runs out is
reported to the caller, leaves NaN where the work was not finished, and leaves
the context usable.

The tensor-core prefill hands each chunk from a preparing CTA to the CTA that
carries the state through a flag in the workspace; every wait on such a flag is
bounded. The test lowers that bound to 1 us, so the state CTAs' first wait
(the first chunk is published ~20 us after launch) runs out: no fault, no
hang, just the designed give-up path. It checks that gdn_chunked_prefill_status
reports GDN_ERR_TIMEOUT, that every output is either NaN (unfinished) or equal
bit for bit to a normal call's, and that a normal call afterwards on the same
workspace reports GDN_OK and reproduces the normal result.
"""
import pytest
import torch

import gdn_inputs as gi
import gated_delta_rule_106_b200 as gdn

pytestmark = pytest.mark.gpu
DEV = "cuda"


def test_wait_that_runs_out_is_reported_and_marked():
    T = 8192
    q = gi.to_bf16(gi.unit_heads(31, "tq", T, 16)).to(DEV)
    k = gi.to_bf16(gi.unit_heads(31, "tk", T, 16)).to(DEV)
    v = gi.to_bf16(gi.normal(31, "tv", (T, 48, 128))).to(DEV)
    g, b = (x.to(DEV) for x in gi.gates(31, T, 48, tag="tg"))
    cu = torch.tensor([0, T], dtype=torch.int32, device=DEV)
    ws = torch.empty(gdn.gdn_chunked_prefill_workspace(1, T), dtype=torch.uint8, device=DEV)

    def run():
        S = torch.full((1, 48, 128, 128), -1.0, device=DEV)
        o = torch.full((T, 48, 128), -1.0, device=DEV)
        gdn.gdn_chunked_prefill(q, k, v, g, b, cu, state_out=S, o=o, workspace=ws)
        return o, S, gdn.gdn_chunked_prefill_status(ws)

    o_ref, S_ref, st = run()
    assert st == 0
    try:
        gdn.gdn_set_wait_limit_ns(1000)
        o, S, st = run()
    finally:
        gdn.gdn_set_wait_limit_ns(0)
    assert st == gdn.GDN_ERR_TIMEOUT, gdn.gdn_status_string(st)
    nan = torch.isnan(o)
    assert nan.any()
    assert torch.equal(o[~nan], o_ref[~nan])          # nothing else is left stale
    head_nan = torch.isnan(S).flatten(2).all(-1)      # a head's state: all NaN or exact
    assert torch.equal(S[~head_nan], S_ref[~head_nan])
    assert torch.equal(torch.isnan(S).flatten(2).any(-1), head_nan)

    o2, S2, st = run()
    assert st == 0
    assert torch.equal(o2, o_ref) and torch.equal(S2, S_ref)
