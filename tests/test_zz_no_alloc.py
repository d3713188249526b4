"""gdn_chunked_prefill_noalloc -- the prefill call that allocates nothing.

Some callers cannot give the library device memory at the call site (an
operator inside a host framework whose allocator it cannot reach, a serving
loop that must not allocate after start-up). For them the library offers a
variant of the chunked prefill that works in its own static device array. This
test calls it through the C ABI twice in a row on the same inputs and checks
each result against the regular entry point (which is given a workspace). The
two run the same kernel with the same launch shape, and its arithmetic does not
depend on which CTA takes which work item, so the results must be identical
bit for bit: a control word or ring slot left stale by the first call would show
up on the second. The Python wrapper is called once as well. The file is named
so that pytest collects it last; it also passes when run alone in a fresh
process. (The size refusal, GDN_ERR_UNSUPPORTED, cannot be reached on a 148-SM
B200: the array holds the rings of the most state CTAs the kernel uses there.)
"""
import ctypes

import numpy as np
import pytest
import torch

import gdn_inputs as gi
import gated_delta_rule_106_b200 as gdn

pytestmark = pytest.mark.gpu
DEV = "cuda"


def test_noalloc_matches_workspace_entry_point_twice():
    lib = gdn.load()
    lens = [130, 1, 64, 300]
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32, device=DEV)
    T, N = int(cu[-1]), len(lens)
    q = torch.from_numpy(gi.unit_heads(21, "zq", T, 16)).to(torch.bfloat16).to(DEV)
    k = torch.from_numpy(gi.unit_heads(21, "zk", T, 16)).to(torch.bfloat16).to(DEV)
    v = torch.from_numpy(gi.normal(21, "zv", (T, 48, 128))).to(torch.bfloat16).to(DEV)
    g, b = (x.to(DEV) for x in gi.gates(21, T, 48, tag="zg"))
    S0 = gi.initial_states(21, N).to(DEV)

    S_ref = torch.empty_like(S0)
    o_ref = gdn.gdn_chunked_prefill(q, k, v, g, b, cu, state_in=S0, state_out=S_ref,
                                    o_dtype=torch.float32)
    assert lib.gdn_chunked_prefill_noalloc_scratch_bytes() >= \
        gdn.gdn_chunked_prefill_workspace(N, T)

    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        o = torch.full((T, 48, 128), float("nan"), device=DEV)
        S = torch.full_like(S0, float("nan"))
        status = lib.gdn_chunked_prefill_noalloc(
            q.data_ptr(), k.data_ptr(), v.data_ptr(), gdn.GDN_BF16,
            q.stride(0), k.stride(0), v.stride(0), g.data_ptr(), b.data_ptr(),
            gdn.GDN_F32, S0.data_ptr(), S.data_ptr(), cu.data_ptr(), N, T, 16, 48,
            ctypes.c_float(1.0), o.data_ptr(), gdn.GDN_F32, stream)
        assert status == 0, gdn.gdn_status_string(status)
        torch.cuda.synchronize()
        assert torch.equal(o, o_ref), (call, float((o - o_ref).abs().max()))
        assert torch.equal(S, S_ref), (call, float((S - S_ref).abs().max()))
    S = torch.full_like(S0, float("nan"))
    o = gdn.gdn_chunked_prefill_noalloc(q, k, v, g, b, cu, state_in=S0, state_out=S,
                                        o_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.equal(o, o_ref) and torch.equal(S, S_ref)
