"""GPU parity: the global-attention layer (gdn_attention_prefill,
gdn_attention_decode) against the fp64 oracle.

Inputs are the layer's shapes (24 query / 4 key-value heads, head dim 256,
rotary on 64 dims, base 1e7) drawn by ``gdn_inputs.attention_inputs``; the
oracle gets the same bf16 values as fp64. The bar is the layer's 1e-2 of rms
for bf16 inputs, read per output row (token, head) -- an attention output is a
convex combination of value rows, and its size falls like 1/sqrt(keys) along
a sequence, so each row is measured against its own rms -- on top of what
bf16 storage of the output costs by itself:

    |o - o_ref| <= 2^-8 |o_ref| + 1e-2 * rms(o_ref row)

(2^-8 |x| bounds half a bf16 ulp of x). The largest max |o - o_ref| / rms
over rows is recorded next to the same figure for the oracle's output rounded
to bf16. The cache rows (fp16) are within fp16 rounding of the oracle's keys
and equal to the values exactly wherever a value is in fp16's normal range
(within 2^-25 below it).

* ragged packed prompts spanning several 64-token tiles, an empty sequence,
  one-token sequences and ragged tails, every output element;
* explicit three-axis positions, and a prompt continuing a cached prefix
  (pos0);
* T = 8192 (the bench's prefill launch): 72 sampled query tokens, among them
  the first, the last and tile edges, all 24 heads;
* decode: pooled slots in permuted order, cache lengths around the 512-token
  split edges, three steps advancing cache_len, against the oracle run on the
  whole sequences; an out-of-range slot is skipped and reported.
"""
import numpy as np
import pytest
import torch

import gdn_inputs as gi
import oracle
import gated_delta_rule_106_b200 as gdn

pytestmark = pytest.mark.gpu
DEV = "cuda"
TOL = 1e-2


def f64(t):
    return gi.as_f64(t)


def bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(torch.bfloat16).double().numpy()


def check(got, ref, rows=None, tol=TOL):
    """Every (token, head) row: each element within 2^-8 |ref| + tol * rms(row).
    Returns (max over rows of max |got - ref| / rms, the same for bf16(ref))."""
    if rows is not None:
        got, ref = got[rows], ref[rows]
    rms = np.sqrt(np.mean(ref ** 2, axis=-1, keepdims=True))
    d = np.abs(got - ref)
    bad = d > 2.0 ** -8 * np.abs(ref) + tol * rms
    assert not bad.any(), (np.argwhere(bad)[:5].tolist(), float((d / rms)[bad].max()))
    return float((d / rms).max()), float((np.abs(bf16(ref) - ref) / rms).max())


def check_cache_rows(k_rot, v_h, kref, v):
    kr = f64(k_rot)
    assert np.all(np.abs(kr - kref) <= 2.0 ** -10 * np.abs(kref) + 1e-3)
    vh, v = f64(v_h), f64(v)
    normal = np.abs(v) >= 2.0 ** -14          # fp16's normal range: exact there
    np.testing.assert_array_equal(vh[normal], v[normal])
    assert np.all(np.abs(vh - v) <= 2.0 ** -25)   # half the fp16 subnormal spacing


def run_prefill(p, cu, **kw):
    d = {k: v.to(DEV) for k, v in p.items()}
    out = gdn.gdn_attention_prefill(d["q"], d["k"], d["v"], d["gate"], d["q_norm_w"],
                                    d["k_norm_w"], cu.to(DEV), **kw)
    torch.cuda.synchronize()
    return out


def run_oracle(p, cu, **kw):
    return oracle.attention(f64(p["q"]), f64(p["k"]), f64(p["v"]), f64(p["gate"]),
                            f64(p["q_norm_w"]), f64(p["k_norm_w"]), cu_seqlens=cu, **kw)


def test_prefill_ragged_packed(record_property):
    lens = [1, 63, 64, 0, 65, 130, 200, 2]
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32)
    T = int(cu[-1])
    p = gi.attention_inputs(T, seed=1)
    o, k_rot, v_h = run_prefill(p, cu)
    ref, _, kref = run_oracle(p, cu.numpy())
    e, e_store = check(f64(o), ref)
    record_property("attn_prefill_ragged_max_over_rms", e)
    record_property("attn_prefill_ragged_storage_only", e_store)
    check_cache_rows(k_rot, v_h, kref, p["v"])


def test_prefill_positions_and_prefix_offset():
    lens = [150, 77]
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32)
    T = int(cu[-1])
    p = gi.attention_inputs(T, seed=2)
    pos3 = torch.from_numpy(
        gi.rng(2, "pos3").integers(0, 4000, size=(3, T)).astype(np.int32))
    o, _, _ = run_prefill(p, cu, positions=pos3.to(DEV))
    ref, _, _ = run_oracle(p, cu.numpy(), positions=pos3.numpy())
    check(f64(o), ref)
    pos0 = torch.tensor([3000, 17], dtype=torch.int32)
    o, k_rot, v_h = run_prefill(p, cu, pos0=pos0.to(DEV))
    ref, _, kref = run_oracle(p, cu.numpy(), pos0=pos0.numpy())
    check(f64(o), ref)
    check_cache_rows(k_rot, v_h, kref, p["v"])


def test_prefill_t8192_sampled_rows(record_property):
    T = 8192
    cu = torch.tensor([0, T], dtype=torch.int32)
    p = gi.attention_inputs(T, seed=0)
    o, _, _ = run_prefill(p, cu)
    rng = gi.rng(0, "attn_rows")
    rows = sorted(set([0, 1, 63, 64, 127, 128, 4095, 4096, T - 65, T - 64, T - 2, T - 1]) |
                  set(rng.integers(0, T, size=60).tolist()))
    ref, _, _ = run_oracle(p, cu.numpy(), rows=rows)
    e, e_store = check(f64(o), ref, rows=rows)
    record_property("attn_prefill_t8192_max_over_rms", e)
    record_property("attn_prefill_t8192_storage_only", e_store)


def test_prefill_repeatable_bits():
    """Same inputs, same launch: identical bits (no order-dependent reduction)."""
    T = 1000
    cu = torch.tensor([0, 300, T], dtype=torch.int32)
    p = gi.attention_inputs(T, seed=3)
    a = run_prefill(p, cu)
    b = run_prefill(p, cu)
    assert all(torch.equal(x, y) for x, y in zip(a, b))


def decode_case(lens, seed, steps, L_max=2048):
    """Sequences with the given cached lengths in permuted pool slots: the
    prompt goes through gdn_attention_prefill into the caches, then `steps`
    decode steps; returns GPU outputs per step and the oracle's."""
    N = len(lens)
    P = N + 3
    tot = [l + steps for l in lens]
    cu_full = np.concatenate([[0], np.cumsum(tot)])
    p = gi.attention_inputs(int(cu_full[-1]), seed=seed)
    slots = gi.rng(seed, "slots").permutation(P)[:N].astype(np.int32)
    kc = torch.zeros(P, L_max, 4, 256, dtype=torch.float16, device=DEV)
    vc = torch.zeros_like(kc)
    for n, l in enumerate(lens):
        if l == 0:
            continue
        a = int(cu_full[n])
        sl = {k: (v[a:a + l] if v.dim() == 3 else v) for k, v in p.items()}
        _, k_rot, v_h = run_prefill(sl, torch.tensor([0, l], dtype=torch.int32))
        kc[slots[n], :l] = k_rot
        vc[slots[n], :l] = v_h
    cache_len = torch.tensor(lens, dtype=torch.int32, device=DEV)
    idx = torch.from_numpy(slots).to(DEV)
    wq, wk = p["q_norm_w"].to(DEV), p["k_norm_w"].to(DEV)
    outs = []
    for s in range(steps):
        rows = [int(cu_full[n]) + lens[n] + s for n in range(N)]
        q, k, v, g = (p[name][rows].to(DEV) for name in ("q", "k", "v", "gate"))
        outs.append(f64(gdn.gdn_attention_decode(q, k, v, g, wq, wk, kc, vc, cache_len,
                                                 cache_idx=idx)))
    torch.cuda.synchronize()
    assert cache_len.cpu().tolist() == [l + steps for l in lens]
    ref, _, _ = run_oracle(p, cu_full)
    refs = [np.stack([ref[int(cu_full[n]) + lens[n] + s] for n in range(N)])
            for s in range(steps)]
    return outs, refs


def test_decode_against_the_oracle(record_property):
    lens = [0, 1, 511, 512, 513, 1023, 1500, 37]
    outs, refs = decode_case(lens, seed=5, steps=3)
    worst = 0.0
    for got, ref in zip(outs, refs):
        worst = max(worst, check(got, ref)[0])
    record_property("attn_decode_max_over_rms", worst)


def test_decode_out_of_range_slot_is_skipped():
    N, P, L = 3, 4, 64
    p = gi.attention_inputs(N, seed=7)
    d = {k: v.to(DEV) for k, v in p.items()}
    kc = torch.zeros(P, L, 4, 256, dtype=torch.float16, device=DEV)
    vc = torch.zeros_like(kc)
    idx = torch.tensor([0, P, 2], dtype=torch.int32, device=DEV)      # slot P is out of range
    cache_len = torch.tensor([0, 0, L], dtype=torch.int32, device=DEV)  # length L is full
    ws = torch.empty(gdn.load().gdn_attention_decode_workspace(N, 24, L, 256), dtype=torch.uint8,
                     device=DEV)
    o = gdn.gdn_attention_decode(d["q"], d["k"], d["v"], d["gate"], d["q_norm_w"],
                                 d["k_norm_w"], kc, vc, cache_len, cache_idx=idx, workspace=ws)
    assert gdn.gdn_attention_status(ws) == -1
    o = o.float().cpu()
    assert torch.isfinite(o[0]).all()
    assert torch.isnan(o[1]).all() and torch.isnan(o[2]).all()
    assert cache_len.cpu().tolist() == [1, 0, L]
    assert not kc[1:].any() and not kc[0, 1:].any()
    # a single cached token attends to itself: its value times the gate
    v0 = p["v"][0].double().repeat_interleave(6, dim=0)
    want = v0 / (1 + np.exp(-p["gate"][0].double()))
    assert torch.allclose(o[0].double(), want, rtol=2 ** -7, atol=1e-3)


@pytest.mark.parametrize("H_q,H_kv", [(8, 4), (16, 2)])
def test_other_head_layouts_fp32_weights_far_positions(H_q, H_kv):
    """GQA groups of 2 and 8 (other instances of the decode kernel), fp32 norm
    weights, and a prompt continuing 250 000 cached positions (rotary angles in
    the long-context range); prefill then one decode step from its cache rows."""
    lens = [90, 33]
    steps = 1
    tot = [l + steps for l in lens]
    cu_full = np.concatenate([[0], np.cumsum(tot)])
    p = gi.attention_inputs(int(cu_full[-1]), seed=11, H_q=H_q, H_kv=H_kv)
    wq = p["q_norm_w"].float()
    wk = p["k_norm_w"].float()
    pos0 = np.array([250_000, 7], dtype=np.int64)
    ref, _, kref = oracle.attention(f64(p["q"]), f64(p["k"]), f64(p["v"]), f64(p["gate"]),
                                    f64(wq), f64(wk), cu_seqlens=cu_full, pos0=pos0)
    rows = np.concatenate([np.arange(cu_full[n], cu_full[n] + l) for n, l in enumerate(lens)])
    sub = {k: p[k][rows].to(DEV) for k in ("q", "k", "v", "gate")}
    cu_p = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32, device=DEV)
    o, k_rot, v_h = gdn.gdn_attention_prefill(
        sub["q"], sub["k"], sub["v"], sub["gate"], wq.to(DEV), wk.to(DEV), cu_p,
        pos0=torch.from_numpy(pos0.astype(np.int32)).to(DEV))
    torch.cuda.synchronize()
    check(f64(o), ref[rows])
    check_cache_rows(k_rot, v_h, kref[rows], p["v"][rows])
    # one decode step at positions 250 000 + 90 and 7 + 33: positions passed explicitly
    kc = torch.zeros(2, 256, H_kv, 256, dtype=torch.float16, device=DEV)
    vc = torch.zeros_like(kc)
    for n, l in enumerate(lens):
        s0 = int(cu_p[n])
        kc[n, :l], vc[n, :l] = k_rot[s0:s0 + l], v_h[s0:s0 + l]
    new = [int(cu_full[n]) + l for n, l in enumerate(lens)]
    pos = torch.tensor([[int(pos0[n]) + l for n, l in enumerate(lens)]] * 3, dtype=torch.int32)
    lens_d = torch.tensor(lens, dtype=torch.int32, device=DEV)
    od = gdn.gdn_attention_decode(*(p[k][new].to(DEV) for k in ("q", "k", "v", "gate")),
                                  wq.to(DEV), wk.to(DEV), kc, vc, lens_d,
                                  positions=pos.to(DEV))
    torch.cuda.synchronize()
    check(f64(od), ref[new])
    assert lens_d.cpu().tolist() == [l + 1 for l in lens]
