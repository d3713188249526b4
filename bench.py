#!/usr/bin/env python3
"""Benchmark of the gated delta-rule layer on B200.

One step = one pass of the layer's prefill hot path over one synthetic batch:
causal conv k=4 + SiLU + q/k L2 (gdn_conv1d_silu) -> chunk-64 gated delta
rule (gdn_chunked_prefill) -> gated RMS-norm (gdn_gated_rmsnorm), on the
prefill workload B=1, T=8192, 16 key / 48 value heads, head dim 128, bf16
activations, fp32 gates and state. That step gives the headline "value".
The same run times, under their own keys:

  prefill_l2_flushed  the same step with a 256 MB L2 flush between steps;
  varlen              16 packed sequences of 512..16384 tokens (seeded), fp32
                      initial states in and final states out, same chain;
  decode              256 sequences, one token per step for 128 steps: conv
                      with in-place cache roll -> gdn_decode_step -> gated
                      RMS-norm, fp32 state [256,48,128,128];
  long_context        T=262144 as 64 calls of 4096 tokens with the recurrent
                      state and the conv history carried between calls (one
                      step = all 64 calls), unflushed and L2-flushed;
  attention_prefill   the decoder's global-attention layer (24 query / 4
                      key-value heads, head dim 256, q/k RMS-norm, rotary,
                      sigmoid gate) over the same B=1, T=8192 prompt;
  attention_decode    that layer's decode step for 256 sequences holding 4096
                      cached tokens each, one token per sequence per step.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
                    [--shard replicas|heads]
    python bench.py --profile-case NAME [--n N] [--t T] [--launches L]

With N > 1 (launched by torch.distributed.run) each rank either runs its own
replica of every workload on its own synthetic data ("replicas", the default:
sequences are independent, weak scaling) or takes 16/N key heads and their
3x value heads of the same workloads ("heads": the head split of a
tensor-parallel layer, strong scaling). Neither needs a data-path collective;
the slowest rank's device time is reported. `--impl reference` times the fp64
CPU oracle on the host cores on a bounded sample of the prefill workload
(rank 0 only). `--profile-case` runs a few fixed launches of one kernel for a
profiler capture and exits.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import gdn_inputs as gi  # noqa: E402

METRIC = "gated-delta-rule prefill tokens/s and decode tokens/s per layer; % of roofline"
T_PREFILL = 8192
N_DECODE = 256
DECODE_STEPS = 128
SEG, N_SEG = 4096, 64
N_VARLEN = 16
H_K, H_V, D, C = 16, 48, 128, 64
L2_FLUSH_BYTES = 256 << 20
# Algorithmic work per token and value head, chunk C=64: 6d^2 (W S^T, Q S^T, U^T K)
# + 6Cd (W, U, M U) + 4Cd/3 (K K^T, Q K^T shared by 3 value heads) + C^2/1.5
# (triangular solve).
FLOP_PER_TOKEN_HEAD = 6 * D * D + 6 * C * D + 4 * C * D / 3 + C * C / 1.5
PREFILL_FLOP_PER_TOKEN = H_V * FLOP_PER_TOKEN_HEAD
# bf16 q,k,v,o + fp32 g,beta per token
PREFILL_BYTES_PER_TOKEN = 2 * (2 * H_K * D) + 2 * H_V * D + 2 * 4 * H_V + 2 * H_V * D
# decode step kernel: fp32 state read + write, plus q,k (bf16), v, o (bf16), g, beta (bf16)
DECODE_BYTES_PER_TOKEN = 2 * H_V * D * D * 4 + 2 * (2 * H_K * D) + 2 * 2 * H_V * D + 2 * 2 * H_V
# fused decode layer step: fp32 state read + write, x (bf16, 10240 channels), the
# 3-row conv cache read and written back rolled (bf16), z and y (bf16), g, beta (bf16)
CONV_CH = 2 * H_K * D + H_V * D
FUSED_DECODE_BYTES_PER_TOKEN = (2 * H_V * D * D * 4 + 2 * CONV_CH + 2 * 3 * 2 * CONV_CH
                                + 2 * 2 * H_V * D + 2 * 2 * H_V)
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}
# Global-attention layer: S = Q K^T and O = P V over the causal triangle,
# 2 * 2 * d flops per (query, key) pair and query head.
A_HQ, A_HKV, A_D = 24, 4, 256
A_CTX = 4096                 # cached tokens per sequence at the first decode step
A_LMAX = A_CTX + 256         # cache rows per slot (room for warm-up + timed steps)


def attn_prefill_flop(T, H_q=A_HQ):
    return 4 * A_D * H_q * T * (T + 1) / 2


def attn_decode_bytes(N, L, H_q=A_HQ, H_kv=A_HKV):
    """Algorithmic bytes of one decode step with L cached tokens per sequence:
    read the L + 1 fp16 key and value rows (the new one included), write the
    new row, read q, k, v, gate (bf16), write o (bf16)."""
    row = H_kv * A_D * 2                       # one token's fp16 keys (or values)
    inputs = 2 * A_D * (2 * H_q + 2 * H_kv)    # q, gate, k, v in bf16
    return N * (2 * (L + 1) * row + 2 * row + inputs + 2 * A_D * H_q)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return PEAKS_FALLBACK, "fallback"


def kernel_traffic(kernel):
    """DRAM bytes per launch from the committed ncu summary, or None when the
    kernel's source changed since the counters were taken."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f).get(kernel)
    if not d:
        return None
    src = os.path.join(ROOT, d["source"])
    if not os.path.exists(src):
        return None
    h = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    return d["bytes_per_launch"] if h == d["source_sha256_16"] else None


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples (50 ms period) taken while
    the timed legs run."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.out = ""

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out, _ = self.proc.communicate()

    def summary(self):
        rows = []
        for line in (self.out or "").splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 8:
                continue
            try:
                rows.append((float(f[1]), float(f[2]), f[4:8]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, r in rows for i, v in enumerate(r)
                          if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in rows),
                "sm_max_mhz": max(r[1] for r in rows), "reasons": reasons,
                "samples": len(rows), "span": "every timed leg of this run"}


def head_shard(rank, world, H_k=H_K, H_v=H_V):
    """Key heads [kh0, kh1) and value heads [vh0, vh1) of one rank when the
    layer's heads are split over `world` ranks (a tensor-parallel layer):
    whole key-head groups, so local value head j reads local key head
    j // (H_v / H_k) exactly as global value head vh0 + j reads global key
    head (vh0 + j) // (H_v / H_k)."""
    if H_k % world:
        raise ValueError(f"{H_k} key heads do not split over {world} ranks")
    per = H_k // world
    grp = H_v // H_k
    kh0 = rank * per
    return kh0, kh0 + per, kh0 * grp, (kh0 + per) * grp


def attn_kv_shard(rank, world, heads):
    """Key-value heads [g0, g1) of the attention layer on one rank: with the
    head split (`heads`) and 4 key-value heads dividing over the ranks, each rank
    takes whole GQA groups (its 6 query heads per key-value head come along);
    otherwise every rank runs the whole layer."""
    if heads and A_HKV % world == 0:
        return rank * A_HKV // world, (rank + 1) * A_HKV // world
    return 0, A_HKV


def shard_channels(kh0, kh1, vh0, vh1, H_k=H_K):
    """Indices of the conv channels (q | k | v of the full layer) that a head
    shard owns, in the order q | k | v."""
    q = np.arange(kh0 * D, kh1 * D)
    k = H_k * D + np.arange(kh0 * D, kh1 * D)
    v = 2 * H_k * D + np.arange(vh0 * D, vh1 * D)
    return np.concatenate([q, k, v])


# ---------------------------------------------------------------- GPU arm --

def device_gates(gen, T, H_v, dev, dtype=torch.float32):
    """beta = sigmoid(N(0,1)), g = exp(-softplus(N(0,1))) drawn on the device."""
    nb = torch.randn((T, H_v), generator=gen, device=dev)
    ng = torch.randn((T, H_v), generator=gen, device=dev)
    return torch.exp(-torch.nn.functional.softplus(ng)).to(dtype), torch.sigmoid(nb).to(dtype)


class Layer:
    """One delta-rule layer (or a head shard of it): conv weights, the norm
    weight, and the chain conv -> chunked prefill -> gated RMS-norm on
    caller-given buffers. H_k / H_v are this rank's heads."""

    def __init__(self, gdn, dev, conv_w, H_k, H_v):
        self.gdn, self.dev = gdn, dev
        self.H_k, self.H_v = H_k, H_v
        self.qc, self.kc = H_k * D, 2 * H_k * D          # channel offsets of k and v
        self.w = conv_w.to(dev)
        self.nw = torch.ones(D, device=dev)

    def views(self, y):
        T = y.shape[0]
        return (y[:, :self.qc].view(T, self.H_k, D), y[:, self.qc:self.kc].view(T, self.H_k, D),
                y[:, self.kc:].view(T, self.H_v, D))

    def chain(self, x, cu, gate, beta, z, y, o, out, ws, state_in=None, state_out=None,
              conv_state=None, ev=None):
        g = self.gdn
        g.gdn_conv1d_silu(x, self.w, cu, conv_state_in=conv_state, conv_state_out=conv_state,
                          l2norm_channels=self.kc, y=y)
        if ev is not None:
            ev[0].record()
        q, k, v = self.views(y)
        g.gdn_chunked_prefill(q, k, v, gate, beta, cu, state_in=state_in, state_out=state_out,
                              o=o, workspace=ws)
        if ev is not None:
            ev[1].record()
        g.gdn_gated_rmsnorm(o, z, self.nw, eps=1e-6, y=out)


class PrefillWorkload:
    """The T=8192 prefill workload, device-resident (host copies kept for the
    end-to-end leg and the CPU oracle)."""

    def __init__(self, gdn, dev, seed, shard):
        kh0, kh1, vh0, vh1 = shard
        p = gi.prefill_inputs(T=T_PREFILL, seed=seed)
        ch = torch.from_numpy(shard_channels(kh0, kh1, vh0, vh1))
        self.full = (kh1 - kh0) == H_K
        self.host = {"x_pre": p["x_pre"] if self.full else p["x_pre"][:, ch].contiguous(),
                     "g": p["g"][:, vh0:vh1].contiguous(), "beta": p["beta"][:, vh0:vh1].contiguous(),
                     "z": p["z"][:, vh0:vh1].contiguous()}
        self.layer = Layer(gdn, dev, p["conv_w"][ch], kh1 - kh0, vh1 - vh0)
        self.x = self.host["x_pre"].to(dev)
        self.g, self.b = self.host["g"].to(dev), self.host["beta"].to(dev)
        self.z = self.host["z"].to(dev)
        self.cu = p["cu_seqlens"].to(dev)
        Hv = vh1 - vh0
        self.y = torch.empty_like(self.x)
        self.o = torch.empty((T_PREFILL, Hv, D), dtype=torch.bfloat16, device=dev)
        self.out = torch.empty_like(self.o)
        self.state = torch.empty((1, Hv, D, D), dtype=torch.float32, device=dev)
        self.ws = torch.empty(max(1, gdn.gdn_chunked_prefill_workspace(1, T_PREFILL, kh1 - kh0, Hv)),
                              dtype=torch.uint8, device=dev)
        self.layer_ws = torch.empty(
            max(1, gdn.gdn_prefill_layer_workspace(1, T_PREFILL, kh1 - kh0, Hv)),
            dtype=torch.uint8, device=dev)
        self.launches_per_step = 3
        self.tokens = T_PREFILL
        self.flop = T_PREFILL * Hv * FLOP_PER_TOKEN_HEAD

    def step(self, i, ev=None):
        self.chain(self.x, self.g, self.b, self.z, self.out, ev)

    def chain(self, x, gate, beta, z, out, ev=None):
        self.layer.chain(x, self.cu, gate, beta, z, self.y, self.o, out, self.ws,
                         state_out=self.state, ev=ev)

    def step_fused(self, i, ev=None):
        """The same pass as one gdn_prefill_layer launch (conv in the load stage,
        norm before the outputs leave)."""
        L = self.layer
        if ev is not None:
            ev[0].record()
        L.gdn.gdn_prefill_layer(self.x, L.w, self.g, self.b, self.cu, self.z, L.nw,
                                state_out=self.state, y=self.out, H_k=L.H_k,
                                workspace=self.layer_ws)
        if ev is not None:
            ev[1].record()


class VarlenWorkload:
    """16 packed sequences, lengths uniform in [512, 16384] (seeded), fp32
    initial states ~N(0, 0.02) in, final states out; inputs drawn on the
    device with the prefill workload's distributions."""

    def __init__(self, gdn, dev, seed, shard):
        kh0, kh1, vh0, vh1 = shard
        Hk, Hv = kh1 - kh0, vh1 - vh0
        cu = gi.varlen_cu_seqlens(N_VARLEN, 512, 16384, seed=seed)
        T = int(cu[-1])
        gen = torch.Generator(device=dev)
        gen.manual_seed(1000 + seed)
        ch = torch.from_numpy(shard_channels(kh0, kh1, vh0, vh1))
        self.layer = Layer(gdn, dev, gi.conv_weight(seed)[ch], Hk, Hv)
        self.cu = cu.to(dev)
        self.x = torch.randn((T, len(ch)), generator=gen, device=dev).to(torch.bfloat16)
        self.g, self.b = device_gates(gen, T, Hv, dev)
        self.z = torch.randn((T, Hv, D), generator=gen, device=dev).to(torch.bfloat16)
        self.s_in = torch.randn((N_VARLEN, Hv, D, D), generator=gen, device=dev) * gi.STATE_VAR ** 0.5
        self.s_out = torch.empty_like(self.s_in)
        self.y = torch.empty_like(self.x)
        self.o = torch.empty((T, Hv, D), dtype=torch.bfloat16, device=dev)
        self.out = torch.empty_like(self.o)
        self.ws = torch.empty(max(1, gdn.gdn_chunked_prefill_workspace(N_VARLEN, T, Hk, Hv)),
                              dtype=torch.uint8, device=dev)
        self.tokens = T
        self.flop = T * Hv * FLOP_PER_TOKEN_HEAD
        self.launches_per_step = 3

    def step(self, i, ev=None):
        self.layer.chain(self.x, self.cu, self.g, self.b, self.z, self.y, self.o, self.out,
                         self.ws, state_in=self.s_in, state_out=self.s_out, ev=ev)


class LongContextWorkload:
    """T=262144 as 64 calls of 4096 tokens; the recurrent state and the conv
    history are carried from call to call. One step = all 64 calls."""

    def __init__(self, gdn, dev, seed, shard):
        kh0, kh1, vh0, vh1 = shard
        Hk, Hv = kh1 - kh0, vh1 - vh0
        gen = torch.Generator(device=dev)
        gen.manual_seed(2000 + seed)
        ch = torch.from_numpy(shard_channels(kh0, kh1, vh0, vh1))
        nch = len(ch)
        self.layer = Layer(gdn, dev, gi.conv_weight(seed)[ch], Hk, Hv)
        T = SEG * N_SEG
        self.x = torch.randn((T, nch), generator=gen, device=dev).to(torch.bfloat16)
        self.g, self.b = device_gates(gen, T, Hv, dev)
        self.z = torch.randn((T, Hv, D), generator=gen, device=dev).to(torch.bfloat16)
        self.cu = torch.tensor([0, SEG], dtype=torch.int32, device=dev)
        self.state = torch.zeros((1, Hv, D, D), device=dev)
        self.cache = torch.zeros((1, 3, nch), dtype=torch.bfloat16, device=dev)
        self.y = torch.empty((SEG, nch), dtype=torch.bfloat16, device=dev)
        self.o = torch.empty((SEG, Hv, D), dtype=torch.bfloat16, device=dev)
        self.out = torch.empty((T, Hv, D), dtype=torch.bfloat16, device=dev)
        self.ws = torch.empty(max(1, gdn.gdn_chunked_prefill_workspace(1, SEG, Hk, Hv)),
                              dtype=torch.uint8, device=dev)
        self.tokens = T
        self.flop = T * Hv * FLOP_PER_TOKEN_HEAD
        self.launches_per_step = N_SEG * 4     # conv, cache roll, prefill, norm

    def segment(self, s, ev=None):
        a, e = s * SEG, (s + 1) * SEG
        self.layer.chain(self.x[a:e], self.cu, self.g[a:e], self.b[a:e], self.z[a:e], self.y,
                         self.o, self.out[a:e], self.ws, state_in=self.state,
                         state_out=self.state, conv_state=self.cache, ev=ev)


class DecodeWorkload:
    """256 sequences, one token per step. fused: one gdn_decode_layer_step per
    step on state and conv-cache pools indexed through a seeded permutation;
    otherwise conv (in-place cache roll) -> gdn_decode_step -> gated RMS-norm."""

    def __init__(self, gdn, dev, seed, steps, shard, fused):
        kh0, kh1, vh0, vh1 = shard
        Hk, Hv = kh1 - kh0, vh1 - vh0
        ch = torch.from_numpy(shard_channels(kh0, kh1, vh0, vh1))
        self.gdn, self.fused = gdn, fused
        self.idx = torch.from_numpy(
            np.random.default_rng(seed).permutation(N_DECODE).astype(np.int32)).to(dev)
        init = gi.decode_initial(N_DECODE, seed)
        self.state = init["state"][:, vh0:vh1].contiguous().to(dev)
        self.cache = init["conv_state"][:, :, ch].contiguous().to(dev)
        self.layer = Layer(gdn, dev, gi.conv_weight(seed)[ch], Hk, Hv)
        self.cu = torch.arange(N_DECODE + 1, dtype=torch.int32, device=dev)
        self.inputs = []
        for s in range(steps):
            st = gi.decode_step_inputs(s, N_DECODE, seed)
            self.inputs.append({"x_pre": st["x_pre"][:, ch].contiguous().to(dev),
                                "g": st["g"][:, vh0:vh1].contiguous().to(dev),
                                "beta": st["beta"][:, vh0:vh1].contiguous().to(dev),
                                "z": st["z"][:, vh0:vh1].contiguous().to(dev)})
        self.y = torch.empty((N_DECODE, len(ch)), dtype=torch.bfloat16, device=dev)
        self.o = torch.empty((N_DECODE, Hv, D), dtype=torch.bfloat16, device=dev)
        self.out = torch.empty_like(self.o)
        self.launches_per_step = 2 if fused else 4
        frac = Hv / H_V
        self.bytes = int(N_DECODE * frac * (FUSED_DECODE_BYTES_PER_TOKEN if fused
                                            else DECODE_BYTES_PER_TOKEN))

    def step(self, s, ev=None):
        g, st, L = self.gdn, self.inputs[s % len(self.inputs)], self.layer
        if self.fused:
            if ev is not None:
                ev[0].record()
            g.gdn_decode_layer_step(st["x_pre"], L.w, self.cache, st["g"], st["beta"],
                                    self.state, self.idx, st["z"], L.nw, y=self.out,
                                    H_k=L.H_k)
            if ev is not None:
                ev[1].record()
            return
        g.gdn_conv1d_silu(st["x_pre"], L.w, self.cu, conv_state_in=self.cache,
                          conv_state_out=self.cache, l2norm_channels=L.kc, y=self.y)
        if ev is not None:
            ev[0].record()
        q, k, v = L.views(self.y)
        g.gdn_decode_step(q, k, v, st["g"], st["beta"], self.state, o=self.o)
        if ev is not None:
            ev[1].record()
        g.gdn_gated_rmsnorm(self.o, st["z"], L.nw, eps=1e-6, y=self.out)


class AttentionPrefillWorkload:
    """The global-attention layer over the B=1, T=8192 prompt: q, k, v, gate
    bf16 N(0, 1), norm weights 1 + N(0, 0.01); one gdn_attention_prefill call
    (q/k norm + rotary launch, attention launch) per step."""

    def __init__(self, gdn, dev, seed, kv=(0, A_HKV)):
        self.gdn = gdn
        G = A_HQ // A_HKV
        self.H_kv = kv[1] - kv[0]
        self.H_q = self.H_kv * G
        p = gi.attention_inputs(T_PREFILL, seed=seed)
        qh = slice(kv[0] * G, kv[1] * G)
        self.q = p["q"][:, qh].contiguous().to(dev)
        self.gate = p["gate"][:, qh].contiguous().to(dev)
        self.k = p["k"][:, kv[0]:kv[1]].contiguous().to(dev)
        self.v = p["v"][:, kv[0]:kv[1]].contiguous().to(dev)
        self.wq, self.wk = p["q_norm_w"].to(dev), p["k_norm_w"].to(dev)
        self.cu = torch.tensor([0, T_PREFILL], dtype=torch.int32, device=dev)
        self.o = torch.empty_like(self.q)
        self.k_rot = torch.empty(self.k.shape, dtype=torch.float16, device=dev)
        self.v_h = torch.empty_like(self.k_rot)
        self.ws = torch.empty(gdn.load().gdn_attention_prefill_workspace(T_PREFILL, self.H_q, A_D),
                              dtype=torch.uint8, device=dev)
        self.flop = attn_prefill_flop(T_PREFILL, self.H_q)

    def step(self, i, ev=None):
        if ev is not None:
            ev[0].record()
        self.gdn.gdn_attention_prefill(self.q, self.k, self.v, self.gate, self.wq, self.wk,
                                       self.cu, o=self.o, k_rot=self.k_rot, v_h=self.v_h,
                                       workspace=self.ws)
        if ev is not None:
            ev[1].record()


class AttentionDecodeWorkload:
    """256 sequences in permuted pool slots, A_CTX cached tokens each (fp16
    keys and values drawn N(0, 1) on the device, seeded); each step decodes
    one new token per sequence (q, k, v, gate bf16 N(0, 1)), which appends to
    the caches and advances cache_len."""

    def __init__(self, gdn, dev, seed, steps, kv=(0, A_HKV), n=N_DECODE):
        self.gdn, self.n = gdn, n
        G = A_HQ // A_HKV
        self.H_kv = kv[1] - kv[0]
        self.H_q = self.H_kv * G
        gen = torch.Generator(device=dev)
        gen.manual_seed(1000 + seed)
        shape = (n, A_LMAX, self.H_kv, A_D)
        self.kc = torch.randn(shape, generator=gen, device=dev, dtype=torch.float16)
        self.vc = torch.randn(shape, generator=gen, device=dev, dtype=torch.float16)
        self.idx = torch.from_numpy(
            np.random.default_rng(seed).permutation(n).astype(np.int32)).to(dev)
        self.len = torch.full((n,), A_CTX, dtype=torch.int32, device=dev)
        self.inputs = []
        for s in range(min(steps, 16)):
            a = gi.attention_inputs(n, seed=seed, tag=("attn_decode", s))
            self.inputs.append({k: (v[:, kv[0] * G:kv[1] * G] if k in ("q", "gate") else
                                    v[:, kv[0]:kv[1]] if k in ("k", "v") else v)
                                .contiguous().to(dev) for k, v in a.items()})
        self.o = torch.empty((n, self.H_q, A_D), dtype=torch.bfloat16, device=dev)
        self.ws = torch.empty(gdn.load().gdn_attention_decode_workspace(n, self.H_q, A_LMAX, A_D),
                              dtype=torch.uint8, device=dev)

    def reset(self):
        self.len.fill_(A_CTX)

    def bytes_for(self, first_len, steps):
        return sum(attn_decode_bytes(self.n, first_len + s, self.H_q, self.H_kv)
                   for s in range(steps))

    def step(self, s, ev=None):
        st = self.inputs[s % len(self.inputs)]
        if ev is not None:
            ev[0].record()
        self.gdn.gdn_attention_decode(st["q"], st["k"], st["v"], st["gate"], st["q_norm_w"],
                                      st["k_norm_w"], self.kc, self.vc, self.len,
                                      cache_idx=self.idx, o=self.o, workspace=self.ws)
        if ev is not None:
            ev[1].record()


class RankGroup:
    """Barrier and max-over-ranks around the timed regions; no-ops at one rank.
    `dist` is torch.distributed with an initialised process group (NCCL on the
    GPUs; gloo works the same on CPU tensors) and `device` where its reductions
    run."""

    def __init__(self, dist=None, device=None):
        self.dist, self.device = dist, device

    def barrier(self):
        if self.dist is not None:
            self.dist.barrier()

    def max(self, v):
        if self.dist is None:
            return v
        t = torch.tensor([v], dtype=torch.float64, device=self.device)
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX)
        return float(t.item())


def throughput(units_per_rank, world, max_ms):
    """Whole-job units per second: the units every rank processed over the
    slowest rank's time."""
    return units_per_rank * world / (max_ms * 1e-3)


class KernelEvents:
    """CUDA-event pairs around a step's calls of its dominant kernel, on the
    launching stream: ev[0].record() opens a pair, ev[1].record() closes it
    (a step that calls the kernel several times records several pairs)."""

    def __init__(self):
        self.pairs = []

    def __getitem__(self, j):
        if j == 0:
            self.pairs.append([torch.cuda.Event(enable_timing=True) for _ in range(2)])
        return self.pairs[-1][j]

    def ms(self):
        return sum(a.elapsed_time(b) for a, b in self.pairs)


def timed_loop(step_fn, steps, warmup, dist_barrier, flush=None):
    """Warm up, then time exactly `steps` steps. Each step's region and its
    dominant kernel are bracketed by CUDA events on the current (launching)
    stream. Without `flush` the steps run back to back (every workload's
    inputs exceed the 126 MB L2, and each step also pays the previous step's
    write-backs); with it, `flush()` writes a buffer larger than L2 between
    steps, outside the events. Returns (per-step ms, per-step kernel ms)."""
    for i in range(warmup):
        step_fn(i, None)
    torch.cuda.synchronize()
    dist_barrier()
    torch.cuda.synchronize()
    rec = []
    for i in range(steps):
        if flush is not None:
            flush()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        kev = KernelEvents()
        a.record()
        step_fn(i, kev)
        b.record()
        rec.append((a, b, kev))
    torch.cuda.synchronize()
    dist_barrier()
    return [a.elapsed_time(b) for a, b, _ in rec], [k.ms() for _, _, k in rec]


def e2e_prefill(wl, dev, steps, warmup):
    """Same workload through the public API from pinned HOST buffers: every
    step's inputs are copied host->device and its output device->host inside
    the timed region. Steps are pipelined as a serving loop would run them:
    copy-in, compute and copy-out each have a stream, and two device sets of
    input and output buffers let step i's copies overlap the compute of steps
    i-1 and i+1 (events order every reuse of a buffer)."""
    h = wl.host
    hx = h["x_pre"].pin_memory()
    hg, hb, hz = h["g"].pin_memory(), h["beta"].pin_memory(), h["z"].pin_memory()
    houts = [torch.empty(wl.out.shape, dtype=wl.out.dtype).pin_memory() for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in (hx, hg, hb, hz))
    d2h = houts[0].numel() * houts[0].element_size()
    sets = [(wl.x, wl.g, wl.b, wl.z, wl.out)]
    sets.append(tuple(torch.empty_like(t) for t in sets[0]))
    s_in, s_comp, s_out = (torch.cuda.Stream(dev) for _ in range(3))
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    used = [False, False]

    def one(i):
        j = i % 2
        x, gate, beta, z, out = sets[j]
        with torch.cuda.stream(s_in):
            if used[j]:
                s_in.wait_event(ev_comp[j])      # step i-2 has read this input set
            x.copy_(hx, non_blocking=True)
            gate.copy_(hg, non_blocking=True)
            beta.copy_(hb, non_blocking=True)
            z.copy_(hz, non_blocking=True)
            ev_in[j].record(s_in)
        with torch.cuda.stream(s_comp):
            s_comp.wait_event(ev_in[j])
            if used[j]:
                s_comp.wait_event(ev_out[j])     # step i-2's output has left this buffer
            wl.chain(x, gate, beta, z, out)
            ev_comp[j].record(s_comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_comp[j])
            houts[j].copy_(out, non_blocking=True)
            ev_out[j].record(s_out)
        used[j] = True

    for i in range(warmup):
        one(i)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(s_in)
    for i in range(steps):
        one(warmup + i)
    s_in.wait_stream(s_out)
    b.record(s_in)
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / steps
    return ms, h2d, d2h


def tensor_roofline(name, flop, kms, peaks, peak_src, traffic):
    ach = flop / (kms * 1e-3) / 1e12
    return {"kernel": name, "bound": "tensor", "achieved": ach, "peak": peaks["bf16_tflops"],
            "unit": "TFLOP/s", "frac": ach / peaks["bf16_tflops"],
            "peak_source": f"{peak_src} bf16 dense (burst)", "traffic": traffic,
            "algorithmic_flop_per_launch": flop, "kernel_ms": kms}


def gpu_arm(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA GPU (B200)")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    group = RankGroup(dist, dev)
    barrier, max_over_ranks = group.barrier, group.max

    import gated_delta_rule_106_b200 as gdn
    gdn.load()
    peaks, peak_src = load_peaks()
    heads = args.shard == "heads" and world > 1
    shard = head_shard(rank, world) if heads else (0, H_K, 0, H_V)
    seed = 0 if heads else rank     # head shards split one workload; replicas draw their own
    flush_buf = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    flush = lambda: flush_buf.fill_(1)
    mean_max = lambda xs: max_over_ranks(statistics.mean(xs))

    pre = PrefillWorkload(gdn, dev, seed, shard)
    with ClockSampler(local) as clk:
        step_ms, kern_ms = timed_loop(pre.step, args.steps, args.warmup, barrier)
        ms, kms = mean_max(step_ms), mean_max(kern_ms)
        f_step, f_kern = timed_loop(pre.step, args.steps, args.warmup, barrier, flush=flush)
        f_ms, f_kms = mean_max(f_step), mean_max(f_kern)
        u_step, _ = timed_loop(pre.step_fused, args.steps, args.warmup, barrier)
        fu_ms = mean_max(u_step)

        var = VarlenWorkload(gdn, dev, seed, shard)
        v_step, v_kern = timed_loop(var.step, args.steps, args.warmup, barrier)
        v_ms, v_kms = mean_max(v_step), mean_max(v_kern)
        v_tokens, v_flop = var.tokens, var.flop
        del var

        dwl = DecodeWorkload(gdn, dev, seed, DECODE_STEPS, shard, fused=True)
        d_step, d_kern = timed_loop(dwl.step, DECODE_STEPS, args.warmup, barrier)
        d_ms, d_kms = mean_max(d_step), mean_max(d_kern)
        d_bytes = dwl.bytes
        del dwl
        uwl = DecodeWorkload(gdn, dev, seed, DECODE_STEPS, shard, fused=False)
        u_step, u_kern = timed_loop(uwl.step, DECODE_STEPS, args.warmup, barrier)
        u_ms, u_kms = mean_max(u_step), mean_max(u_kern)
        u_bytes = uwl.bytes
        del uwl

        lc = LongContextWorkload(gdn, dev, seed, shard)
        lsteps = max(1, min(args.steps, 5))
        lc_fn = lambda i, ev: [lc.segment(s, ev) for s in range(N_SEG)]
        l_step, l_kern = timed_loop(lc_fn, lsteps, 1, barrier)
        l_ms, l_kms = mean_max(l_step), mean_max(l_kern)
        # flushed: L2 written between the 64 calls (outside the events)
        seg_ms, seg_kern = timed_loop(lambda i, ev: lc.segment(i % N_SEG, ev), N_SEG, 1,
                                      barrier, flush=flush)
        lf_ms, lf_kms = max_over_ranks(sum(seg_ms)), max_over_ranks(sum(seg_kern))
        l_tokens, l_flop = lc.tokens, lc.flop
        del lc

        # global-attention layer; head shards split its 4 key-value heads
        akv = attn_kv_shard(rank, world, heads)
        apre = AttentionPrefillWorkload(gdn, dev, seed, akv)
        a_step, a_kern = timed_loop(apre.step, args.steps, args.warmup, barrier)
        a_ms, a_kms = mean_max(a_step), mean_max(a_kern)
        a_flop = apre.flop
        del apre
        adec = AttentionDecodeWorkload(gdn, dev, seed, DECODE_STEPS, akv)
        adec.reset()
        ad_step, ad_kern = timed_loop(adec.step, DECODE_STEPS, args.warmup, barrier)
        ad_ms, ad_kms = mean_max(ad_step), mean_max(ad_kern)
        ad_bytes = adec.bytes_for(A_CTX + args.warmup, DECODE_STEPS) / DECODE_STEPS
        del adec
    e2e_ms, h2d, d2h = e2e_prefill(pre, dev, max(4, args.steps), 2)
    e2e_ms = max_over_ranks(e2e_ms)

    Hv = shard[3] - shard[2]
    flops = pre.flop
    dec_ach = d_bytes / (d_kms * 1e-3) / 1e9
    u_ach = u_bytes / (u_kms * 1e-3) / 1e9
    units = 1 if heads else world       # head shards together make one workload
    line = {
        "metric": METRIC,
        "value": throughput(T_PREFILL, units, ms),
        "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms,
        "higher_is_better": True,
        "scaling": "strong" if heads else "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded; shapes and distributions of the layer)",
        "config": {
            "workload": "prefill: one delta-rule layer, B=1, T=8192, 16 key / 48 value "
                        "heads, d=128; conv k=4+SiLU+L2 -> chunked C=64 -> gated RMSNorm",
            "global_batch": units, "seq_len": T_PREFILL,
            "parallelism": (f"heads{world} ({shard[1] - shard[0]} key / {Hv} value heads per rank)"
                            if heads else (f"replicas{world}" if world > 1 else "single")),
            "l2": "no flush: inputs exceed L2 (x_pre 168 MB; decode state 768 MiB); steps run "
                  "back to back (flushed variant under prefill_l2_flushed)",
        },
        "roofline": tensor_roofline("gdn_chunked_prefill", flops, kms, peaks, peak_src,
                                    kernel_traffic("prefill") if not heads else None),
        "e2e": {"value": throughput(T_PREFILL, units, e2e_ms), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": e2e_ms},
        "gpu_launches": pre.launches_per_step * args.steps,
        "clocks": clk.summary(),
        "prefill_layer_fused": {
            "workload": "the same prefill step as one gdn_prefill_layer call: q/k conv + "
                        "SiLU + L2 once per key head, then the chunk kernel with the v conv in "
                        "its load stage and the gated RMSNorm before the outputs leave",
            "value": throughput(T_PREFILL, units, fu_ms), "unit": "tokens/s",
            "ms_per_step": fu_ms, "gpu_launches": 2 * args.steps,
            "roofline": tensor_roofline("gdn_prefill_layer", flops, fu_ms, peaks, peak_src, None)},
        "prefill_l2_flushed": {
            "value": throughput(T_PREFILL, units, f_ms), "unit": "tokens/s", "ms_per_step": f_ms,
            "l2": f"{L2_FLUSH_BYTES >> 20} MB written between steps (outside the events)",
            "roofline": tensor_roofline("gdn_chunked_prefill", flops, f_kms, peaks, peak_src,
                                        None)},
        "varlen": {
            "workload": f"{N_VARLEN} packed sequences, lengths uniform in [512, 16384] "
                        f"({v_tokens} tokens), fp32 initial/final states; conv -> chunked "
                        "prefill -> gated RMSNorm",
            "value": throughput(v_tokens, units, v_ms), "unit": "tokens/s", "ms_per_step": v_ms,
            "roofline": tensor_roofline("gdn_chunked_prefill", v_flop, v_kms, peaks, peak_src,
                                        None),
            "gpu_launches": 3 * args.steps},
        "decode": {
            "workload": "decode: 256 sequences x 128 steps, 1 token each, fp32 state pool "
                        "[256,48,128,128] and conv-cache pool through a permuted state_idx; "
                        "one fused launch per step (conv roll + SiLU + L2 -> recurrence -> "
                        "gated RMSNorm)",
            "value": throughput(N_DECODE, units, d_ms), "unit": "tokens/s",
            "ms_per_step": d_ms,
            "roofline": {"kernel": "gdn_decode_layer_step", "bound": "hbm",
                         "achieved": dec_ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": dec_ach / peaks["hbm_gbs"],
                         "peak_source": f"{peak_src} HBM copy",
                         "traffic": kernel_traffic("decode_layer") if not heads else None,
                         "algorithmic_bytes_per_launch": d_bytes, "kernel_ms": d_kms},
            "gpu_launches": 2 * DECODE_STEPS,
        },
        "decode_unfused": {
            "workload": "the same decode workload as three calls per step: conv (cache roll) "
                        "-> decode step -> gated RMSNorm",
            "value": throughput(N_DECODE, units, u_ms), "unit": "tokens/s",
            "ms_per_step": u_ms,
            "roofline": {"kernel": "gdn_decode_step", "bound": "hbm",
                         "achieved": u_ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": u_ach / peaks["hbm_gbs"],
                         "peak_source": f"{peak_src} HBM copy",
                         "traffic": kernel_traffic("decode") if not heads else None,
                         "algorithmic_bytes_per_launch": u_bytes, "kernel_ms": u_kms},
            "gpu_launches": 4 * DECODE_STEPS,
        },
        "long_context": {
            "workload": f"T={SEG * N_SEG} as {N_SEG} calls of {SEG} tokens, recurrent state "
                        "and conv history carried; one step = all calls",
            "value": throughput(l_tokens, units, l_ms), "unit": "tokens/s", "ms_per_step": l_ms,
            "steps": lsteps,
            "roofline": tensor_roofline("gdn_chunked_prefill", l_flop, l_kms, peaks, peak_src,
                                        None),
            "l2_flushed": {"value": throughput(l_tokens, units, lf_ms), "unit": "tokens/s",
                           "ms_per_step": lf_ms,
                           "l2": f"{L2_FLUSH_BYTES >> 20} MB written between the calls",
                           "roofline": tensor_roofline("gdn_chunked_prefill", l_flop, lf_kms,
                                                       peaks, peak_src, None)},
            "gpu_launches": 4 * N_SEG * lsteps,
        },
    }
    a_units = 1 if (heads and A_HKV % world == 0) else world
    ad_ach = ad_bytes / (ad_kms * 1e-3) / 1e9
    line["attention_prefill"] = {
        "workload": "global-attention layer (24 query / 4 key-value heads, head dim 256, q/k "
                    "RMS-norm, rotary on 64 dims, causal, sigmoid gate), B=1, T=8192; one "
                    "gdn_attention_prefill call (norm+rotary launch, attention launch)",
        "value": throughput(T_PREFILL, a_units, a_ms), "unit": "tokens/s", "ms_per_step": a_ms,
        "roofline": dict(tensor_roofline("gdn_attention_prefill", a_flop, a_kms, peaks, peak_src,
                                         kernel_traffic("attention") if not heads else None),
                         dtype="fp16 operands (same dense rate as bf16)",
                         kernel_ms_includes="the q/k norm + rotary launch"),
        "gpu_launches": 2 * args.steps}
    line["attention_decode"] = {
        "workload": f"global-attention decode: {N_DECODE} sequences in permuted pool slots, "
                    f"{A_CTX} cached tokens each at the first step (+1 per step), fp16 KV "
                    "cache, one token per sequence per step",
        "value": throughput(N_DECODE, a_units, ad_ms), "unit": "tokens/s", "ms_per_step": ad_ms,
        "roofline": {"kernel": "gdn_attention_decode", "bound": "hbm", "achieved": ad_ach,
                     "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": ad_ach / peaks["hbm_gbs"],
                     "peak_source": f"{peak_src} HBM copy",
                     "traffic": kernel_traffic("attention_decode") if not heads else None,
                     "algorithmic_bytes_per_launch": ad_bytes, "kernel_ms": ad_kms},
        "gpu_launches": 3 * DECODE_STEPS}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        acb = attention_cpu_baseline()
        line["attention_prefill"]["cpu_baseline"] = acb["prefill"]
        line["attention_decode"]["cpu_baseline"] = acb["decode"]
        cb, ref_out, nheads = cpu_baseline(args.cpu_budget_s)
        line["cpu_baseline"] = cb
        got = pre.out[:, :nheads].double().cpu().numpy()
        d = got - ref_out
        line["chain_error"] = {
            "what": "normed layer output of the timed step vs the fp64 oracle chain (conv -> "
                    "recurrence -> gated RMSNorm) from the same x_pre, no GPU intermediate",
            "value_heads": nheads,
            "max_abs_over_rms": float(np.abs(d).max() / np.sqrt(np.mean(ref_out ** 2))),
            "rel_frobenius": float(np.linalg.norm(d) / np.linalg.norm(ref_out))}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


# ---------------------------------------------------------------- CPU arm --

def oracle_sample(threads=0, heads=H_V, tokens=T_PREFILL, seed=0):
    """The oracle on (part of) the prefill workload: conv of every channel of
    `tokens` tokens, the recurrence for `heads` value heads (whole key-head
    groups) and the gated RMS-norm of those heads. Returns (seconds, threads,
    normed output [tokens, heads, 128])."""
    import oracle
    p = gi.prefill_inputs(T=tokens, seed=seed)
    x = gi.as_f64(p["x_pre"])
    w = gi.as_f64(p["conv_w"])
    cu = np.array([0, tokens], dtype=np.int32)
    hw = oracle.hardware_threads()
    nthreads = min(threads or hw, heads)
    t0 = time.perf_counter()
    y, _ = oracle.conv1d_silu_l2(x, w, None, cu, None, gi.L2_CHANNELS, 1e-6)
    nk = heads // 3
    q = y[:, :2048].reshape(tokens, H_K, D)[:, :nk]
    k = y[:, 2048:4096].reshape(tokens, H_K, D)[:, :nk]
    v = y[:, 4096:].reshape(tokens, H_V, D)[:, :heads]
    o, _ = oracle.recurrence(q, k, v, gi.as_f64(p["g"])[:, :heads],
                             gi.as_f64(p["beta"])[:, :heads], None, cu,
                             threads=nthreads)
    out = oracle.gated_rmsnorm(o, gi.as_f64(p["z"])[:, :heads], gi.as_f64(p["norm_w"]),
                               1e-6, threads=nthreads)
    return time.perf_counter() - t0, nthreads, out


def cpu_baseline(budget_s=20.0):
    """Oracle throughput on the host cores, scaled to tokens/s of the whole
    layer: a short probe on 3 heads sizes a sample of ~budget_s seconds.
    Returns (baseline dict, the oracle's normed output, its value heads)."""
    probe_s, _, _ = oracle_sample(heads=3, tokens=1024)
    hw = os.cpu_count() or 1
    # conv dominates the probe's fixed part; size heads so the sample fits
    est_per_head = probe_s / 3 * (T_PREFILL / 1024)
    heads = int(max(3, min(H_V, (budget_s / max(est_per_head, 1e-9)) * min(hw, H_V))))
    heads -= heads % 3
    sec, threads, out = oracle_sample(heads=heads)
    # the conv covers all heads already; scale the recurrence+norm share
    layer_s = sec * (H_V / heads) if heads < H_V else sec
    return ({"value": T_PREFILL / layer_s, "unit": "tokens/s", "cores": threads,
             "kind": "oracle",
             "sample": f"T={T_PREFILL}: full conv, recurrence + gated RMSNorm for "
                       f"{heads}/{H_V} value heads ({sec:.1f} s), scaled to 48 heads"},
            out, heads)


def attention_cpu_baseline(rows=64, dec_seqs=4):
    """The attention oracle (fp64, host threads over (sequence, query head)) on
    bounded samples of the two attention legs, scaled to a whole call:
    prefill -- the last `rows` query rows of the T=8192 prompt (each attends to
    ~8k keys), scaled by the number of (query, key) pairs of the causal call;
    decode -- `dec_seqs` sequences whose last row attends to A_CTX + 1 keys, scaled
    to the leg's 256 sequences."""
    import oracle
    f = gi.as_f64
    out = {}
    a = gi.attention_inputs(T_PREFILL, seed=0)
    want = list(range(T_PREFILL - rows, T_PREFILL))
    t0 = time.perf_counter()
    oracle.attention(*(f(a[k]) for k in ("q", "k", "v", "gate", "q_norm_w", "k_norm_w")),
                     rows=want)
    sec = time.perf_counter() - t0
    pairs_sampled = sum(t + 1 for t in want)
    call_s = sec * (T_PREFILL * (T_PREFILL + 1) / 2) / pairs_sampled
    out["prefill"] = {"value": T_PREFILL / call_s, "unit": "tokens/s",
                      "cores": min(oracle.hardware_threads(), A_HQ), "kind": "oracle",
                      "sample": f"T={T_PREFILL}: the last {rows} query rows, all 24 heads "
                                f"({sec:.1f} s), scaled by (query, key) pairs to the call"}
    L = A_CTX + 1
    cu = np.arange(dec_seqs + 1, dtype=np.int64) * L
    d = gi.attention_inputs(int(cu[-1]), seed=1)
    t0 = time.perf_counter()
    oracle.attention(*(f(d[k]) for k in ("q", "k", "v", "gate", "q_norm_w", "k_norm_w")),
                     cu_seqlens=cu.astype(np.int32), rows=list(cu[1:] - 1))
    sec = time.perf_counter() - t0
    step_s = sec * N_DECODE / dec_seqs
    out["decode"] = {"value": N_DECODE / step_s, "unit": "tokens/s",
                     "cores": min(oracle.hardware_threads(), dec_seqs * A_HQ), "kind": "oracle",
                     "sample": f"{dec_seqs} sequences x {L} keys, the last row each ({sec:.1f} s, "
                               f"q/k norm and rotary of every row included), scaled to "
                               f"{N_DECODE} sequences"}
    return out


def reference_arm(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    # each step: the oracle on a bounded sample of the prefill workload
    heads = 3
    for _ in range(args.warmup):
        oracle_sample(heads=heads, tokens=1024)
    secs = []
    threads = 0
    for _ in range(args.steps):
        s, threads, _ = oracle_sample(heads=heads, tokens=1024)
        secs.append(s)
    per_step = statistics.mean(secs)
    # tokens/s of the whole layer: 1024 tokens, 3 of 48 heads (conv: all)
    value = 1024 / (per_step * H_V / heads)
    line = {
        "impl": "reference",
        "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": int(os.environ.get("WORLD_SIZE", "1")), "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": per_step * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic",
        "config": {"workload": "prefill: one delta-rule layer, B=1, T=8192, 16 key / 48 "
                               "value heads, d=128 (sampled: 1024 tokens, 3 heads per step)",
                   "global_batch": 1, "seq_len": T_PREFILL, "parallelism": "host threads"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads,
                         "kind": "oracle",
                         "sample": "1024 tokens: full conv, recurrence + norm for 3 of 48 "
                                   "value heads, scaled to the layer"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------- profiler cases --

def profile_case(args):
    """A few fixed launches of one kernel, for a profiler capture. Inputs are
    synthetic and seeded, larger than the 126 MB L2 at the defaults (so DRAM
    counters mean something) and a few GB at most. Prints the mean CUDA-event
    time per launch, for reference only."""
    import gated_delta_rule_106_b200 as gdn
    gdn.load()
    dev = "cuda"
    name, N, T = args.profile_case, args.n, args.t
    if name == "decode":
        st = gi.decode_step_inputs(0, N, seed=0)
        state = gi.initial_states(0, N, tag="pstate").to(dev)
        q = gi.to_bf16(gi.unit_heads(0, "pq", N, 16)).to(dev)
        k = gi.to_bf16(gi.unit_heads(0, "pk", N, 16)).to(dev)
        v = gi.to_bf16(gi.normal(0, "pv", (N, 48, 128))).to(dev)
        g, b = st["g"].to(dev), st["beta"].to(dev)
        o = torch.empty((N, 48, 128), dtype=torch.bfloat16, device=dev)
        run = lambda: gdn.gdn_decode_step(q, k, v, g, b, state, o=o, scale=0.05)
    elif name in ("prefill", "varlen"):
        cu = (torch.tensor([0, T], dtype=torch.int32) if name == "prefill"
              else gi.varlen_cu_seqlens(N_VARLEN, 512, 16384, seed=0))
        T = int(cu[-1])
        p = gi.prefill_inputs(T=T, seed=0, cu_seqlens=cu, with_state=name == "varlen")
        y = gdn.gdn_conv1d_silu(p["x_pre"].to(dev), p["conv_w"].to(dev), cu.to(dev))
        q, k, v = (y[:, :2048].view(T, 16, 128), y[:, 2048:4096].view(T, 16, 128),
                   y[:, 4096:].view(T, 48, 128))
        g, b, cud = p["g"].to(dev), p["beta"].to(dev), cu.to(dev)
        si = p["state_in"].to(dev) if p["state_in"] is not None else None
        o = torch.empty((T, 48, 128), dtype=torch.bfloat16, device=dev)
        S = torch.empty((cu.numel() - 1, 48, 128, 128), device=dev)
        run = lambda: gdn.gdn_chunked_prefill(q, k, v, g, b, cud, state_in=si, state_out=S, o=o)
    elif name == "dlayer":
        # the fused decode layer step on pools of N slots (identity slots)
        st = gi.decode_step_inputs(0, N, seed=0)
        state = gi.initial_states(0, N, tag="pstate").to(dev)
        cache = gi.to_bf16(gi.normal(0, "dconv", (N, 3, gi.CONV_CHANNELS))).to(dev)
        x, g, b, z = (st[k].to(dev) for k in ("x_pre", "g", "beta", "z"))
        w = gi.conv_weight(0).to(dev)
        nw = torch.ones(128, device=dev)
        idx = torch.arange(N, dtype=torch.int32, device=dev)
        yo = torch.empty((N, 48, 128), dtype=torch.bfloat16, device=dev)
        run = lambda: gdn.gdn_decode_layer_step(x, w, cache, g, b, state, idx, z, nw, y=yo)
    elif name == "layer":
        p = gi.prefill_inputs(T=T, seed=0)
        x, w, g, b, z, nw, cu = (p[k].to(dev) for k in ("x_pre", "conv_w", "g", "beta", "z",
                                                         "norm_w", "cu_seqlens"))
        S = torch.empty((1, 48, 128, 128), device=dev)
        yo = torch.empty((T, 48, 128), dtype=torch.bfloat16, device=dev)
        run = lambda: gdn.gdn_prefill_layer(x, w, g, b, cu, z, nw, state_out=S, y=yo)
    elif name == "conv":
        p = gi.prefill_inputs(T=T, seed=0)
        x, w, cu = p["x_pre"].to(dev), p["conv_w"].to(dev), p["cu_seqlens"].to(dev)
        y = torch.empty_like(x)
        run = lambda: gdn.gdn_conv1d_silu(x, w, cu, y=y)
    elif name == "norm":
        x = gi.gate_z(1, T, tag="px").to(dev)
        z = gi.gate_z(0, T).to(dev)
        w = torch.ones(128, device=dev)
        y = torch.empty_like(x)
        run = lambda: gdn.gdn_gated_rmsnorm(x, z, w, eps=1e-6, y=y)
    elif name == "dconv":
        cache = gi.to_bf16(gi.normal(0, "dconv", (N, 3, gi.CONV_CHANNELS))).to(dev)
        x = gi.decode_step_inputs(0, N, 0)["x_pre"].to(dev)
        w = gi.conv_weight(0).to(dev)
        cu = torch.arange(N + 1, dtype=torch.int32, device=dev)
        y = torch.empty((N, gi.CONV_CHANNELS), dtype=torch.bfloat16, device=dev)
        run = lambda: gdn.gdn_conv1d_silu(x, w, cu, conv_state_in=cache, conv_state_out=cache,
                                          y=y)
    elif name == "attn":
        wl = AttentionPrefillWorkload(gdn, dev, 0) if T == T_PREFILL else None
        if wl is None:
            raise SystemExit("attn case runs the T=8192 workload (--t 8192)")
        run = lambda: wl.step(0)
    elif name == "adec":
        # N sequences (--n) of 4096 cached tokens: 64 hold 1.1 GB of cache
        wl = AttentionDecodeWorkload(gdn, dev, 0, 1, n=N)
        run = lambda: (wl.reset(), wl.step(0))
    else:
        raise SystemExit(f"unknown profile case {name}")
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(args.launches):
        run()
    e.record()
    torch.cuda.synchronize()
    print(f"{name}: {s.elapsed_time(e) / args.launches:.4f} ms per launch")


PROFILE_CASES = ("decode", "dlayer", "prefill", "layer", "varlen", "conv", "norm", "dconv",
                 "attn", "adec")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="gdn", choices=["gdn", "reference"])
    ap.add_argument("--shard", default="replicas", choices=["replicas", "heads"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget-s", type=float, default=20.0)
    ap.add_argument("--profile-case", choices=PROFILE_CASES)
    ap.add_argument("--n", type=int, default=64)
    ap.add_argument("--t", type=int, default=8192)
    ap.add_argument("--launches", type=int, default=4)
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.profile_case:
        profile_case(args)
    elif args.impl == "reference":
        reference_arm(args)
    else:
        gpu_arm(args)


if __name__ == "__main__":
    main()
