"""Seeded synthetic inputs for the gated delta-rule layer.

This module is the one piece shared by the CUDA-path tests/bench and the CPU
oracle. It draws random numbers and rounds them to the storage dtype; it holds
none of the layer's arithmetic (no conv, no recurrence, no norm).

Shapes follow the Agnes-3.0-Flash Preview model card (section 架构) and the
leaderboard commentary (section 二.1): 16 key heads, 48 value heads, head dim
128, kernel-4 causal conv over the q|k|v projection channels
(2048 + 2048 + 6144 = 10240). Distributions:

* pre-conv activations x ~ N(0, 1); conv weights ~ N(0, 1/4) (std 0.5);
* beta = sigmoid(N(0,1)); g = exp(-softplus(N(0,1))) per token and value head;
* output gate z ~ N(0, 1); gated RMS-norm weight = ones;
* initial recurrent states ~ N(0, 0.02) (variance 0.02);
* packed varlen lengths: integers uniform in [512, 16384].

The global-attention layer of the same decoder (model card, section 架构,
rows 全局注意力 and 位置编码): 24 query / 4 key-value heads, head dim 256.
Its projections q, k, v and the output gate are drawn N(0, 1) and stored
bf16; the q/k RMS-norm weights are 1 + N(0, 0.1^2).

Every generator is a numpy PCG64 stream keyed by (seed, tag), so any part can
be regenerated alone. bf16 rounding uses torch's CPU cast (round to nearest
even); the oracle is always handed the rounded values.
"""
from __future__ import annotations

import zlib

import numpy as np
import torch

H_K = 16
H_V = 48
D = 128
CONV_K = 4
Q_CHANNELS = H_K * D                 # 2048
K_CHANNELS = H_K * D                 # 2048
V_CHANNELS = H_V * D                 # 6144
CONV_CHANNELS = Q_CHANNELS + K_CHANNELS + V_CHANNELS   # 10240
L2_CHANNELS = Q_CHANNELS + K_CHANNELS                  # 4096
STATE_VAR = 0.02
CONV_W_VAR = 0.25


def rng(seed: int, *tag) -> np.random.Generator:
    """Independent PCG64 stream for (seed, tag...)."""
    key = [int(seed) & 0xFFFFFFFF]
    for t in tag:
        key.append(zlib.crc32(str(t).encode()) if not isinstance(t, int)
                   else int(t) & 0xFFFFFFFF)
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(key)))


def normal(seed, tag, shape, std=1.0) -> np.ndarray:
    """float32 N(0, std^2) array."""
    a = rng(seed, tag).standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        a *= np.float32(std)
    return a


def to_bf16(a) -> torch.Tensor:
    """Round (nearest even) to a CPU bfloat16 tensor."""
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(
        torch.bfloat16)


def as_f64(t) -> np.ndarray:
    """Exact float64 copy of a (CPU or CUDA) tensor or array."""
    if isinstance(t, torch.Tensor):
        return t.detach().to("cpu", torch.float64).numpy()
    return np.asarray(t, dtype=np.float64)


def gates(seed, T, H_v=H_V, dtype=torch.float32, tag="gates"):
    """(g, beta) [T, H_v]: beta = sigmoid(N(0,1)), g = exp(-softplus(N(0,1))),
    drawn in float64 then rounded to ``dtype``."""
    r = rng(seed, tag)
    nb = r.standard_normal((T, H_v))
    ng = r.standard_normal((T, H_v))
    beta = 1.0 / (1.0 + np.exp(-nb))
    g = np.exp(-np.logaddexp(0.0, ng))
    return (torch.from_numpy(g).to(dtype), torch.from_numpy(beta).to(dtype))


def unit_heads(seed, tag, T, H, d=D) -> np.ndarray:
    """float32 [T, H, d] vectors uniform on the unit sphere (a Gaussian draw
    divided by its length)."""
    a = rng(seed, tag).standard_normal((T, H, d))
    a /= np.linalg.norm(a, axis=-1, keepdims=True)
    return a.astype(np.float32)


def recurrence_inputs(T=256, seed=0, H_k=H_K, H_v=H_V, d=D):
    """Small fp32 recurrence case: q, k unit vectors per head, v ~ N(0,1),
    beta/g as :func:`gates`, zero initial state. CPU float32 tensors."""
    q = torch.from_numpy(unit_heads(seed, "q", T, H_k, d))
    k = torch.from_numpy(unit_heads(seed, "k", T, H_k, d))
    v = torch.from_numpy(normal(seed, "v", (T, H_v, d)))
    g, beta = gates(seed, T, H_v)
    return dict(q=q, k=k, v=v, g=g, beta=beta,
                cu_seqlens=torch.tensor([0, T], dtype=torch.int32))


def varlen_cu_seqlens(n_seqs=16, lo=512, hi=16384, seed=0) -> torch.Tensor:
    """cu_seqlens [n+1] int32 for lengths uniform in [lo, hi] (inclusive)."""
    lens = rng(seed, "varlen").integers(lo, hi + 1, size=n_seqs)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    return torch.from_numpy(cu)


def conv_weight(seed=0, channels=CONV_CHANNELS) -> torch.Tensor:
    """[channels, 4] float32 ~ N(0, 1/4); tap 3 multiplies the current token."""
    return torch.from_numpy(normal(seed, "conv_w", (channels, CONV_K),
                                   std=CONV_W_VAR ** 0.5))


def pre_conv(seed, T, tag="x", channels=CONV_CHANNELS) -> torch.Tensor:
    """[T, channels] bf16 pre-conv activations ~ N(0, 1)."""
    return to_bf16(normal(seed, tag, (T, channels)))


def initial_states(seed, N, H_v=H_V, d=D, tag="state") -> torch.Tensor:
    """[N, H_v, d_v, d_k] float32 ~ N(0, 0.02)."""
    return torch.from_numpy(normal(seed, tag, (N, H_v, d, d),
                                   std=STATE_VAR ** 0.5))


def gate_z(seed, T, H_v=H_V, d=D, tag="z") -> torch.Tensor:
    """[T, H_v, d] bf16 output gate ~ N(0, 1)."""
    return to_bf16(normal(seed, tag, (T, H_v, d)))


def prefill_inputs(T=8192, seed=0, cu_seqlens=None, with_state=False,
                   gate_dtype=torch.float32, tag=""):
    """Prefill layer inputs (CPU tensors): x_pre bf16 [T,10240], conv_w fp32
    [10240,4], g/beta [T,48] (gate_dtype), z bf16 [T,48,128], norm_w fp32
    [128] ones, cu_seqlens int32, state_in fp32 [N,48,128,128] or None."""
    if cu_seqlens is None:
        cu_seqlens = torch.tensor([0, T], dtype=torch.int32)
    N = cu_seqlens.numel() - 1
    g, beta = gates(seed, T, dtype=gate_dtype, tag=f"gates{tag}")
    return dict(
        x_pre=pre_conv(seed, T, tag=f"x{tag}"),
        conv_w=conv_weight(seed),
        g=g, beta=beta,
        z=gate_z(seed, T, tag=f"z{tag}"),
        norm_w=torch.ones(D, dtype=torch.float32),
        cu_seqlens=cu_seqlens,
        state_in=initial_states(seed, N) if with_state else None,
    )


def decode_step_inputs(step, N=256, seed=0):
    """Per-step decode inputs (CPU tensors, all bf16): x_pre [N,10240],
    g/beta [N,48], z [N,48,128]."""
    g, beta = gates(seed, N, dtype=torch.bfloat16, tag=f"dgates{step}")
    return dict(x_pre=pre_conv(seed, N, tag=f"dx{step}"), g=g, beta=beta,
                z=gate_z(seed, N, tag=f"dz{step}"))


def decode_initial(N=256, seed=0):
    """Decode start: fp32 state [N,48,128,128] ~ N(0,0.02) and a bf16
    pre-conv cache [N,3,10240] ~ N(0,1) (the 3 prior tokens, oldest first)."""
    return dict(state=initial_states(seed, N, tag="dstate"),
                conv_state=to_bf16(normal(seed, "dconv", (N, 3, CONV_CHANNELS))))


ATTN_H_Q, ATTN_H_KV, ATTN_D = 24, 4, 256


def attention_inputs(T, seed=0, H_q=ATTN_H_Q, H_kv=ATTN_H_KV, d=ATTN_D, tag="attn"):
    """q, gate [T, H_q, d]; k, v [T, H_kv, d] (bf16, N(0,1)); q_norm_w, k_norm_w
    [d] (bf16, 1 + N(0, 0.01))."""
    out = {}
    for name, H in (("q", H_q), ("k", H_kv), ("v", H_kv), ("gate", H_q)):
        out[name] = to_bf16(normal(seed, (tag, name), (T, H, d)))
    for name in ("q_norm_w", "k_norm_w"):
        out[name] = to_bf16(1.0 + normal(seed, (tag, name), (d,), std=0.1))
    return out

