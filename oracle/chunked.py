"""Chunked (WY / UT-transform) form of the gated delta rule, numpy fp64.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``). This is not the oracle
of record -- :func:`oracle.recurrence` is. It restates the chunk-64 prefill
form that the "Agnes-3.0-Flash Preview" leaderboard commentary (section 二.1,
``delta_rule_chunked``, chunk = 64) names beside the stepwise decode form, so
that tests can check that chunking reaches the stepwise result, and so that
the precision of each tensor-core operand can be budgeted by rounding it
(``round_ops``) exactly where a kernel would.

Derivation (per sequence, value head, and chunk of L <= C tokens; rows are
tokens; S0 is the state entering the chunk, [d_v, d_k]):

    G_t   = sum_{s<=t} log g_s          gamma_t = exp(G_t)
    A_tj  = beta_t exp(G_t - G_j) (k_t . k_j)          j < t, else 0
    T     = (I + A)^{-1}
    W     = T diag(beta gamma) K        U~ = T diag(beta) V
    Delta = U~ - W S0^T                 (row t = beta_t (v_t - g_t S_{t-1} k_t))
    M_tj  = exp(G_t - G_j) (q_t . k_j)                 j <= t, else 0
    O     = scale (diag(gamma) Q S0^T + M Delta)
    S_L   = gamma_L S0 + Delta^T diag(exp(G_L - G)) K

Only differences G_t - G_j with t >= j (all <= 0) are exponentiated, so no
factor above 1 is ever formed.
"""
from __future__ import annotations

import numpy as np
import scipy.linalg


def round_bf16(a):
    """Round to bfloat16 (nearest, ties to even), returned as float64."""
    f = np.asarray(a, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000).astype(np.uint32)
    return r.view(np.float32).astype(np.float64)


def round_fp16(a):
    """Round to IEEE binary16 (nearest even, with subnormals), as float64."""
    return np.asarray(a, dtype=np.float64).astype(np.float16).astype(np.float64)


def round_tf32(a):
    """Round to TF32 (10 stored mantissa bits, nearest even), as float64."""
    f = np.asarray(a, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    r = ((u + 0xFFF + ((u >> 13) & 1)) & 0xFFFFE000).astype(np.uint32)
    return r.view(np.float32).astype(np.float64)


ROUNDERS = {"bf16": round_bf16, "fp16": round_fp16, "tf32": round_tf32,
            None: None}


def _rounder(round_ops, name):
    if not round_ops:
        return lambda a: a
    fn = round_ops.get(name)
    if isinstance(fn, str) or fn is None:
        fn = ROUNDERS[fn]
    return fn if fn is not None else (lambda a: a)


def chunk_step(Q, K, V, g, beta, S0, scale=1.0, round_ops=None):
    """One chunk. Q, K [L, d_k]; V [L, d_v]; g, beta [L]; S0 [d_v, d_k].

    ``round_ops`` maps operand names to a rounding ("bf16", "fp16", "tf32"
    or a callable) applied where that operand would enter a tensor-core
    product: "T" (T diag(beta gamma) and T diag(beta)), "W", "S" (state as
    an operand), "D" (Delta), "Dk" (Delta scaled by exp(G_L - G)), "M",
    "Qg" (diag(gamma) Q). Returns (O [L, d_v], S_L [d_v, d_k]).
    """
    r = lambda n: _rounder(round_ops, n)
    L = Q.shape[0]
    G = np.cumsum(np.log(g))
    gamma = np.exp(G)
    diffG = G[:, None] - G[None, :]
    lower = np.tril(np.ones((L, L), dtype=bool), -1)
    lower_incl = np.tril(np.ones((L, L), dtype=bool), 0)
    decay = np.where(lower_incl, np.exp(np.where(lower_incl, diffG, 0.0)), 0.0)
    A = np.where(lower, beta[:, None] * decay * (K @ K.T), 0.0)
    Tm = scipy.linalg.solve_triangular(np.eye(L) + A, np.eye(L), lower=True,
                                       unit_diagonal=True)
    W = r("T")(Tm * (beta * gamma)[None, :]) @ K
    U = r("T")(Tm * beta[None, :]) @ V
    Delta = U - r("W")(W) @ r("S")(S0).T
    M = np.where(lower_incl, decay * (Q @ K.T), 0.0)
    O = scale * (r("Qg")(gamma[:, None] * Q) @ r("S")(S0).T
                 + r("M")(M) @ r("D")(Delta))
    tail = np.exp(G[-1] - G)
    S_L = gamma[-1] * S0 + r("Dk")(tail[:, None] * Delta).T @ K
    return O, S_L


def chunked(q, k, v, g, beta, state_in=None, cu_seqlens=None, scale=1.0,
            chunk=64, round_ops=None):
    """Chunked gated delta rule over packed sequences (same layouts and
    results as :func:`oracle.recurrence`). Chunks start at each sequence's
    first token; the last chunk of a sequence may be partial."""
    q, k, v, g, beta = (np.asarray(a, dtype=np.float64)
                        for a in (q, k, v, g, beta))
    T, H_k, d_k = q.shape
    H_v, d_v = v.shape[1], v.shape[2]
    group = H_v // H_k
    cu = np.asarray([0, T] if cu_seqlens is None else cu_seqlens,
                    dtype=np.int64)
    N = len(cu) - 1
    o = np.zeros((T, H_v, d_v))
    so = np.zeros((N, H_v, d_v, d_k))
    for n in range(N):
        for h in range(H_v):
            kh = h // group
            S = (np.zeros((d_v, d_k)) if state_in is None
                 else np.array(state_in[n, h], dtype=np.float64))
            for c0 in range(int(cu[n]), int(cu[n + 1]), chunk):
                c1 = min(c0 + chunk, int(cu[n + 1]))
                O, S = chunk_step(q[c0:c1, kh], k[c0:c1, kh], v[c0:c1, h],
                                  g[c0:c1, h], beta[c0:c1, h], S, scale,
                                  round_ops)
                o[c0:c1, h] = O
            so[n, h] = S
    return o, so
