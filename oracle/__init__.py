"""fp64 CPU oracle of the gated delta-rule layer.

TEST INFRASTRUCTURE ONLY: the test suite, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` are the only callers. The CUDA library never
imports, links or runs anything here, and nothing here imports the CUDA
package. The two share only the seeded input generators (``gdn_inputs``),
which hold none of the layer's arithmetic.

Functions (sources: "Agnes-3.0-Flash Preview" leaderboard commentary,
section 二.1, and the Agnes-3.0-Flash Preview model card, section 架构):

* :func:`conv1d_silu_l2` -- kernel-4 causal depthwise conv, SiLU, per-head L2
  normalisation of the q/k channels, conv-history carry.
* :func:`recurrence` -- the stepwise gated delta rule
  ``S_t = g_t S_{t-1}(I - b_t k_t k_t^T) + b_t v_t k_t^T``, ``o_t = scale S_t q_t``.
* :func:`gated_rmsnorm` -- ``x / sqrt(mean x^2 + eps) * w * SiLU(z)``.
* :func:`attention` -- the hybrid decoder's global-attention layer (model card,
  架构 table; commentary section 二.1): q/k RMS-norm, rotary on the first 64
  dims, causal GQA softmax attention, sigmoid output gate.
* :mod:`oracle.chunked` -- the chunk-64 (WY / UT-transform) form of the same
  recurrence in numpy fp64, with optional operand-rounding emulation; a
  test-only cross-check, not the oracle of record.

The arithmetic lives in ``gdn_oracle.cpp`` (plain C++17, fp64); this module
only marshals numpy arrays. Each function's pins are in
``tests/test_oracle_*.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn_oracle.cpp")
_LIB_PATH = os.path.join(_HERE, "liboracle_gdn.so")
# Tests that plant a mistake in the oracle point this at a mutant build.
_LIB_OVERRIDE = os.environ.get("GDN_ORACLE_LIB")
_lib = None
_lock = threading.Lock()

_dp = ctypes.POINTER(ctypes.c_double)
_ip = ctypes.POINTER(ctypes.c_int32)


def build(force: bool = False) -> str:
    """Compile ``gdn_oracle.cpp`` into ``liboracle_gdn.so`` (generic x86-64)."""
    if force or not os.path.exists(_LIB_PATH) or (
        os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)
    ):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["g++", "-O2", "-std=c++17", "-fPIC", "-shared", "-pthread",
               _SRC, "-o", tmp]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if _LIB_OVERRIDE:
            lib = ctypes.CDLL(_LIB_OVERRIDE)
        else:
            build()
            lib = ctypes.CDLL(_LIB_PATH)
        lib.oracle_hardware_threads.restype = ctypes.c_int
        lib.oracle_conv1d_silu_l2.restype = None
        lib.oracle_conv1d_silu_l2.argtypes = [
            _dp, ctypes.c_int64, ctypes.c_int, _dp, _dp, _ip, ctypes.c_int, _dp,
            ctypes.c_int, ctypes.c_double, _dp, _dp, ctypes.c_int]
        lib.oracle_recurrence.restype = None
        lib.oracle_recurrence.argtypes = [
            _dp, _dp, _dp, _dp, _dp, _dp, _ip, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, ctypes.c_int, ctypes.c_double, _dp, _dp, ctypes.c_int]
        lib.oracle_attention.restype = None
        lib.oracle_attention.argtypes = [
            _dp, _dp, _dp, _dp, _ip, ctypes.POINTER(ctypes.c_int64),
            ctypes.POINTER(ctypes.c_int64), ctypes.c_int,
            ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int, _dp, _dp,
            ctypes.c_double, ctypes.c_int, ctypes.c_double, ctypes.c_double,
            ctypes.POINTER(ctypes.c_uint8), _dp, _dp, _dp, ctypes.c_int]
        lib.oracle_gated_rmsnorm.restype = None
        lib.oracle_gated_rmsnorm.argtypes = [
            _dp, _dp, _dp, ctypes.c_int64, ctypes.c_int, ctypes.c_double, _dp,
            ctypes.c_int]
        _lib = lib
        return lib


def hardware_threads() -> int:
    return int(_load().oracle_hardware_threads())


def _f64(a):
    if a is None:
        return None
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(_dp)


def _cu(cu_seqlens, T):
    if cu_seqlens is None:
        cu_seqlens = [0, T]
    cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int32))
    if cu.ndim != 1 or cu[0] != 0 or cu[-1] != T or np.any(np.diff(cu) < 0):
        raise ValueError("cu_seqlens must start at 0, end at T and not decrease")
    return cu


def conv1d_silu_l2(x, w, bias=None, cu_seqlens=None, conv_state_in=None,
                   l2_channels=0, l2_eps=1e-6, threads=0):
    """Causal kernel-4 conv + SiLU + per-128-channel L2 norm (fp64).

    x [T, C]; w [C, 4] (tap 3 = current token); bias [C] or None;
    conv_state_in [N, 3, C] or None (zeros). Returns (y [T, C],
    conv_state_out [N, 3, C]).
    """
    x = _f64(x)
    T, C = x.shape
    w = _f64(w).reshape(C, 4)
    bias = _f64(bias)
    cu = _cu(cu_seqlens, T)
    N = len(cu) - 1
    csi = _f64(conv_state_in)
    if csi is not None:
        csi = csi.reshape(N, 3, C)
    if l2_channels % 128 or l2_channels > C:
        raise ValueError("l2_channels must be a multiple of 128 within C")
    y = np.zeros((T, C))
    cso = np.zeros((N, 3, C))
    _load().oracle_conv1d_silu_l2(
        _ptr(x), T, C, _ptr(w), _ptr(bias), cu.ctypes.data_as(_ip), N,
        _ptr(csi), l2_channels, float(l2_eps), _ptr(y), _ptr(cso), int(threads))
    return y, cso


def recurrence(q, k, v, g, beta, state_in=None, cu_seqlens=None, scale=1.0,
               threads=0):
    """Stepwise gated delta rule (fp64).

    q, k [T, H_k, d]; v [T, H_v, d]; g, beta [T, H_v]; state_in
    [N, H_v, d, d] ([d_v, d_k] per head) or None. Returns (o [T, H_v, d],
    state_out [N, H_v, d, d]).
    """
    q, k, v, g, beta = (_f64(a) for a in (q, k, v, g, beta))
    T, H_k, d = q.shape
    H_v = v.shape[1]
    if k.shape != q.shape or v.shape != (T, H_v, d) or g.shape != (T, H_v) \
            or beta.shape != (T, H_v) or H_v % H_k:
        raise ValueError("inconsistent shapes")
    cu = _cu(cu_seqlens, T)
    N = len(cu) - 1
    si = _f64(state_in)
    if si is not None:
        si = si.reshape(N, H_v, d, d)
    o = np.zeros((T, H_v, d))
    so = np.zeros((N, H_v, d, d))
    _load().oracle_recurrence(
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(si),
        cu.ctypes.data_as(_ip), N, H_k, H_v, d, float(scale), _ptr(o), _ptr(so),
        int(threads))
    return o, so


def gated_rmsnorm(x, z, w, eps=1e-6, threads=0):
    """Gated RMS-norm over the last axis (fp64): x/rms(x) * w * SiLU(z)."""
    x = _f64(x)
    shape = x.shape
    dim = shape[-1]
    x2 = x.reshape(-1, dim)
    z2 = _f64(z).reshape(-1, dim)
    w = _f64(w).reshape(dim)
    y = np.zeros_like(x2)
    _load().oracle_gated_rmsnorm(_ptr(x2), _ptr(z2), _ptr(w), x2.shape[0], dim,
                                 float(eps), _ptr(y), int(threads))
    return y.reshape(shape)


def attention(q, k, v, gate, wq, wk, cu_seqlens=None, pos0=None, positions=None,
              eps=1e-6, rope_dims=64, rope_base=1e7, scale=None, rows=None, threads=0):
    """Global-attention layer (fp64): per token and head, q and k RMS-normed
    over the head dim with weights wq / wk, rotary (rotate-half pairs
    (i, i + R/2), theta = p * base^(-2i/R)) on the first ``rope_dims`` dims,
    causal softmax attention with query head h reading kv head h // (Hq/Hkv),
    output times sigmoid(gate).

    Pair i turns by the token's position on axis i % 3 (text, height, width):
    ``positions`` [3, T] gives them; without it every axis carries the token's
    index within its sequence plus ``pos0[n]`` (0 without pos0).

    q, gate [T, Hq, D]; k, v [T, Hkv, D]; wq, wk [D]; pos0 [N] or None.
    Returns (out [T, Hq, D], q_rot [T, Hq, D], k_rot [T, Hkv, D]); scale
    defaults to D**-0.5. ``rows`` (token indices) limits the output rows that
    are computed; the others are returned as zeros."""
    q, k, v, gate, wq, wk = (_f64(a) for a in (q, k, v, gate, wq, wk))
    T, Hq, D = q.shape
    Hkv = k.shape[1]
    if k.shape != (T, Hkv, D) or v.shape != (T, Hkv, D) or gate.shape != q.shape \
            or Hq % Hkv or wq.shape != (D,) or wk.shape != (D,) or rope_dims % 2 \
            or rope_dims > D:
        raise ValueError("inconsistent shapes")
    cu = _cu(cu_seqlens, T)
    N = len(cu) - 1
    p0 = None
    if pos0 is not None:
        p0 = np.ascontiguousarray(np.asarray(pos0, dtype=np.int64))
    p3 = None
    if positions is not None:
        p3 = np.ascontiguousarray(np.asarray(positions, dtype=np.int64))
        if p3.shape != (3, T):
            raise ValueError("positions must be [3, T]")
    out = np.zeros_like(q)
    qr = np.zeros_like(q)
    kr = np.zeros_like(k)
    i64 = ctypes.POINTER(ctypes.c_int64)
    want = None
    if rows is not None:
        want = np.zeros(T, dtype=np.uint8)
        want[np.asarray(rows, dtype=np.int64)] = 1
    _load().oracle_attention(
        _ptr(q), _ptr(k), _ptr(v), _ptr(gate), cu.ctypes.data_as(_ip),
        None if p0 is None else p0.ctypes.data_as(i64),
        None if p3 is None else p3.ctypes.data_as(i64), N, T, Hq,
        Hkv, D, _ptr(wq), _ptr(wk), float(eps), int(rope_dims), float(rope_base),
        float(D ** -0.5 if scale is None else scale),
        None if want is None else want.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8)),
        _ptr(out), _ptr(qr), _ptr(kr),
        int(threads))
    return out, qr, kr
