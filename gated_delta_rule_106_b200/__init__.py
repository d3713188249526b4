"""gated_delta_rule_106_b200 -- B200-native gated delta-rule layer.

Thin ctypes binding over the C ABI of ``libgdn.so`` (declared in
``include/gdn.h``). Each function here has the name of its C entry point and
only marshals arguments: torch CUDA tensors supply device memory and the
current CUDA stream; every step of the computation runs in the library's
sm_100a kernels. There is no CPU or PyTorch fallback: if ``libgdn.so`` is
missing, or a tensor is not on a CUDA device, the call raises.

Sources of the layer: "Agnes-3.0-Flash Preview" leaderboard commentary,
section 二.1 (16 key / 48 value heads, head dim 128, kernel-4 causal conv,
fp32 state, chunked prefill with chunk 64 and stepwise decode) and the
Agnes-3.0-Flash Preview model card, 架构 table (gated RMS-norm).
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

__all__ = ["GDN_BF16", "GDN_F32", "GdnError", "library_path", "load",
           "gdn_conv1d_silu", "gdn_chunked_prefill",
           "gdn_chunked_prefill_workspace", "gdn_chunked_prefill_noalloc",
           "gdn_stepwise_prefill", "gdn_decode_layer_step", "gdn_prefill_layer",
           "gdn_chunked_prefill_status", "gdn_set_wait_limit_ns", "GDN_ERR_TIMEOUT",
           "gdn_prefill_layer_workspace",
           "gdn_decode_step",
           "gdn_gated_rmsnorm", "gdn_status_string", "gdn_version",
           "gdn_attention_prefill", "gdn_attention_decode", "gdn_attention_status",
           "ATTN_H_Q", "ATTN_H_KV", "ATTN_HEAD_DIM",
           "H_K", "H_V", "HEAD_DIM", "CHUNK"]

GDN_BF16 = 0
GDN_F32 = 1
GDN_ERR_TIMEOUT = -5
H_K, H_V, HEAD_DIM, CHUNK = 16, 48, 128, 64

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libgdn.so")
_lib = None
_lock = threading.Lock()

_vp = ctypes.c_void_p
_i64 = ctypes.c_int64
_int = ctypes.c_int
_f32 = ctypes.c_float

# name -> (restype, argtypes)
_SIGNATURES = {
    "gdn_attention_prefill_workspace": (ctypes.c_size_t, [_i64, _int, _int]),
    "gdn_attention_prefill": (_int, [_vp, _i64, _vp, _i64, _vp, _i64, _vp, _i64, _vp, _vp, _int,
                                     _vp, _vp, _vp, _int, _i64, _int, _int, _int, _f32, _int,
                                     _f32, _f32, _vp, _vp, _vp, _vp, ctypes.c_size_t, _vp]),
    "gdn_attention_decode_workspace": (ctypes.c_size_t, [_int, _int, _int, _int]),
    "gdn_attention_decode": (_int, [_vp, _i64, _vp, _i64, _vp, _i64, _vp, _i64, _vp, _vp, _int,
                                    _vp, _vp, _vp, _vp, _vp, _int, _int, _int, _int, _int, _int,
                                    _f32, _int, _f32, _f32, _vp, _vp, ctypes.c_size_t, _vp]),
    "gdn_attention_status": (_int, [_vp, _vp]),
    "gdn_status_string": (ctypes.c_char_p, [_int]),
    "gdn_version": (ctypes.c_char_p, []),
    "gdn_conv1d_silu": (_int, [_vp, _i64, _int, _vp, _int, _vp, _int, _int, _f32,
                               _vp, _int, _i64, _vp, _vp, _vp, _i64, _int, _vp]),
    "gdn_chunked_prefill": (_int, [_vp, _vp, _vp, _int, _i64, _i64, _i64, _vp,
                                   _vp, _int, _vp, _vp, _vp, _int, _i64, _int,
                                   _int, _f32, _vp, _int, _vp, ctypes.c_size_t,
                                   _vp]),
    "gdn_chunked_prefill_workspace": (ctypes.c_size_t, [_int, _i64, _int, _int]),
    "gdn_prefill_layer_workspace": (ctypes.c_size_t, [_int, _i64, _int, _int]),
    "gdn_chunked_prefill_status": (_int, [_vp, _vp]),
    "gdn_prefill_layer": (_int, [_vp, _i64, _vp, _int, _vp, _vp, _vp, _vp, _vp, _int, _vp,
                                 _vp, _vp, _int, _i64, _int, _int, _f32, _f32, _vp, _vp,
                                 _f32, _vp, _int, _vp, ctypes.c_size_t, _vp]),
    "gdn_set_wait_limit_ns": (None, [ctypes.c_uint64]),
    "gdn_stepwise_prefill": (_int, [_vp, _vp, _vp, _int, _i64, _i64, _i64, _vp,
                                    _vp, _int, _vp, _vp, _vp, _int, _i64, _int,
                                    _int, _f32, _vp, _int, _vp]),
    "gdn_chunked_prefill_noalloc": (_int, [_vp, _vp, _vp, _int, _i64, _i64, _i64, _vp,
                                           _vp, _int, _vp, _vp, _vp, _int, _i64, _int,
                                           _int, _f32, _vp, _int, _vp]),
    "gdn_chunked_prefill_noalloc_scratch_bytes": (ctypes.c_size_t, []),
    "gdn_decode_step": (_int, [_vp, _vp, _vp, _int, _i64, _i64, _i64, _vp, _vp,
                               _int, _vp, _int, _int, _int, _f32, _vp, _int,
                               _vp]),
    "gdn_decode_layer_step": (_int, [_vp, _i64, _int, _vp, _int, _vp, _vp, _vp, _vp, _int,
                                      _vp, _vp, _int, _int, _int, _int, _f32, _f32, _vp,
                                      _vp, _f32, _vp, _int, _vp]),
    "gdn_gated_rmsnorm": (_int, [_vp, _int, _vp, _int, _vp, _int, _i64, _int,
                                 _f32, _vp, _int, _vp]),
}


class GdnError(RuntimeError):
    """A libgdn entry point returned a non-zero gdn_status."""

    def __init__(self, fn, status):
        self.status = status
        super().__init__(f"{fn}: {gdn_status_string(status)} ({status})")


def library_path() -> str:
    return _LIB_PATH


def load():
    """Load libgdn.so (in-tree). Raises if it has not been built."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(_LIB_PATH):
                raise RuntimeError(
                    f"{_LIB_PATH} is missing: build it with "
                    "`python -m gated_delta_rule_106_b200._build` (nvcc, sm_100a)")
            lib = ctypes.CDLL(_LIB_PATH)
            for name, (res, args) in _SIGNATURES.items():
                fn = getattr(lib, name)
                fn.restype = res
                fn.argtypes = args
            _lib = lib
        return _lib


def gdn_status_string(status: int) -> str:
    return load().gdn_status_string(int(status)).decode()


def gdn_version() -> str:
    return load().gdn_version().decode()


def _dtype_code(t: torch.dtype) -> int:
    if t == torch.bfloat16:
        return GDN_BF16
    if t == torch.float32:
        return GDN_F32
    raise TypeError(f"unsupported dtype {t}; use torch.bfloat16 or torch.float32")


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libgdn takes CUDA tensors only (no CPU path)")
    return t.data_ptr()


def _row_stride(t):
    """Token-row stride (elements) of a tensor whose trailing dims are dense."""
    if t.dim() >= 2:
        inner = 1
        for size, stride in zip(reversed(t.shape[1:]), reversed(t.stride()[1:])):
            if size != 1 and stride != inner:
                raise ValueError("trailing dimensions must be contiguous")
            inner *= size
    return t.stride(0)


def _expect(t, shape, name, dtype=None, contiguous=True):
    """Shape (and dtype, contiguity) the C ABI assumes for a tensor argument;
    checked before any pointer is taken, since the kernels write dense layouts."""
    if t is None:
        return
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name}: dtype {t.dtype}, expected {dtype}")
    if contiguous and not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _stream(stream, device):
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return stream.cuda_stream if isinstance(stream, torch.cuda.Stream) else int(stream)


def _check(fn, status):
    if status != 0:
        raise GdnError(fn, status)


def gdn_conv1d_silu(x, w, cu_seqlens, *, bias=None, conv_state_in=None,
                    conv_state_out=None, l2norm_channels=2 * H_K * HEAD_DIM,
                    l2_eps=1e-6, y=None, y_dtype=None, stream=None):
    """Causal kernel-4 conv + SiLU + per-head L2 norm of the leading
    ``l2norm_channels`` channels. x [T, C]; w [C, 4]; cu_seqlens int32 [N+1];
    conv states [N, 3, C] (x's dtype). Returns y [T, C]."""
    T, C = x.shape
    N = cu_seqlens.numel() - 1
    _expect(cu_seqlens, (N + 1,), "cu_seqlens", torch.int32)
    _expect(w, (C, 4), "w")
    _expect(bias, (C,), "bias", w.dtype)
    _expect(conv_state_in, (N, 3, C), "conv_state_in", x.dtype)
    _expect(conv_state_out, (N, 3, C), "conv_state_out", x.dtype)
    _expect(y, (T, C), "y", contiguous=False)
    if y is None:
        y = torch.empty((T, C), dtype=y_dtype or x.dtype, device=x.device)
    _check("gdn_conv1d_silu", load().gdn_conv1d_silu(
        _ptr(x), _row_stride(x), _dtype_code(x.dtype), _ptr(w),
        _dtype_code(w.dtype), _ptr(bias), C, l2norm_channels, l2_eps,
        _ptr(cu_seqlens), N, T, _ptr(conv_state_in), _ptr(conv_state_out),
        _ptr(y), _row_stride(y), _dtype_code(y.dtype), _stream(stream, x.device)))
    return y


def _check_prefill_shapes(q, k, v, g, beta, cu_seqlens, state_in, state_out, o, T,
                          H_k, H_v, N):
    # one qkv dtype crosses the C ABI (q's): k and v must share it
    _expect(q, (T, H_k, HEAD_DIM), "q", contiguous=False)
    _expect(k, (T, H_k, HEAD_DIM), "k", q.dtype, contiguous=False)
    _expect(v, (T, H_v, HEAD_DIM), "v", q.dtype, contiguous=False)
    _expect(cu_seqlens, (N + 1,), "cu_seqlens", torch.int32)
    _expect(g, (T, H_v), "g")
    _expect(beta, (T, H_v), "beta", g.dtype)
    _expect(state_in, (N, H_v, HEAD_DIM, HEAD_DIM), "state_in", torch.float32)
    _expect(state_out, (N, H_v, HEAD_DIM, HEAD_DIM), "state_out", torch.float32)
    _expect(o, (T, H_v, HEAD_DIM), "o")


def gdn_chunked_prefill_workspace(N, T_total, H_k=H_K, H_v=H_V) -> int:
    return int(load().gdn_chunked_prefill_workspace(N, T_total, H_k, H_v))


def gdn_chunked_prefill(q, k, v, g, beta, cu_seqlens, *, state_in=None,
                        state_out=None, scale=1.0, o=None, o_dtype=None,
                        workspace=None, stream=None):
    """Chunked (C=64) gated delta rule over packed sequences.
    q, k [T, H_k, 128] (views with any token stride); v [T, H_v, 128];
    g, beta [T, H_v]; states fp32 [N, H_v, 128, 128]. Returns o [T, H_v, 128]."""
    T, H_k, _ = q.shape
    H_v = v.shape[1]
    N = cu_seqlens.numel() - 1
    _check_prefill_shapes(q, k, v, g, beta, cu_seqlens, state_in, state_out, o, T,
                          H_k, H_v, N)
    if o is None:
        o = torch.empty((T, H_v, HEAD_DIM), dtype=o_dtype or v.dtype, device=v.device)
    # only the tensor-core path (bf16 inputs) works in a workspace
    need = gdn_chunked_prefill_workspace(N, T, H_k, H_v) if q.dtype == torch.bfloat16 else 0
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=v.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check("gdn_chunked_prefill", load().gdn_chunked_prefill(
        _ptr(q), _ptr(k), _ptr(v), _dtype_code(q.dtype), _row_stride(q),
        _row_stride(k), _row_stride(v), _ptr(g), _ptr(beta), _dtype_code(g.dtype),
        _ptr(state_in), _ptr(state_out), _ptr(cu_seqlens), N, T, H_k, H_v,
        scale, _ptr(o), _dtype_code(o.dtype), _ptr(workspace), ws_bytes,
        _stream(stream, v.device)))
    return o


def gdn_prefill_layer(x, conv_w, g, beta, cu_seqlens, z, norm_w, *, conv_bias=None,
                      conv_state_in=None, conv_state_out=None, state_in=None,
                      state_out=None, scale=1.0, l2_eps=1e-6, norm_eps=1e-6, y=None,
                      y_dtype=None, H_k=H_K, workspace=None, stream=None):
    """The whole prefill of the layer in one kernel: conv + SiLU + q/k L2 from the
    pre-conv x [T, C] (bf16, C = 2*H_k*128 + H_v*128), the chunked gated delta
    rule, and the gated RMS-norm with gate z [T, H_v, 128] (bf16) and weight
    norm_w [128] (conv_w's dtype). Returns the normed output y [T, H_v, 128]."""
    T, C = x.shape
    H_v = g.shape[1]
    N = cu_seqlens.numel() - 1
    if x.dtype != torch.bfloat16:
        raise ValueError("x must be bf16")
    if C != (2 * H_k + H_v) * HEAD_DIM:
        raise ValueError(f"x: {C} channels, expected {(2 * H_k + H_v) * HEAD_DIM}")
    _expect(conv_w, (C, 4), "conv_w")
    _expect(conv_bias, (C,), "conv_bias", conv_w.dtype)
    _expect(conv_state_in, (N, 3, C), "conv_state_in", torch.bfloat16)
    _expect(conv_state_out, (N, 3, C), "conv_state_out", torch.bfloat16)
    _expect(cu_seqlens, (N + 1,), "cu_seqlens", torch.int32)
    _expect(g, (T, H_v), "g")
    _expect(beta, (T, H_v), "beta", g.dtype)
    _expect(state_in, (N, H_v, HEAD_DIM, HEAD_DIM), "state_in", torch.float32)
    _expect(state_out, (N, H_v, HEAD_DIM, HEAD_DIM), "state_out", torch.float32)
    _expect(z, (T, H_v, HEAD_DIM), "z", torch.bfloat16)
    _expect(norm_w, (HEAD_DIM,), "norm_w", conv_w.dtype)
    _expect(y, (T, H_v, HEAD_DIM), "y")
    if y is None:
        y = torch.empty((T, H_v, HEAD_DIM), dtype=y_dtype or torch.bfloat16, device=x.device)
    need = gdn_prefill_layer_workspace(N, T, H_k, H_v)
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check("gdn_prefill_layer", load().gdn_prefill_layer(
        _ptr(x), _row_stride(x), _ptr(conv_w), _dtype_code(conv_w.dtype), _ptr(conv_bias),
        _ptr(conv_state_in), _ptr(conv_state_out), _ptr(g), _ptr(beta), _dtype_code(g.dtype),
        _ptr(state_in), _ptr(state_out), _ptr(cu_seqlens), N, T, H_k, H_v, scale, l2_eps,
        _ptr(z), _ptr(norm_w), norm_eps, _ptr(y), _dtype_code(y.dtype), _ptr(workspace),
        ws_bytes, _stream(stream, x.device)))
    return y


def gdn_prefill_layer_workspace(N, T_total, H_k=H_K, H_v=H_V) -> int:
    """Bytes of workspace gdn_prefill_layer needs (chunk ring + q/k conv scratch)."""
    return int(load().gdn_prefill_layer_workspace(N, T_total, H_k, H_v))


def gdn_chunked_prefill_status(workspace=None, stream=None) -> int:
    """Waits for `stream`, then returns 0 if the last gdn_chunked_prefill that
    worked in `workspace` (None: the no-alloc call's own array) completed, or
    GDN_ERR_TIMEOUT if a bounded wait inside it gave up (its unfinished outputs
    are NaN). Not for the hot path: it synchronises."""
    dev = workspace.device if workspace is not None else torch.device("cuda")
    return int(load().gdn_chunked_prefill_status(_ptr(workspace), _stream(stream, dev)))


def gdn_set_wait_limit_ns(ns: int) -> None:
    """Bound (ns) on each wait of the chunked prefill kernel for another CTA's
    flag; 0 restores the default (2 s). Process-wide."""
    load().gdn_set_wait_limit_ns(int(ns))


def gdn_stepwise_prefill(q, k, v, g, beta, cu_seqlens, *, state_in=None,
                         state_out=None, scale=1.0, o=None, o_dtype=None,
                         stream=None):
    """The same recurrence as gdn_chunked_prefill advanced token by token (the
    stepwise path), fp32 on the CUDA cores. Same arguments, no workspace."""
    T, H_k, _ = q.shape
    H_v = v.shape[1]
    N = cu_seqlens.numel() - 1
    _check_prefill_shapes(q, k, v, g, beta, cu_seqlens, state_in, state_out, o, T,
                          H_k, H_v, N)
    if o is None:
        o = torch.empty((T, H_v, HEAD_DIM), dtype=o_dtype or v.dtype, device=v.device)
    _check("gdn_stepwise_prefill", load().gdn_stepwise_prefill(
        _ptr(q), _ptr(k), _ptr(v), _dtype_code(q.dtype), _row_stride(q),
        _row_stride(k), _row_stride(v), _ptr(g), _ptr(beta), _dtype_code(g.dtype),
        _ptr(state_in), _ptr(state_out), _ptr(cu_seqlens), N, T, H_k, H_v,
        scale, _ptr(o), _dtype_code(o.dtype), _stream(stream, v.device)))
    return o


def gdn_chunked_prefill_noalloc(q, k, v, g, beta, cu_seqlens, *, state_in=None,
                                state_out=None, scale=1.0, o=None, o_dtype=None,
                                stream=None):
    """gdn_chunked_prefill working in the library's own static device scratch
    instead of a caller-provided workspace (for callers that cannot allocate
    at the call site). Calls that overlap on the GPU must not share it."""
    T, H_k, _ = q.shape
    H_v = v.shape[1]
    N = cu_seqlens.numel() - 1
    _check_prefill_shapes(q, k, v, g, beta, cu_seqlens, state_in, state_out, o, T,
                          H_k, H_v, N)
    if o is None:
        o = torch.empty((T, H_v, HEAD_DIM), dtype=o_dtype or v.dtype, device=v.device)
    _check("gdn_chunked_prefill_noalloc", load().gdn_chunked_prefill_noalloc(
        _ptr(q), _ptr(k), _ptr(v), _dtype_code(q.dtype), _row_stride(q),
        _row_stride(k), _row_stride(v), _ptr(g), _ptr(beta), _dtype_code(g.dtype),
        _ptr(state_in), _ptr(state_out), _ptr(cu_seqlens), N, T, H_k, H_v,
        scale, _ptr(o), _dtype_code(o.dtype), _stream(stream, v.device)))
    return o


def gdn_decode_step(q, k, v, g, beta, state, *, scale=1.0, o=None,
                    o_dtype=None, stream=None):
    """One decode token per sequence: q, k [N, H_k, 128]; v [N, H_v, 128];
    g, beta [N, H_v]; state fp32 [N, H_v, 128, 128] updated in place.
    Returns o [N, H_v, 128]."""
    N, H_k, _ = q.shape
    H_v = v.shape[1]
    _expect(q, (N, H_k, HEAD_DIM), "q", contiguous=False)
    _expect(k, (N, H_k, HEAD_DIM), "k", q.dtype, contiguous=False)
    _expect(v, (N, H_v, HEAD_DIM), "v", q.dtype, contiguous=False)
    _expect(g, (N, H_v), "g")
    _expect(beta, (N, H_v), "beta", g.dtype)
    _expect(state, (N, H_v, HEAD_DIM, HEAD_DIM), "state", torch.float32)
    _expect(o, (N, H_v, HEAD_DIM), "o")
    if o is None:
        o = torch.empty((N, H_v, HEAD_DIM), dtype=o_dtype or v.dtype, device=v.device)
    _check("gdn_decode_step", load().gdn_decode_step(
        _ptr(q), _ptr(k), _ptr(v), _dtype_code(q.dtype), _row_stride(q),
        _row_stride(k), _row_stride(v), _ptr(g), _ptr(beta), _dtype_code(g.dtype),
        _ptr(state), N, H_k, H_v, scale, _ptr(o), _dtype_code(o.dtype),
        _stream(stream, v.device)))
    return o


def gdn_decode_layer_step(x, conv_w, conv_state, g, beta, state, state_idx, z, norm_w, *,
                          conv_bias=None, scale=1.0, l2_eps=1e-6, norm_eps=1e-6, y=None,
                          y_dtype=None, H_k=H_K, stream=None):
    """One decode token of the whole layer for N sequences (conv roll + SiLU +
    q/k L2, the recurrence, gated RMS-norm) on pooled states: x [N, C] (C =
    2*H_k*128 + H_v*128); conv_w [C, 4]; conv_state [P, 3, C] (x's dtype) and
    state fp32 [P, H_v, 128, 128], both updated in place at the slots
    state_idx int32 [N] (a slot outside [0, P) marks padding); g, beta [N, H_v];
    z [N, H_v, 128] (x's dtype); norm_w [128] (conv_w's dtype). Returns the
    normed output y [N, H_v, 128]."""
    N, C = x.shape
    P, H_v = state.shape[0], state.shape[1]
    if C != (2 * H_k + H_v) * HEAD_DIM:
        raise ValueError(f"x: {C} channels, expected {(2 * H_k + H_v) * HEAD_DIM}")
    _expect(conv_w, (C, 4), "conv_w")
    _expect(conv_bias, (C,), "conv_bias", conv_w.dtype)
    _expect(conv_state, (P, 3, C), "conv_state", x.dtype)
    _expect(g, (N, H_v), "g")
    _expect(beta, (N, H_v), "beta", g.dtype)
    _expect(state, (P, H_v, HEAD_DIM, HEAD_DIM), "state", torch.float32)
    _expect(state_idx, (N,), "state_idx", torch.int32)
    _expect(z, (N, H_v, HEAD_DIM), "z", x.dtype)
    _expect(norm_w, (HEAD_DIM,), "norm_w", conv_w.dtype)
    _expect(y, (N, H_v, HEAD_DIM), "y")
    if y is None:
        y = torch.empty((N, H_v, HEAD_DIM), dtype=y_dtype or x.dtype, device=x.device)
    _check("gdn_decode_layer_step", load().gdn_decode_layer_step(
        _ptr(x), _row_stride(x), _dtype_code(x.dtype), _ptr(conv_w), _dtype_code(conv_w.dtype),
        _ptr(conv_bias), _ptr(conv_state), _ptr(g), _ptr(beta), _dtype_code(g.dtype),
        _ptr(state), _ptr(state_idx), N, P, H_k, H_v, scale, l2_eps, _ptr(z), _ptr(norm_w),
        norm_eps, _ptr(y), _dtype_code(y.dtype), _stream(stream, x.device)))
    return y


def gdn_gated_rmsnorm(x, z, w, *, eps=1e-6, y=None, y_dtype=None, stream=None):
    """y = x / sqrt(mean(x^2) + eps) * w * SiLU(z) over the last dim (128)."""
    dim = x.shape[-1]
    rows = x.numel() // dim if dim else 0
    _expect(z, tuple(x.shape), "z")
    _expect(w, (dim,), "w")
    _expect(y, tuple(x.shape), "y")
    if y is None:
        y = torch.empty(x.shape, dtype=y_dtype or x.dtype, device=x.device)
    for t in (x, z, y):
        if not t.is_contiguous():
            raise ValueError("gdn_gated_rmsnorm takes contiguous tensors")
    _check("gdn_gated_rmsnorm", load().gdn_gated_rmsnorm(
        _ptr(x), _dtype_code(x.dtype), _ptr(z), _dtype_code(z.dtype), _ptr(w),
        _dtype_code(w.dtype), rows, dim, eps, _ptr(y), _dtype_code(y.dtype),
        _stream(stream, x.device)))
    return y


# ------------------------------------------------------------ global attention
ATTN_H_Q, ATTN_H_KV, ATTN_HEAD_DIM = 24, 4, 256


def _head_rows(t, n, H, name):
    """[n, H, 256] bf16 with dense heads and any row stride: returns the stride."""
    _expect(t, (n, H, ATTN_HEAD_DIM), name, torch.bfloat16, contiguous=False)
    return _row_stride(t)


def gdn_attention_prefill(q, k, v, gate, q_norm_w, k_norm_w, cu_seqlens, *, positions=None,
                          pos0=None, eps=1e-6, rope_dims=64, rope_base=1e7, scale=None,
                          o=None, k_rot=None, v_h=None, workspace=None, stream=None):
    """Global-attention layer over packed prompts: q/k RMS-norm, rotary, causal
    GQA attention, sigmoid output gate. q, gate [T, H_q, 256]; k, v [T, H_kv,
    256] (bf16, any token stride); norm weights [256] (bf16 or fp32, one
    dtype); positions [3, T] int32 or pos0 [N] int32. Returns (o, k_rot, v_h):
    o bf16; k_rot, v_h the cache rows in fp16 (normed rotated keys, values)."""
    T, H_q, _ = q.shape
    H_kv = k.shape[1]
    N = cu_seqlens.numel() - 1
    qs = _head_rows(q, T, H_q, "q")
    ks = _head_rows(k, T, H_kv, "k")
    vs = _head_rows(v, T, H_kv, "v")
    gs = _head_rows(gate, T, H_q, "gate")
    _expect(q_norm_w, (ATTN_HEAD_DIM,), "q_norm_w")
    _expect(k_norm_w, (ATTN_HEAD_DIM,), "k_norm_w", q_norm_w.dtype)
    _expect(cu_seqlens, (N + 1,), "cu_seqlens", torch.int32)
    _expect(positions, (3, T), "positions", torch.int32)
    _expect(pos0, (N,), "pos0", torch.int32)
    _expect(o, (T, H_q, ATTN_HEAD_DIM), "o", torch.bfloat16)
    _expect(k_rot, (T, H_kv, ATTN_HEAD_DIM), "k_rot", torch.float16)
    _expect(v_h, (T, H_kv, ATTN_HEAD_DIM), "v_h", torch.float16)
    if o is None:
        o = torch.empty((T, H_q, ATTN_HEAD_DIM), dtype=torch.bfloat16, device=q.device)
    if k_rot is None:
        k_rot = torch.empty((T, H_kv, ATTN_HEAD_DIM), dtype=torch.float16, device=q.device)
    if v_h is None:
        v_h = torch.empty((T, H_kv, ATTN_HEAD_DIM), dtype=torch.float16, device=q.device)
    need = load().gdn_attention_prefill_workspace(T, H_q, ATTN_HEAD_DIM)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    ws_bytes = workspace.numel() * workspace.element_size()
    _check("gdn_attention_prefill", load().gdn_attention_prefill(
        _ptr(q), qs, _ptr(k), ks, _ptr(v), vs, _ptr(gate), gs, _ptr(q_norm_w), _ptr(k_norm_w),
        _dtype_code(q_norm_w.dtype), _ptr(cu_seqlens), _ptr(positions), _ptr(pos0), N, T, H_q,
        H_kv, ATTN_HEAD_DIM, eps, rope_dims, rope_base,
        ATTN_HEAD_DIM ** -0.5 if scale is None else scale, _ptr(o), _ptr(k_rot), _ptr(v_h),
        _ptr(workspace), ws_bytes, _stream(stream, q.device)))
    return o, k_rot, v_h


def gdn_attention_decode(q, k, v, gate, q_norm_w, k_norm_w, k_cache, v_cache, cache_len, *,
                         cache_idx=None, positions=None, eps=1e-6, rope_dims=64, rope_base=1e7,
                         scale=None, o=None, workspace=None, stream=None):
    """One decode step of the global-attention layer for N sequences: appends
    the new rotated k and v at row cache_len[n] of slot cache_idx[n] of the
    fp16 caches [P, L_max, H_kv, 256], attends over rows 0..cache_len[n], and
    advances cache_len (int32 [N], on the device) by one. Returns o [N, H_q, 256]."""
    N, H_q, _ = q.shape
    H_kv = k.shape[1]
    P, L_max = k_cache.shape[0], k_cache.shape[1]
    qs = _head_rows(q, N, H_q, "q")
    ks = _head_rows(k, N, H_kv, "k")
    vs = _head_rows(v, N, H_kv, "v")
    gs = _head_rows(gate, N, H_q, "gate")
    _expect(q_norm_w, (ATTN_HEAD_DIM,), "q_norm_w")
    _expect(k_norm_w, (ATTN_HEAD_DIM,), "k_norm_w", q_norm_w.dtype)
    _expect(k_cache, (P, L_max, H_kv, ATTN_HEAD_DIM), "k_cache", torch.float16)
    _expect(v_cache, (P, L_max, H_kv, ATTN_HEAD_DIM), "v_cache", torch.float16)
    _expect(cache_len, (N,), "cache_len", torch.int32)
    _expect(cache_idx, (N,), "cache_idx", torch.int32)
    _expect(positions, (3, N), "positions", torch.int32)
    _expect(o, (N, H_q, ATTN_HEAD_DIM), "o", torch.bfloat16)
    if o is None:
        o = torch.empty((N, H_q, ATTN_HEAD_DIM), dtype=torch.bfloat16, device=q.device)
    need = load().gdn_attention_decode_workspace(N, H_q, L_max, ATTN_HEAD_DIM)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    ws_bytes = workspace.numel() * workspace.element_size()
    _check("gdn_attention_decode", load().gdn_attention_decode(
        _ptr(q), qs, _ptr(k), ks, _ptr(v), vs, _ptr(gate), gs, _ptr(q_norm_w), _ptr(k_norm_w),
        _dtype_code(q_norm_w.dtype), _ptr(k_cache), _ptr(v_cache), _ptr(cache_idx),
        _ptr(cache_len), _ptr(positions), N, P, L_max, H_q, H_kv, ATTN_HEAD_DIM, eps,
        rope_dims, rope_base, ATTN_HEAD_DIM ** -0.5 if scale is None else scale, _ptr(o),
        _ptr(workspace), ws_bytes, _stream(stream, q.device)))
    return o


def gdn_attention_status(workspace, stream=None) -> int:
    """Waits for `stream`, then returns the status the last attention call left
    in `workspace`: 0, GDN_ERR_TIMEOUT, or GDN_ERR_INVALID_ARG (a decode
    sequence with an out-of-range slot or length)."""
    return int(load().gdn_attention_status(_ptr(workspace), _stream(stream, workspace.device)))

