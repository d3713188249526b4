"""The C ABI: libgdn.so loads, exports every function include/gdn.h declares,
and rejects bad arguments on the host before launching anything.

These run without a GPU: every call here fails validation, which happens
before any CUDA call, so no device work is attempted.
"""
import ctypes
import os
import re
import subprocess

import pytest

import gated_delta_rule_106_b200 as gdn
from gated_delta_rule_106_b200 import _build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gdn.h")

OK, INVALID, UNSUPPORTED, MISALIGNED = 0, -1, -2, -3
BF16, F32 = gdn.GDN_BF16, gdn.GDN_F32
A = 0x10000          # a 16-byte aligned fake device address (never dereferenced)


@pytest.fixture(scope="module")
def lib():
    _build.build()
    return gdn.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gdn_\w+)\s*\(", text)))


def test_header_declares_the_four_entry_points():
    names = declared_functions()
    for n in ("gdn_conv1d_silu", "gdn_chunked_prefill", "gdn_decode_step",
              "gdn_gated_rmsnorm"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", gdn.library_path()],
                         capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\b(gdn_\w+)$", out, flags=re.M))
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, missing
    for n in declared_functions():
        getattr(lib, n)


def test_header_compiles_as_plain_c(tmp_path):
    src = tmp_path / "t.c"
    src.write_text('#include "gdn.h"\nint main(void){return (int)GDN_OK;}\n')
    subprocess.run(["gcc", "-std=c99", "-fsyntax-only", "-I", os.path.join(ROOT, "include"),
                    "-I", "/usr/local/cuda/include", str(src)], check=True)


def test_status_strings(lib):
    assert gdn.gdn_status_string(0) == "GDN_OK"
    for s in (INVALID, UNSUPPORTED, MISALIGNED, -4):
        assert "GDN_ERR" in gdn.gdn_status_string(s)
    assert gdn.gdn_version().count(".") == 2


def conv(lib, **kw):
    a = dict(x=A, xs=10240, xdt=BF16, w=A, wdt=F32, bias=None, C=10240,
             l2c=4096, eps=1e-6, cu=A, N=1, T=8, csi=None, cso=None, y=A,
             ys=10240, ydt=BF16, s=None)
    a.update(kw)
    return lib.gdn_conv1d_silu(*a.values())


def test_conv_validation(lib):
    assert conv(lib, C=10241) == INVALID                 # channels % 8
    assert conv(lib, l2c=100) == INVALID                 # not a multiple of 128
    assert conv(lib, l2c=20480) == INVALID               # beyond channels
    assert conv(lib, xdt=7) == INVALID
    assert conv(lib, N=-1) == INVALID
    assert conv(lib, T=-1) == INVALID
    assert conv(lib, x=None) == INVALID
    assert conv(lib, cu=None) == INVALID
    assert conv(lib, xs=100) == INVALID                  # stride < channels
    assert conv(lib, x=A + 2) == MISALIGNED
    assert conv(lib, y=A + 8) == MISALIGNED
    assert conv(lib, xs=10244) == MISALIGNED             # 20488 B not /16
    assert conv(lib, csi=A + 4) == MISALIGNED
    assert conv(lib, csi=A, cso=A + 16) == INVALID       # partial overlap
    assert conv(lib, N=0, T=0) == OK                     # nothing to do
    assert conv(lib, N=0, T=5) == INVALID


def prefill(lib, **kw):
    a = dict(q=A, k=A, v=A, dt=BF16, qs=10240, ks=10240, vs=10240, g=A, b=A,
             gdt=F32, si=None, so=None, cu=A, N=1, T=64, Hk=16, Hv=48,
             scale=1.0, o=A, odt=BF16, ws=None, wsb=0, s=None)
    a.update(kw)
    return lib.gdn_chunked_prefill(*a.values())


def test_prefill_validation(lib):
    assert prefill(lib, Hv=40) == INVALID                # H_v % H_k
    assert prefill(lib, Hk=0) == INVALID
    assert prefill(lib, qs=100) == INVALID               # stride < H_k * 128
    assert prefill(lib, q=None) == INVALID
    assert prefill(lib, cu=None) == INVALID
    assert prefill(lib, dt=5) == INVALID
    assert prefill(lib, q=A + 2) == MISALIGNED
    assert prefill(lib, o=A + 4) == MISALIGNED
    assert prefill(lib, qs=10244) == MISALIGNED
    assert prefill(lib, g=A + 2) == MISALIGNED           # fp32 gate needs 4 B
    assert prefill(lib, si=A + 8) == MISALIGNED
    st = 48 * 128 * 128 * 4
    assert prefill(lib, si=A, so=A + st // 2) == INVALID  # partial overlap
    assert prefill(lib, N=0, T=0) == OK
    assert prefill(lib, N=0, T=3) == INVALID
    assert prefill(lib, N=-1) == INVALID


def test_prefill_workspace_query(lib):
    assert gdn.gdn_chunked_prefill_workspace(16, 135000) >= 0


def decode(lib, **kw):
    a = dict(q=A, k=A, v=A, dt=BF16, qs=10240, ks=10240, vs=10240, g=A, b=A,
             gdt=BF16, state=A, N=256, Hk=16, Hv=48, scale=1.0, o=A, odt=BF16,
             s=None)
    a.update(kw)
    return lib.gdn_decode_step(*a.values())


def test_decode_validation(lib):
    assert decode(lib, state=None) == INVALID
    assert decode(lib, state=A + 4) == MISALIGNED
    assert decode(lib, Hv=47) == INVALID
    assert decode(lib, v=A + 2) == MISALIGNED
    assert decode(lib, N=-2) == INVALID
    assert decode(lib, N=0) == OK


def norm(lib, **kw):
    a = dict(x=A, xdt=BF16, z=A, zdt=BF16, w=A, wdt=F32, rows=10, dim=128,
             eps=1e-6, y=A, ydt=BF16, s=None)
    a.update(kw)
    return lib.gdn_gated_rmsnorm(*a.values())


def test_rmsnorm_validation(lib):
    assert norm(lib, dim=64) == UNSUPPORTED
    assert norm(lib, rows=-1) == INVALID
    assert norm(lib, z=None) == INVALID
    assert norm(lib, eps=-1.0) == INVALID
    assert norm(lib, x=A + 2) == MISALIGNED
    assert norm(lib, ydt=F32) == INVALID                 # y aliases x, other dtype
    assert norm(lib, rows=0) == OK


def test_binding_refuses_cpu_tensors(lib):
    import torch
    x = torch.zeros(4, 16, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        gdn.gdn_gated_rmsnorm(torch.zeros(2, 128), torch.zeros(2, 128),
                              torch.ones(128))
    del x


def test_binding_checks_shapes_before_pointers(lib):
    """The kernels write dense layouts, so the binding refuses a tensor of the
    wrong shape, dtype or layout before any pointer reaches the library (the
    tensors here are on the CPU: the check must come first to be seen)."""
    import torch
    T, N = 8, 1
    q = torch.zeros(T, 16, 128, dtype=torch.bfloat16)
    v = torch.zeros(T, 48, 128, dtype=torch.bfloat16)
    g, b = torch.ones(T, 48), torch.ones(T, 48)
    cu = torch.tensor([0, T], dtype=torch.int32)
    pre = lambda **kw: gdn.gdn_chunked_prefill(q, q, v, g, b, cu, **kw)
    with pytest.raises(ValueError, match="o: shape"):
        pre(o=torch.empty(T, 47, 128))
    with pytest.raises(ValueError, match="o must be contiguous"):
        pre(o=torch.empty(T, 128, 48).transpose(1, 2))
    with pytest.raises(ValueError, match="state_out: dtype"):
        pre(state_out=torch.empty(N, 48, 128, 128, dtype=torch.float64))
    with pytest.raises(ValueError, match="state_in: shape"):
        pre(state_in=torch.empty(2, 48, 128, 128))
    with pytest.raises(ValueError, match="beta: dtype"):
        gdn.gdn_chunked_prefill(q, q, v, g, b.double(), cu)
    with pytest.raises(ValueError, match="g: shape"):
        gdn.gdn_chunked_prefill(q, q, v, g[:, :47], b, cu)
    with pytest.raises(ValueError, match="k: shape"):
        gdn.gdn_chunked_prefill(q, q[:, :8], v, g, b, cu)
    with pytest.raises(ValueError, match="state: shape"):
        gdn.gdn_decode_step(q[:1], q[:1], v[:1], g[:1], b[:1], torch.empty(2, 48, 128, 128))
    with pytest.raises(ValueError, match="conv_state_out: dtype"):
        gdn.gdn_conv1d_silu(torch.zeros(T, 256, dtype=torch.bfloat16), torch.ones(256, 4), cu,
                            conv_state_out=torch.empty(N, 3, 256))
    with pytest.raises(ValueError, match="w: shape"):
        gdn.gdn_conv1d_silu(torch.zeros(T, 256, dtype=torch.bfloat16), torch.ones(256, 3), cu)
    with pytest.raises(ValueError, match="z: shape"):
        gdn.gdn_gated_rmsnorm(torch.zeros(T, 128), torch.zeros(T, 64), torch.ones(128))


def test_binding_refuses_mixed_dtypes(lib):
    """One qkv dtype crosses the C ABI (q's), and the conv bias is read in w's
    dtype, cu_seqlens as int32: a k or v of another dtype than q, a bias of
    another dtype than w, or int64 cu_seqlens would be read past their bytes
    or misread, so the binding refuses them before any pointer is taken."""
    import torch
    T = 8
    q32 = torch.zeros(T, 16, 128)
    k16 = torch.zeros(T, 16, 128, dtype=torch.bfloat16)
    v16 = torch.zeros(T, 48, 128, dtype=torch.bfloat16)
    v32 = torch.zeros(T, 48, 128)
    g, b = torch.ones(T, 48), torch.ones(T, 48)
    cu = torch.tensor([0, T], dtype=torch.int32)
    with pytest.raises(ValueError, match="k: dtype"):
        gdn.gdn_chunked_prefill(q32, k16, v32, g, b, cu)
    with pytest.raises(ValueError, match="v: dtype"):
        gdn.gdn_chunked_prefill(q32, q32, v16, g, b, cu)
    with pytest.raises(ValueError, match="k: dtype"):
        gdn.gdn_chunked_prefill_noalloc(q32, k16, v32, g, b, cu)
    with pytest.raises(ValueError, match="cu_seqlens: dtype"):
        gdn.gdn_chunked_prefill(q32, q32, v32, g, b, cu.long())
    with pytest.raises(ValueError, match="k: dtype"):
        gdn.gdn_decode_step(q32[:1], k16[:1], v32[:1], g[:1], b[:1],
                            torch.zeros(1, 48, 128, 128))
    with pytest.raises(ValueError, match="v: dtype"):
        gdn.gdn_decode_step(q32[:1], q32[:1], v16[:1], g[:1], b[:1],
                            torch.zeros(1, 48, 128, 128))
    x = torch.zeros(T, 256, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="bias: dtype"):
        gdn.gdn_conv1d_silu(x, torch.ones(256, 4), cu,
                            bias=torch.zeros(256, dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="cu_seqlens: dtype"):
        gdn.gdn_conv1d_silu(x, torch.ones(256, 4), cu.long())


def decode_layer(lib, **kw):
    a = dict(x=A, xs=10240, xdt=BF16, w=A, wdt=F32, bias=None, cache=A, g=A, beta=A,
             gdt=F32, state=A, idx=A, N=4, P=8, H_k=16, H_v=48, scale=1.0, l2_eps=1e-6,
             z=A, nw=A, norm_eps=1e-6, y=A, ydt=BF16, s=None)
    a.update(kw)
    return lib.gdn_decode_layer_step(*a.values())


def test_decode_layer_validation(lib):
    assert decode_layer(lib, N=-1) == INVALID
    assert decode_layer(lib, H_v=47) == INVALID            # H_v % H_k
    assert decode_layer(lib, H_k=4, H_v=48, xs=7168) == UNSUPPORTED  # 12 per key head
    assert decode_layer(lib, xs=10239) == INVALID           # stride below C = 10240
    assert decode_layer(lib, P=0) == INVALID
    assert decode_layer(lib, idx=None) == INVALID
    assert decode_layer(lib, z=None) == INVALID
    assert decode_layer(lib, x=A + 2) == MISALIGNED
    assert decode_layer(lib, state=A + 8) == MISALIGNED
    assert decode_layer(lib, idx=A + 2) == MISALIGNED
    assert decode_layer(lib, xs=10244) == MISALIGNED        # 20488 bytes, not 16-aligned
    assert decode_layer(lib, l2_eps=-1.0) == INVALID
    assert decode_layer(lib, xdt=7) == INVALID
    assert decode_layer(lib, N=0) == OK


def test_decode_layer_binding_checks(lib):
    import torch
    N, P = 2, 3
    x = torch.zeros(N, 10240, dtype=torch.bfloat16)
    w = torch.zeros(10240, 4)
    cache = torch.zeros(P, 3, 10240, dtype=torch.bfloat16)
    g = torch.ones(N, 48)
    S = torch.zeros(P, 48, 128, 128)
    idx = torch.zeros(N, dtype=torch.int32)
    z = torch.zeros(N, 48, 128, dtype=torch.bfloat16)
    nw = torch.ones(128)
    call = lambda **kw: gdn.gdn_decode_layer_step(
        kw.get("x", x), w, kw.get("cache", cache), g, g, S, kw.get("idx", idx),
        kw.get("z", z), kw.get("nw", nw))
    with pytest.raises(ValueError, match="channels"):
        call(x=torch.zeros(N, 10112, dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="conv_state: dtype"):
        call(cache=cache.float())
    with pytest.raises(ValueError, match="state_idx: dtype"):
        call(idx=idx.long())
    with pytest.raises(ValueError, match="z: dtype"):
        call(z=z.float())
    with pytest.raises(ValueError, match="norm_w: dtype"):
        call(nw=nw.bfloat16())


def attn_prefill(lib, **kw):
    a = dict(q=A, qs=24 * 256, k=A, ks=4 * 256, v=A, vs=4 * 256, gate=A, gs=24 * 256, wq=A,
             wk=A, wdt=BF16, cu=A, pos=None, pos0=None, N=1, T=128, Hq=24, Hkv=4, D=256,
             eps=1e-6, R=64, base=1e7, scale=0.0625, o=A, k_rot=A, v_h=A, ws=A,
             ws_bytes=1 << 40, s=None)
    a.update(kw)
    return lib.gdn_attention_prefill(*a.values())


def attn_decode(lib, **kw):
    a = dict(q=A, qs=24 * 256, k=A, ks=4 * 256, v=A, vs=4 * 256, gate=A, gs=24 * 256, wq=A,
             wk=A, wdt=BF16, kc=A, vc=A, idx=None, len=A, pos=None, N=4, P=4, L=1024, Hq=24,
             Hkv=4, D=256, eps=1e-6, R=64, base=1e7, scale=0.0625, o=A, ws=A,
             ws_bytes=1 << 40, s=None)
    a.update(kw)
    return lib.gdn_attention_decode(*a.values())


def test_attention_prefill_validation(lib):
    assert attn_prefill(lib, D=128) == UNSUPPORTED
    assert attn_prefill(lib, Hkv=5) == INVALID               # 24 % 5
    assert attn_prefill(lib, Hq=12, Hkv=4, qs=12 * 256, gs=12 * 256) == UNSUPPORTED  # 3 per group
    assert attn_prefill(lib, R=66) == UNSUPPORTED
    assert attn_prefill(lib, R=63) == UNSUPPORTED
    assert attn_prefill(lib, base=1.0) == INVALID
    assert attn_prefill(lib, eps=-1.0) == INVALID
    assert attn_prefill(lib, wdt=7) == INVALID
    assert attn_prefill(lib, N=0) == INVALID                 # tokens but no sequence
    assert attn_prefill(lib, qs=24 * 256 - 8) == MISALIGNED  # stride below H_q * 256
    assert attn_prefill(lib, vs=4 * 256 + 4) == MISALIGNED   # not a multiple of 8 elements
    assert attn_prefill(lib, cu=None) == INVALID
    assert attn_prefill(lib, k_rot=None) == INVALID
    assert attn_prefill(lib, v_h=None) == INVALID
    assert attn_prefill(lib, v_h=A + 8) == MISALIGNED
    assert attn_prefill(lib, ws_bytes=1024) == INVALID
    assert attn_prefill(lib, q=A + 2) == MISALIGNED
    assert attn_prefill(lib, ws=A + 8) == MISALIGNED
    assert attn_prefill(lib, wq=A + 2, wdt=F32) == MISALIGNED
    assert attn_prefill(lib, T=0) == OK
    need = lib.gdn_attention_prefill_workspace(8192, 24, 256)
    assert need >= 8192 * 24 * 256 * 2
    assert lib.gdn_attention_prefill_workspace(8192, 24, 128) == 0


def test_attention_decode_validation(lib):
    assert attn_decode(lib, D=128) == UNSUPPORTED
    assert attn_decode(lib, Hq=12, Hkv=4, qs=12 * 256, gs=12 * 256) == UNSUPPORTED  # 3 per group
    assert attn_decode(lib, N=-1) == INVALID
    assert attn_decode(lib, N=70000) == INVALID
    assert attn_decode(lib, P=0) == INVALID
    assert attn_decode(lib, L=0) == INVALID
    assert attn_decode(lib, len=None) == INVALID
    assert attn_decode(lib, kc=None) == INVALID
    assert attn_decode(lib, kc=A + 8) == MISALIGNED
    assert attn_decode(lib, ks=4 * 256 + 2) == MISALIGNED
    assert attn_decode(lib, ws_bytes=256) == INVALID
    assert attn_decode(lib, N=0) == OK
    assert lib.gdn_attention_decode_workspace(256, 24, 4224, 256) > 256 * 24 * 256 * 4
    assert lib.gdn_attention_status(None, None) == INVALID
    assert lib.gdn_attention_status(A + 4, None) == MISALIGNED


def test_attention_binding_checks(lib):
    import torch
    T, N = 16, 1
    q = torch.zeros(T, 24, 256, dtype=torch.bfloat16)
    k = torch.zeros(T, 4, 256, dtype=torch.bfloat16)
    w = torch.ones(256, dtype=torch.bfloat16)
    cu = torch.tensor([0, T], dtype=torch.int32)
    with pytest.raises(ValueError, match="k: dtype"):
        gdn.gdn_attention_prefill(q, k.float(), k, q, w, w, cu)
    with pytest.raises(ValueError, match="gate: shape"):
        gdn.gdn_attention_prefill(q, k, k, k, w, w, cu)
    with pytest.raises(ValueError, match="k_norm_w: dtype"):
        gdn.gdn_attention_prefill(q, k, k, q, w, w.float(), cu)
    with pytest.raises(ValueError, match="cu_seqlens: dtype"):
        gdn.gdn_attention_prefill(q, k, k, q, w, w, cu.long())
    with pytest.raises(ValueError, match="positions: shape"):
        gdn.gdn_attention_prefill(q, k, k, q, w, w, cu,
                                  positions=torch.zeros(T, 3, dtype=torch.int32))
    with pytest.raises(ValueError, match="CUDA tensors only"):
        gdn.gdn_attention_prefill(q, k, k, q, w, w, cu)
    kc = torch.zeros(2, 64, 4, 256, dtype=torch.float16)
    vb = torch.zeros(2, 64, 4, 256, dtype=torch.bfloat16)
    ln = torch.zeros(N, dtype=torch.int32)
    with pytest.raises(ValueError, match="k_cache: dtype"):
        gdn.gdn_attention_decode(q[:N], k[:N], k[:N], q[:N], w, w, vb, kc, ln)
    with pytest.raises(ValueError, match="v_cache: dtype"):
        gdn.gdn_attention_decode(q[:N], k[:N], k[:N], q[:N], w, w, kc, vb, ln)
    with pytest.raises(ValueError, match="cache_len: dtype"):
        gdn.gdn_attention_decode(q[:N], k[:N], k[:N], q[:N], w, w, kc, kc, ln.long())
    with pytest.raises(ValueError, match="v_h: dtype"):
        gdn.gdn_attention_prefill(q, k, k, q, w, w, cu,
                                  v_h=torch.zeros(T, 4, 256, dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="k_rot: dtype"):
        gdn.gdn_attention_prefill(q, k, k, q, w, w, cu,
                                  k_rot=torch.zeros(T, 4, 256, dtype=torch.bfloat16))
