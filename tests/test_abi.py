"""Host-side checks of the C ABI: the library loads, exports every function
declared in include/deltanet.h, and rejects bad arguments before touching a
GPU (these calls never reach the device)."""
import ctypes
import os
import re

import pytest

from deltanet_chunkwise_delta_b200 import _lib as L
from deltanet_chunkwise_delta_b200 import build as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    src = open(os.path.join(ROOT, "include", "deltanet.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b((?:gated_)?delta(?:net|product)_\w+|kda_\w+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    B.build()
    return L.load()


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert set(names) == set(L.EXPORTED)
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings(lib):
    for code in range(8):
        s = L.status_string(code)
        assert s.startswith("DN_")
    assert "unknown" in L.status_string(99)


def desc(shape, dtype=L.DN_BF16, data=0x10000, strides=None):
    d = L.DnTensor()
    d.data = data
    d.dtype = dtype
    d.ndim = len(shape)
    if strides is None:
        strides, acc = [], 1
        for s in reversed(shape):
            strides.insert(0, acc)
            acc *= s
    for i in range(4):
        d.shape[i] = shape[i] if i < len(shape) else 0
        d.stride[i] = strides[i] if i < len(shape) else 0
    return d


def call(lib, q, k, v, beta, s0=None, cu=None, chunk=64, out=None, sT=None):
    r = lambda x: None if x is None else ctypes.byref(x)
    return lib.deltanet_fwd(r(q), r(k), r(v), r(beta), r(s0), r(cu), chunk, r(out), r(sT), None)


def good(B=2, T=100, H=3, dk=128, dv=64, dtype=L.DN_BF16):
    base = 0x100000000
    es = 2 if dtype == L.DN_BF16 else 4
    q = desc([B, T, H, dk], dtype, base)
    k = desc([B, T, H, dk], dtype, base + 1 * 2**28)
    v = desc([B, T, H, dv], dtype, base + 2 * 2**28)
    beta = desc([B, T, H], L.DN_F32, base + 3 * 2**28)
    out = desc([B, T, H, dv], dtype, base + 4 * 2**28)
    s0 = desc([B, H, dk, dv], L.DN_F32, base + 5 * 2**28)
    sT = desc([B, H, dk, dv], L.DN_F32, base + 6 * 2**28)
    return q, k, v, beta, s0, out, sT


def test_rejects_null_and_bad_shapes(lib):
    q, k, v, beta, s0, out, sT = good()
    assert call(lib, None, k, v, beta, out=out) == L.DN_ERR_INVALID_ARG
    assert call(lib, q, k, v, beta, out=None) == L.DN_ERR_INVALID_ARG
    kb = desc([2, 100, 3, 64], L.DN_BF16, 0x200000000)
    assert call(lib, q, kb, v, beta, out=out) == L.DN_ERR_INVALID_ARG
    bb = desc([2, 100, 4], L.DN_F32, 0x300000000)
    assert call(lib, q, k, v, bb, out=out) == L.DN_ERR_INVALID_ARG
    s_bad = desc([2, 3, 64, 64], L.DN_F32, 0x500000000)
    assert call(lib, q, k, v, beta, s0=s_bad, out=out) == L.DN_ERR_INVALID_ARG


def test_rejects_dtype_stride_alignment(lib):
    q, k, v, beta, s0, out, sT = good()
    kf = good(dtype=L.DN_F32)[1]
    assert call(lib, q, kf, v, beta, out=out) == L.DN_ERR_INVALID_ARG
    bb = good()[3]
    bb.dtype = L.DN_BF16
    assert call(lib, q, k, v, bb, out=out) == L.DN_ERR_INVALID_ARG
    qs = good()[0]
    qs.stride[3] = 2
    assert call(lib, qs, k, v, beta, out=out) == L.DN_ERR_INVALID_ARG
    qa = good()[0]
    qa.data = qa.data + 2
    assert call(lib, qa, k, v, beta, out=out) == L.DN_ERR_INVALID_ARG
    qh = good()[0]
    qh.stride[2] = 129            # 258-byte head stride: not a multiple of 16
    assert call(lib, qh, k, v, beta, out=out) == L.DN_ERR_INVALID_ARG


def test_rejects_unsupported(lib):
    q, k, v, beta, s0, out, sT = good()
    assert call(lib, q, k, v, beta, out=out, chunk=32) == L.DN_ERR_UNSUPPORTED
    q2, k2, v2, b2, _, o2, _ = good(dk=96)
    assert call(lib, q2, k2, v2, b2, out=o2) == L.DN_ERR_UNSUPPORTED
    q3, k3, v3, b3, _, o3, _ = good(dk=128, dv=128, dtype=L.DN_F32)
    assert call(lib, q3, k3, v3, b3, out=o3) == L.DN_ERR_UNSUPPORTED


def test_rejects_aliasing(lib):
    q, k, v, beta, s0, out, sT = good()
    o_on_q = desc([2, 100, 3, 64], L.DN_BF16, q.data + 4096)
    assert call(lib, q, k, v, beta, out=o_on_q) == L.DN_ERR_ALIAS
    same = desc([2, 3, 128, 64], L.DN_F32, s0.data)
    assert call(lib, q, k, v, beta, s0=s0, out=out, sT=same) == L.DN_ERR_ALIAS
    sT_on_out = desc([2, 3, 128, 64], L.DN_F32, out.data)
    assert call(lib, q, k, v, beta, out=out, sT=sT_on_out) == L.DN_ERR_ALIAS


def test_rejects_bad_varlen_descriptors(lib):
    q, k, v, beta, s0, out, sT = good()          # B = 2
    cu = desc([3], L.DN_I32, 0x700000000)
    assert call(lib, q, k, v, beta, cu=cu, out=out) == L.DN_ERR_INVALID_ARG
    q1, k1, v1, b1, _, o1, _ = good(B=1)
    cu_f = desc([3], L.DN_F32, 0x700000000)
    assert call(lib, q1, k1, v1, b1, cu=cu_f, out=o1) == L.DN_ERR_INVALID_ARG
    s_wrong_n = desc([1, 3, 128, 64], L.DN_F32, 0x500000000)   # N = 2 from cu
    assert call(lib, q1, k1, v1, b1, s0=s_wrong_n, cu=cu, out=o1) == L.DN_ERR_INVALID_ARG


def call_gated(lib, q, k, v, beta, g, s0=None, cu=None, chunk=64, out=None, sT=None):
    r = lambda x: None if x is None else ctypes.byref(x)
    return lib.gated_deltanet_fwd(r(q), r(k), r(v), r(beta), r(g), r(s0), r(cu), chunk, r(out),
                                  r(sT), None)


def test_gated_rejects_bad_gate(lib):
    """The log-decay tensor follows beta's rules: [B, T, H] fp32, 4-byte aligned,
    non-negative strides, required, and no output may overlap it."""
    q, k, v, beta, s0, out, sT = good()
    g = desc([2, 100, 3], L.DN_F32, 0x100000000 + 7 * 2**28)
    assert call_gated(lib, q, k, v, beta, None, out=out) == L.DN_ERR_INVALID_ARG
    g_shape = desc([2, 100, 4], L.DN_F32, g.data)
    assert call_gated(lib, q, k, v, beta, g_shape, out=out) == L.DN_ERR_INVALID_ARG
    g_type = desc([2, 100, 3], L.DN_BF16, g.data)
    assert call_gated(lib, q, k, v, beta, g_type, out=out) == L.DN_ERR_INVALID_ARG
    g_align = desc([2, 100, 3], L.DN_F32, g.data + 2)
    assert call_gated(lib, q, k, v, beta, g_align, out=out) == L.DN_ERR_INVALID_ARG
    g_neg = desc([2, 100, 3], L.DN_F32, g.data, strides=[300, -3, 1])
    assert call_gated(lib, q, k, v, beta, g_neg, out=out) == L.DN_ERR_INVALID_ARG
    o_on_g = desc([2, 100, 3, 64], L.DN_BF16, g.data)
    assert call_gated(lib, q, k, v, beta, g, out=o_on_g) == L.DN_ERR_ALIAS
    assert call_gated(lib, q, k, v, beta, g, out=out, chunk=32) == L.DN_ERR_UNSUPPORTED
    r = lambda x: ctypes.byref(x)
    assert lib.gated_deltanet_fwd_ex(r(q), r(k), r(v), r(beta), None, None, None, 64, r(out),
                                     None, None, 2) == L.DN_ERR_INVALID_ARG


def test_gdp_rejects_bad_rows(lib):
    """Gated Delta Product: k, v and beta hold n_h rows per token of q; g and out
    one; n_h >= 1; the gate is required."""
    r = lambda x: None if x is None else ctypes.byref(x)
    base = 0x100000000
    q = desc([2, 50, 3, 128], L.DN_BF16, base)
    k = desc([2, 100, 3, 128], L.DN_BF16, base + 1 * 2**28)
    v = desc([2, 100, 3, 64], L.DN_BF16, base + 2 * 2**28)
    beta = desc([2, 100, 3], L.DN_F32, base + 3 * 2**28)
    out = desc([2, 50, 3, 64], L.DN_BF16, base + 4 * 2**28)
    g = desc([2, 50, 3], L.DN_F32, base + 7 * 2**28)
    f = lambda qq, kk, vv, bb, gg, nh, oo: lib.gated_deltaproduct_fwd(
        r(qq), r(kk), r(vv), r(bb), r(gg), None, None, nh, 64, r(oo), None, None)
    assert f(q, k, v, beta, None, 2, out) == L.DN_ERR_INVALID_ARG
    assert f(q, k, v, beta, g, 0, out) == L.DN_ERR_INVALID_ARG
    assert f(q, k, v, beta, g, 3, out) == L.DN_ERR_INVALID_ARG          # k has 2 rows per token
    g_rows = desc([2, 100, 3], L.DN_F32, g.data)
    assert f(q, k, v, beta, g_rows, 2, out) == L.DN_ERR_INVALID_ARG     # g is per token
    o_rows = desc([2, 100, 3, 64], L.DN_BF16, out.data)
    assert f(q, k, v, beta, g, 2, o_rows) == L.DN_ERR_INVALID_ARG       # out is per token
    b_tok = desc([2, 50, 3], L.DN_F32, beta.data)
    assert f(q, k, v, b_tok, g, 2, out) == L.DN_ERR_INVALID_ARG         # beta is per write
    assert lib.gated_deltaproduct_fwd(r(q), r(k), r(v), r(beta), r(g), None, None, 2, 32,
                                      r(out), None, None) == L.DN_ERR_UNSUPPORTED


def test_states_rejects_bad_buffer(lib):
    """deltanet_fwd_states: chunk_states is required, fp32 [rows, H, d_k, d_v] with
    rows = B * ceil(T / 64) (dense), and may not overlap another tensor."""
    r = lambda x: None if x is None else ctypes.byref(x)
    q, k, v, beta, s0, out, sT = good()           # B = 2, T = 100: 2 chunks per row
    cs = desc([4, 3, 128, 64], L.DN_F32, 0x100000000 + 8 * 2**28)
    f = lambda c, o=out: lib.deltanet_fwd_states(r(q), r(k), r(v), r(beta), None, None, None,
                                                 64, r(o), None, r(c), None, 0)
    assert f(None) == L.DN_ERR_INVALID_ARG
    assert f(desc([3, 3, 128, 64], L.DN_F32, cs.data)) == L.DN_ERR_INVALID_ARG
    assert f(desc([4, 3, 128, 64], L.DN_BF16, cs.data)) == L.DN_ERR_INVALID_ARG
    assert f(desc([4, 3, 64, 128], L.DN_F32, cs.data)) == L.DN_ERR_INVALID_ARG
    assert f(desc([4, 3, 128, 64], L.DN_F32, q.data)) == L.DN_ERR_ALIAS
    assert f(cs, desc([2, 100, 3, 64], L.DN_BF16, cs.data)) == L.DN_ERR_ALIAS


def test_binding_host_logic():
    """Row count of the chunk-states buffer, and the wrappers refuse CPU tensors
    (there is no host implementation to fall back to)."""
    import torch
    import deltanet_chunkwise_delta_b200 as dn
    assert dn.chunk_state_rows(8, 2048) == 8 * 32
    assert dn.chunk_state_rows(3, 65) == 3 * 2
    cu = torch.tensor([0, 1, 65, 65, 200], dtype=torch.int32)   # 1 + 1 + 0 + 3 = 5 chunks
    assert dn.chunk_state_rows(1, 200, cu) == 4 + 4 >= 5
    x = torch.zeros(1, 4, 1, 64)
    b = torch.zeros(1, 4, 1)
    with pytest.raises(ValueError):
        dn.gated_deltanet_fwd(x, x, x, b, b)
    with pytest.raises(ValueError):
        dn.gated_deltaproduct_fwd(x, x, x, b, b, 1)
    with pytest.raises(ValueError):
        dn.deltanet_fwd_states(x, x, x, b)


def call_kda(lib, q, k, v, beta, g, s0=None, cu=None, chunk=64, out=None, sT=None):
    r = lambda x: None if x is None else ctypes.byref(x)
    return lib.kda_fwd(r(q), r(k), r(v), r(beta), r(g), r(s0), r(cu), chunk, r(out), r(sT), None)


def test_kda_rejects_bad_gates_and_types(lib):
    """Kimi Delta Attention takes one log decay per key channel [B, T, H, d_k] fp32 with
    16-byte aligned rows, bf16 inputs only; all checked before the device."""
    q, k, v, beta, s0, out, sT = good(dk=128, dv=128)
    g_ok = desc([2, 100, 3, 128], L.DN_F32, 0x100000000 + 7 * 2**28)
    assert call_kda(lib, q, k, v, beta, None, out=out) == L.DN_ERR_INVALID_ARG
    g_scalar = desc([2, 100, 3], L.DN_F32, 0x100000000 + 7 * 2**28)
    assert call_kda(lib, q, k, v, beta, g_scalar, out=out) == L.DN_ERR_INVALID_ARG
    g_bf16 = desc([2, 100, 3, 128], L.DN_BF16, 0x100000000 + 7 * 2**28)
    assert call_kda(lib, q, k, v, beta, g_bf16, out=out) == L.DN_ERR_INVALID_ARG
    g_odd = desc([2, 100, 3, 128], L.DN_F32, 0x100000000 + 7 * 2**28,
                 strides=[100 * 3 * 130, 3 * 130, 130, 1])   # rows not 16-byte multiples
    assert call_kda(lib, q, k, v, beta, g_odd, out=out) == L.DN_ERR_INVALID_ARG
    g_mis = desc([2, 100, 3, 128], L.DN_F32, 0x100000000 + 7 * 2**28 + 4)
    assert call_kda(lib, q, k, v, beta, g_mis, out=out) == L.DN_ERR_INVALID_ARG
    qf, kf, vf, bf, s0f, outf, sTf = good(dk=64, dv=64, dtype=L.DN_F32)
    gf = desc([2, 100, 3, 64], L.DN_F32, 0x100000000 + 7 * 2**28)
    assert call_kda(lib, qf, kf, vf, bf, gf, out=outf) == L.DN_ERR_UNSUPPORTED
    # an output over the gate is refused like any other aliasing
    out_on_g = desc([2, 100, 3, 128], L.DN_BF16, 0x100000000 + 7 * 2**28)
    assert call_kda(lib, q, k, v, beta, g_ok, out=out_on_g) == L.DN_ERR_ALIAS
