"""The oracle for the DeltaNet forward pass.

TEST INFRASTRUCTURE ONLY: only ``tests/``, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline / reference arm may import this package.  The product
path (``deltanet_chunkwise_delta_b200``) never imports it, and it never imports
the product.

Two independent float64 statements of the method:

* ``token_recurrence`` -- the plain definition, a C float64 token-serial loop
  ("Linear Attention, Visualized", DeltaNet, "Recurrent form"), threaded over
  (sequence, head); with a gate ``g`` = ln a_t it runs the Gated DeltaNet
  recurrence of the same page (section "Gated DeltaNet (GDN)"), and with
  ``n_sub`` > 1 the Gated Delta Product (section "Gated Delta Product (GDP)");
  with a gate per key channel, Kimi Delta Attention (section "Kimi Delta
  Attention (KDA)").  Built from
  ``deltanet_oracle.c`` with gcc.
* ``chunkwise`` (module) -- numpy float64 statements of the chunk form, the
  WY transition product, the segment composition and the full-sequence closed
  form, for tiny inputs, and of the gated chunk form ("Complete per-chunk
  algorithm" of the GDN section).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from typing import Optional

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "deltanet_oracle.c")
_LIB_PATH = os.path.join(_HERE, "_build", "libdeltanet_oracle.so")
_lib = None
_lock = threading.Lock()


def build(force: bool = False) -> str:
    """Compile the C oracle with gcc (plain -O2, no fast-math)."""
    os.makedirs(os.path.dirname(_LIB_PATH), exist_ok=True)
    if force or not os.path.exists(_LIB_PATH) or \
            os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            f = lib.delta_oracle_fwd
            f.restype = ctypes.c_int
            f.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
                          ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
                          ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64,
                          ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                          ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                          ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_int]
            _lib = lib
    return _lib


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def token_recurrence(q, k, v, beta, initial_state=None, cu_seqlens=None,
                     heads=None, out_dtype=torch.float64, want_out=True,
                     n_threads: Optional[int] = None, g=None, n_sub: int = 1):
    """Run the float64 token recurrence on CPU tensors.

    q, k: [B, T, H, dk]; v: [B, T, H, dv] (fp32, bf16 or fp64); beta: [B, T, H]
    fp32; initial_state: [N, H, dk, dv] or None; cu_seqlens: int32 [N+1] or None;
    g: [B, T, H] fp32 log decay (Gated DeltaNet), [B, T, H, dk] one log decay per
    key channel (Kimi Delta Attention), or None (plain DeltaNet).
    n_sub > 1: Gated Delta Product with n_sub writes per token; k, v, beta then
    hold [B, T * n_sub, H, .] rows (substep-major within a token) while q, g, out
    and cu_seqlens count tokens.
    ``heads``: (h_begin, h_end) to compute a subset of heads (others are NaN).
    Returns (out [B, T, H, dv] in ``out_dtype`` or None, final_state [N, H, dk, dv]
    float64).
    """
    lib = _load()
    q = q.contiguous(); k = k.contiguous(); v = v.contiguous()
    beta = beta.to(torch.float32).contiguous()
    gate = None if g is None else g.to(torch.float32).contiguous()
    B, T, H, dk = q.shape
    if n_sub < 1 or tuple(k.shape) != (B, T * n_sub, H, dk) or v.shape[:3] != (B, T * n_sub, H) \
            or tuple(beta.shape) != (B, T * n_sub, H):
        raise ValueError("k, v, beta must hold n_sub rows per token of q")
    dv = v.shape[-1]
    codes = {torch.float32: 0, torch.bfloat16: 1, torch.float64: 2}
    if not (q.dtype == k.dtype == v.dtype) or q.dtype not in codes:
        raise TypeError("q, k, v must share one of fp32 / bf16 / fp64")
    cu = None
    n_seq = B
    if cu_seqlens is not None:
        cu = cu_seqlens.to(torch.int32).contiguous()
        n_seq = cu.numel() - 1
    s0 = None if initial_state is None else initial_state.to(torch.float64).contiguous()
    h0, h1 = heads if heads is not None else (0, H)
    out = None
    if want_out:
        if out_dtype not in (torch.float32, torch.float64):
            raise TypeError("out_dtype must be fp32 or fp64")
        out = torch.full((B, T, H, dv), float("nan"), dtype=out_dtype)
    fs = torch.full((n_seq, H, dk, dv), float("nan"), dtype=torch.float64)
    if n_threads is None:
        n_threads = os.cpu_count() or 1
    per_key = gate is not None and gate.dim() == 4
    if gate is not None and tuple(gate.shape) not in ((B, T, H), (B, T, H, dk)):
        raise ValueError("g must hold one value per (token, head) or per key channel")
    rc = lib.delta_oracle_fwd(_ptr(q), _ptr(k), _ptr(v), codes[q.dtype], _ptr(beta),
                              _ptr(gate), int(per_key), _ptr(s0), _ptr(cu), n_seq, B, T, H, dk,
                              dv, int(n_sub), h0, h1, _ptr(out),
                              0 if out_dtype == torch.float32 else 2, _ptr(fs), int(n_threads))
    if rc != 0:
        raise ValueError(f"oracle rejected its arguments (code {rc})")
    return out, fs
