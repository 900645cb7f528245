"""Seeded synthetic inputs for the DeltaNet forward pass.

This module is shared by the CUDA path's callers (tests, bench) and by the
oracle's callers.  It holds no part of the delta-rule arithmetic: it only draws
random tensors, normalises q and k (input preparation, done by the model before
the attention kernel), casts them to the storage dtype and packs variable-length
batches.

Workloads follow the shapes named in "Parallelizing Linear Transformers with the
Delta Rule over Sequence Length" (the 1.3B model's layer shape) and the long /
1M-token contexts of "Context Parallelism for DeltaNet" (section 1, Background).

Recipe (all on the CPU, so every consumer sees bit-identical inputs):
  * one ``torch.Generator('cpu')`` seeded with ``seed``;
  * tensors drawn in the order q, k, v, beta, initial_state;
  * each of q, k, v is drawn in token blocks of ``_BLOCK_TOKENS`` tokens
    (fp32 N(0,1)), so that the 1M-token case never holds a full fp32 copy;
  * q and k are L2-normalised per (token, head) over the key dimension in fp32
    and then cast to the storage dtype (bf16 rounds to nearest-even);
  * beta = sigmoid(N(0,1)) in fp32, shape [B, T, H];
  * initial_state ~ N(0, 0.02) (standard deviation 0.02) in fp32, or zeros;
  * gated workloads (Gated DeltaNet, "Linear Attention, Visualized", section
    "Gated DeltaNet (GDN)") then draw the log decay g = ln a = logsigmoid(z + 4),
    z ~ N(0,1) in fp32, shape [B, T, H]: a has median 0.982 and 5 % below 0.91,
    so a state keeps about a third of itself across one 64-token chunk;
  * Gated Delta Product workloads (same page, section "Gated Delta Product
    (GDP)") draw n_h key, value and beta rows per token (substep-major, i.e.
    k [B, T n_h, H, d]) where the others draw one; q, the initial state and g
    keep one row per token;
  * Kimi Delta Attention workloads (same page, section "Kimi Delta Attention
    (KDA)") draw one log decay per key channel instead, g = logsigmoid(z + 4),
    z ~ N(0,1) in fp32, shape [B, T, H, d_k], after everything else;
  * variable-length batches draw 32 lengths with ``numpy.random.default_rng(seed)``
    log-uniformly in [ln 128, ln 32768], L = floor(exp(u)), packed in draw order.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np
import torch

_BLOCK_TOKENS = 1 << 16


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    T: int                      # tokens per batch row (packed total for varlen)
    H: int
    dk: int
    dv: int
    dtype: torch.dtype          # storage dtype of q, k, v, out
    init_state: bool            # draw a nonzero initial state
    seqlens: Optional[tuple] = None   # varlen: per-sequence lengths (B == 1)
    chunk: int = 64
    gated: bool = False               # Gated DeltaNet: draw the log decay g
    nh: int = 1                       # Gated Delta Product: writes per token (gated)
    kda: bool = False                 # Kimi Delta Attention: a log decay per key channel

    @property
    def n_seq(self) -> int:
        return len(self.seqlens) if self.seqlens is not None else self.B

    @property
    def tokens(self) -> int:
        return self.B * self.T

    def cu_seqlens(self) -> Optional[torch.Tensor]:
        if self.seqlens is None:
            return None
        cu = np.zeros(len(self.seqlens) + 1, dtype=np.int64)
        cu[1:] = np.cumsum(self.seqlens)
        return torch.tensor(cu, dtype=torch.int32)


def varlen_lengths(n: int = 32, lo: int = 128, hi: int = 32768, seed: int = 0) -> tuple:
    rng = np.random.default_rng(seed)
    u = rng.uniform(math.log(lo), math.log(hi), size=n)
    return tuple(int(x) for x in np.floor(np.exp(u)).astype(np.int64))


def _workloads() -> dict:
    vl = varlen_lengths()
    return {
        "tiny_fp32": Workload("tiny_fp32", 1, 256, 2, 64, 64, torch.float32, False),
        "layer_1p3b": Workload("layer_1p3b", 8, 2048, 16, 128, 128, torch.bfloat16, False),
        "long_65k": Workload("long_65k", 1, 65536, 16, 128, 128, torch.bfloat16, True),
        "ctx_1m": Workload("ctx_1m", 1, 1 << 20, 8, 128, 128, torch.bfloat16, False),
        # the first 131,072 tokens of the 1M-token context: the same kernels at one eighth of
        # the size, small enough for a profiler capture
        "ctx_128k": Workload("ctx_128k", 1, 1 << 17, 8, 128, 128, torch.bfloat16, False),
        "varlen_32": Workload("varlen_32", 1, sum(vl), 16, 128, 128, torch.bfloat16, True, vl),
        "gdn_1p3b": Workload("gdn_1p3b", 8, 2048, 16, 128, 128, torch.bfloat16, False, gated=True),
        "gdn_65k": Workload("gdn_65k", 1, 65536, 16, 128, 128, torch.bfloat16, True, gated=True),
        "gdp_1p3b": Workload("gdp_1p3b", 8, 2048, 16, 128, 128, torch.bfloat16, False,
                             gated=True, nh=2),
        "kda_1p3b": Workload("kda_1p3b", 8, 2048, 16, 128, 128, torch.bfloat16, False, kda=True),
    }


WORKLOADS = _workloads()


def custom(B, T, H, dk, dv, dtype=torch.bfloat16, init_state=False, seqlens=None,
           name="custom", gated=False, nh=1, kda=False) -> Workload:
    if seqlens is not None:
        seqlens = tuple(int(x) for x in seqlens)
        B, T = 1, sum(seqlens)
    if nh > 1 and not gated:
        raise ValueError("several writes per token is the gated product")
    if kda and gated:
        raise ValueError("one kind of gate")
    return Workload(name, B, T, H, dk, dv, dtype, init_state, seqlens, gated=gated, nh=nh, kda=kda)


def _draw_tokens(gen, B, T, H, d, dtype, normalise):
    out = torch.empty((B, T, H, d), dtype=dtype)
    for b in range(B):
        for t0 in range(0, T, _BLOCK_TOKENS):
            t1 = min(T, t0 + _BLOCK_TOKENS)
            x = torch.randn((t1 - t0, H, d), generator=gen, dtype=torch.float32)
            if normalise:
                x = x / x.norm(dim=-1, keepdim=True).clamp_min(1e-12)
            out[b, t0:t1] = x.to(dtype)
    return out


def generate(w: Workload, seed: int = 0, beta_mode: str = "sigmoid") -> dict:
    """Draw the inputs of workload ``w`` on the CPU.

    ``beta_mode``: "sigmoid" (the workloads' recipe), "zero" or "one"
    (special cases of the update's step size, drawn after the same stream).
    """
    gen = torch.Generator("cpu")
    gen.manual_seed(seed)
    Tw = w.T * w.nh                   # rows of k, v, beta
    q = _draw_tokens(gen, w.B, w.T, w.H, w.dk, w.dtype, True)
    k = _draw_tokens(gen, w.B, Tw, w.H, w.dk, w.dtype, True)
    v = _draw_tokens(gen, w.B, Tw, w.H, w.dv, w.dtype, False)
    beta = torch.sigmoid(torch.randn((w.B, Tw, w.H), generator=gen, dtype=torch.float32))
    if beta_mode == "zero":
        beta = torch.zeros_like(beta)
    elif beta_mode == "one":
        beta = torch.ones_like(beta)
    elif beta_mode != "sigmoid":
        raise ValueError(beta_mode)
    n = w.n_seq
    if w.init_state:
        s0 = torch.randn((n, w.H, w.dk, w.dv), generator=gen, dtype=torch.float32) * 0.02
    else:
        s0 = None
    g = None
    if w.gated:
        z = torch.randn((w.B, w.T, w.H), generator=gen, dtype=torch.float32)
        g = torch.nn.functional.logsigmoid(z + 4.0)
    elif w.kda:
        z = torch.randn((w.B, w.T, w.H, w.dk), generator=gen, dtype=torch.float32)
        g = torch.nn.functional.logsigmoid(z + 4.0)
    return {"q": q, "k": k, "v": v, "beta": beta, "initial_state": s0,
            "cu_seqlens": w.cu_seqlens(), "g": g}
