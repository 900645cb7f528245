"""GPU parity: the CUDA path (through the C ABI) against the float64 oracle on
the same seeded inputs.

Bar (max-normalised error, on both out and final_state):
    max|x_gpu - x_ref| / max|x_ref| <= 1e-2 for bf16 inputs, 1e-4 for fp32.
"""
import os

import numpy as np
import pytest
import torch

import oracle
import deltanet_chunkwise_delta_b200 as dn
from deltanet_chunkwise_delta_b200 import workloads as wl

pytestmark = pytest.mark.gpu

TOL = {torch.bfloat16: 1e-2, torch.float32: 1e-4}
DEV = torch.device("cuda:0")


def rel_err(x, ref):
    x = x.double().cpu()
    ref = ref.double().cpu()
    m = ref.abs().max().item()
    return (x - ref).abs().max().item() / (m if m > 0 else 1.0)


def to_dev(x):
    return {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in x.items()}


def run_gpu(x, seg_chunks=0, with_state=True):
    g = to_dev(x)
    out, fs = dn.deltanet_fwd(g["q"], g["k"], g["v"], g["beta"], g["initial_state"],
                              g["cu_seqlens"], output_final_state=with_state,
                              seg_chunks=seg_chunks)
    assert dn.get_error() == 0
    return out.cpu(), (fs.cpu() if fs is not None else None)


def check(w, x, seg_chunks=0, heads=None, log=None, name=None):
    out, fs = run_gpu(x, seg_chunks)
    ref_o, ref_s = oracle.token_recurrence(x["q"], x["k"], x["v"], x["beta"],
                                           x["initial_state"], x["cu_seqlens"], heads=heads)
    h0, h1 = heads if heads else (0, w.H)
    eo = rel_err(out[:, :, h0:h1], ref_o[:, :, h0:h1])
    es = rel_err(fs[:, h0:h1], ref_s[:, h0:h1])
    tol = TOL[w.dtype]
    if log is not None:
        log.append((name or w.name, eo, es, tol))
    assert eo <= tol and es <= tol, (eo, es)
    return eo, es


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dn.load()


def test_tiny_fp32_config(margins):
    w = wl.WORKLOADS["tiny_fp32"]
    check(w, wl.generate(w, 0), log=margins)


@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 64), (128, 64), (64, 128)])
@pytest.mark.parametrize("T", [1, 63, 64, 200, 333])
def test_bf16_shapes_and_ragged_tails(dk, dv, T):
    w = wl.custom(2, T, 3, dk, dv, torch.bfloat16, init_state=True)
    check(w, wl.generate(w, seed=T + dk))


@pytest.mark.parametrize("seg", [1, 2, 3, 5])
def test_forced_segmentation_is_exact(seg):
    """Any split of the chunk chain into runs gives the serial result."""
    w = wl.custom(1, 64 * 13 - 5, 2, 128, 128, torch.bfloat16, init_state=True)
    x = wl.generate(w, seed=7)
    e_seg = check(w, x, seg_chunks=seg)
    e_one = check(w, x, seg_chunks=1000)
    assert max(e_seg) <= 1e-2 and max(e_one) <= 1e-2


@pytest.mark.parametrize("first", [1, 3])
def test_split_with_a_shorter_first_run(first):
    """Run 0 (on the tensor-core path computed by the boundary kernel next to the
    summary items) may be shorter than the other runs, which the schedule uses
    when a summary chunk is cheaper than a boundary chunk; the result equals the
    serial pass."""
    w = wl.custom(2, 64 * 13 - 5, 1, 128, 128, torch.bfloat16, init_state=True)
    x = wl.generate(w, seed=16)
    check(w, x, seg_chunks=5 | (first << 16))
    G, s, s0 = dn.last_schedule(with_first=True)
    assert (G, s, s0) == (1 + (13 - first + 4) // 5, 5, first), (G, s, s0)


def test_segmentation_short_memory_case():
    """Short runs (1 chunk) with a slowly forgetting state: beta small so the
    transition products stay far from zero and the composition matters."""
    w = wl.custom(1, 64 * 9, 2, 64, 64, torch.bfloat16, init_state=True)
    x = wl.generate(w, seed=8)
    x["beta"] = x["beta"] * 0.05
    check(w, x, seg_chunks=1)


@pytest.mark.parametrize("mode", ["zero", "one"])
def test_beta_special_cases(mode):
    w = wl.custom(2, 150, 2, 128, 128, torch.bfloat16, init_state=True)
    x = wl.generate(w, seed=9, beta_mode=mode)
    check(w, x, seg_chunks=1)
    if mode == "zero":
        _, fs = run_gpu(x)
        assert torch.equal(fs, x["initial_state"])


def test_fp32_small_segments():
    w = wl.custom(2, 64 * 5 + 7, 2, 64, 64, torch.float32, init_state=True)
    x = wl.generate(w, seed=10)
    check(w, x, seg_chunks=2)


@pytest.mark.parametrize("seg", [0, 1, 3])
def test_varlen_with_empty_and_tiny_sequences(seg):
    lens = [0, 1, 64, 200, 0, 129, 700, 63]
    w = wl.custom(1, 0, 2, 128, 128, torch.bfloat16, init_state=True, seqlens=lens)
    x = wl.generate(w, seed=11)
    check(w, x, seg_chunks=seg)


def test_varlen_zero_length_keeps_initial_state():
    lens = [0, 5, 0]
    w = wl.custom(1, 0, 1, 64, 64, torch.bfloat16, init_state=True, seqlens=lens)
    x = wl.generate(w, seed=12)
    _, fs = run_gpu(x)
    assert torch.equal(fs[0], x["initial_state"][0])
    assert torch.equal(fs[2], x["initial_state"][2])


def test_chained_calls_equal_one_call():
    """Splitting a sequence at a chunk boundary into two calls chained through
    final_state -> initial_state equals one call (the state carries the whole
    history)."""
    w = wl.custom(1, 64 * 8, 2, 128, 128, torch.bfloat16, init_state=True)
    x = wl.generate(w, seed=13)
    g = to_dev(x)
    one = 1000   # no split: both ways run the same chunk steps in the same order
    o_full, s_full = dn.deltanet_fwd(g["q"], g["k"], g["v"], g["beta"], g["initial_state"],
                                     seg_chunks=one)
    c = 64 * 3
    sl = lambda t, a, b: t[:, a:b].contiguous()
    o1, s1 = dn.deltanet_fwd(sl(g["q"], 0, c), sl(g["k"], 0, c), sl(g["v"], 0, c),
                             sl(g["beta"], 0, c), g["initial_state"], seg_chunks=one)
    o2, s2 = dn.deltanet_fwd(sl(g["q"], c, None), sl(g["k"], c, None), sl(g["v"], c, None),
                             sl(g["beta"], c, None), s1, seg_chunks=one)
    assert torch.equal(torch.cat([o1, o2], 1), o_full)
    assert torch.equal(s2, s_full)


def test_strided_inputs():
    """Non-contiguous views (head-major storage) give the same result."""
    w = wl.custom(2, 130, 3, 128, 128, torch.bfloat16, init_state=True)
    x = wl.generate(w, seed=14)
    g = to_dev(x)
    o_ref, s_ref = dn.deltanet_fwd(g["q"], g["k"], g["v"], g["beta"], g["initial_state"])
    perm = lambda t: t.permute(0, 2, 1, 3).contiguous().permute(0, 2, 1, 3)
    o, s = dn.deltanet_fwd(perm(g["q"]), perm(g["k"]), perm(g["v"]),
                           g["beta"].permute(0, 2, 1).contiguous().permute(0, 2, 1),
                           g["initial_state"])
    assert torch.equal(o, o_ref) and torch.equal(s, s_ref)


def test_bad_cu_seqlens_reported_on_device():
    w = wl.custom(1, 100, 1, 64, 64, torch.bfloat16)
    x = wl.generate(w, seed=15)
    g = to_dev(x)
    cu = torch.tensor([0, 60, 40, 100], dtype=torch.int32, device=DEV)
    dn.deltanet_fwd(g["q"], g["k"], g["v"], g["beta"], None, cu)
    assert dn.get_error() == 6      # DN_ERR_SEQLENS
    assert dn.get_error() == 0      # cleared once read
    cu = torch.tensor([0, 60, 90], dtype=torch.int32, device=DEV)   # does not end at T
    dn.deltanet_fwd(g["q"], g["k"], g["v"], g["beta"], None, cu)
    assert dn.get_error() == 6


def test_schedule_of_config_shapes():
    """The automatic split uses every SM for the long single sequences and
    none for the many-chain layer shape."""
    q = torch.zeros((8, 2048, 16, 128), dtype=torch.bfloat16, device=DEV)
    v = torch.zeros_like(q)
    b = torch.zeros((8, 2048, 16), device=DEV)
    dn.deltanet_fwd(q, q, v, b)
    assert dn.last_schedule()[0] == 1
    q = torch.zeros((1, 65536, 16, 128), dtype=torch.bfloat16, device=DEV)
    b = torch.zeros((1, 65536, 16), device=DEV)
    dn.deltanet_fwd(q, q, torch.zeros_like(q), b)
    G, s, s0 = dn.last_schedule(with_first=True)
    assert G >= 4 and s0 + (G - 1) * s >= 1024 and 1 <= s0 <= s


# ---- full-size configs: every output of a subset of heads ------------------

@pytest.mark.slow
def test_config_layer_1p3b(margins):
    w = wl.WORKLOADS["layer_1p3b"]
    check(w, wl.generate(w, 0), heads=(0, 4), log=margins, name="layer_1p3b (heads 0-3)")


@pytest.mark.slow
def test_config_long_65k(margins):
    w = wl.WORKLOADS["long_65k"]
    check(w, wl.generate(w, 0), heads=(0, 2), log=margins, name="long_65k (heads 0-1)")


@pytest.mark.slow
def test_config_varlen_32(margins):
    w = wl.WORKLOADS["varlen_32"]
    check(w, wl.generate(w, 0), heads=(0, 2), log=margins, name="varlen_32 (heads 0-1)")


@pytest.mark.slow
def test_config_ctx_1m(margins):
    w = wl.WORKLOADS["ctx_1m"]
    x = wl.generate(w, 0)
    out, fs = run_gpu(x)
    ref_o, ref_s = oracle.token_recurrence(x["q"], x["k"], x["v"], x["beta"], None,
                                           heads=(0, 1), out_dtype=torch.float32)
    eo = rel_err(out[:, :, 0:1], ref_o[:, :, 0:1])
    es = rel_err(fs[:, 0:1], ref_s[:, 0:1])
    margins.append(("ctx_1m (head 0, 1048576 tokens)", eo, es, 1e-2))
    assert eo <= 1e-2 and es <= 1e-2, (eo, es)
