"""GPU parity of Gated DeltaNet ("Linear Attention, Visualized", section "Gated
DeltaNet (GDN)"): the CUDA path through gated_deltanet_fwd against the float64
oracle's gated token recurrence on the same seeded inputs.

Bar as for DeltaNet (max-normalised error on out and final_state): 1e-2 for
bf16 inputs, 1e-4 for fp32.
"""
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


def run_gpu(x, seg_chunks=0):
    g = to_dev(x)
    out, fs = dn.gated_deltanet_fwd(g["q"], g["k"], g["v"], g["beta"], g["g"],
                                    g["initial_state"], g["cu_seqlens"], seg_chunks=seg_chunks)
    assert dn.get_error() == 0
    return out.cpu(), fs.cpu()


def check(w, x, seg_chunks=0, heads=None, log=None, name=None):
    out, fs = run_gpu(x, seg_chunks)
    ref_o, ref_s = oracle.token_recurrence(x["q"], x["k"], x["v"], x["beta"],
                                           x["initial_state"], x["cu_seqlens"], heads=heads,
                                           g=x["g"])
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


@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 64), (128, 64), (64, 128)])
@pytest.mark.parametrize("T", [1, 63, 64, 200, 333])
def test_gated_bf16_shapes_and_ragged_tails(dk, dv, T):
    w = wl.custom(2, T, 3, dk, dv, torch.bfloat16, init_state=True, gated=True)
    check(w, wl.generate(w, seed=T + dk + 1))


def test_gated_fp32():
    w = wl.custom(2, 64 * 5 + 7, 2, 64, 64, torch.float32, init_state=True, gated=True)
    x = wl.generate(w, seed=20)
    check(w, x)
    check(w, x, seg_chunks=2)


@pytest.mark.parametrize("seg", [1, 2, 3, 5])
def test_gated_forced_segmentation_is_exact(seg):
    """The gated segment maps compose exactly: any split gives the serial result."""
    w = wl.custom(1, 64 * 13 - 5, 2, 128, 128, torch.bfloat16, init_state=True, gated=True)
    x = wl.generate(w, seed=21)
    check(w, x, seg_chunks=seg)
    check(w, x, seg_chunks=1000)


def test_gated_strong_decay():
    """Per-token decays down to e^-4: chunk products far below fp32's normal range
    are formed as exponentials of running-sum differences, never as ratios."""
    w = wl.custom(1, 64 * 6 + 9, 2, 128, 128, torch.bfloat16, init_state=True, gated=True)
    x = wl.generate(w, seed=22)
    gen = torch.Generator().manual_seed(22)
    x["g"] = -4.0 * torch.rand(x["g"].shape, generator=gen)
    check(w, x)
    check(w, x, seg_chunks=2)


def test_unit_gates_match_deltanet_oracle():
    """g = 0 (a = 1) is plain DeltaNet."""
    w = wl.custom(2, 150, 2, 128, 128, torch.bfloat16, init_state=True, gated=True)
    x = wl.generate(w, seed=23)
    x["g"] = torch.zeros_like(x["g"])
    out, fs = run_gpu(x)
    ref_o, ref_s = oracle.token_recurrence(x["q"], x["k"], x["v"], x["beta"],
                                           x["initial_state"])
    assert rel_err(out, ref_o) <= 1e-2 and rel_err(fs, ref_s) <= 1e-2


def test_gated_zero_beta_is_pure_decay():
    """beta = 0: the final state is the initial state times exp(sum of g)."""
    w = wl.custom(2, 130, 2, 64, 64, torch.bfloat16, init_state=True, gated=True)
    x = wl.generate(w, seed=24, beta_mode="zero")
    check(w, x, seg_chunks=1)
    _, fs = run_gpu(x)
    decay = torch.exp(x["g"].double().sum(dim=1))            # [B, H]
    ref = x["initial_state"].double() * decay[:, :, None, None]
    assert rel_err(fs, ref) <= 1e-5


@pytest.mark.parametrize("seg", [0, 1, 3])
def test_gated_varlen_with_empty_and_tiny_sequences(seg):
    lens = [0, 1, 64, 200, 0, 129, 700, 63]
    w = wl.custom(1, 0, 2, 128, 128, torch.bfloat16, init_state=True, seqlens=lens, gated=True)
    x = wl.generate(w, seed=25)
    check(w, x, seg_chunks=seg)


def test_gated_chained_calls_equal_one_call():
    """Two calls chained through final_state -> initial_state at a chunk boundary
    equal one call: the state carries the decayed history."""
    w = wl.custom(1, 64 * 8, 2, 128, 128, torch.bfloat16, init_state=True, gated=True)
    x = wl.generate(w, seed=26)
    g = to_dev(x)
    one = 1000
    o_full, s_full = dn.gated_deltanet_fwd(g["q"], g["k"], g["v"], g["beta"], g["g"],
                                           g["initial_state"], seg_chunks=one)
    c = 64 * 3
    sl = lambda t, a, b: t[:, a:b].contiguous()
    o1, s1 = dn.gated_deltanet_fwd(sl(g["q"], 0, c), sl(g["k"], 0, c), sl(g["v"], 0, c),
                                   sl(g["beta"], 0, c), sl(g["g"], 0, c), g["initial_state"],
                                   seg_chunks=one)
    o2, s2 = dn.gated_deltanet_fwd(sl(g["q"], c, None), sl(g["k"], c, None),
                                   sl(g["v"], c, None), sl(g["beta"], c, None),
                                   sl(g["g"], c, None), s1, seg_chunks=one)
    assert torch.equal(torch.cat([o1, o2], 1), o_full)
    assert torch.equal(s2, s_full)


def test_gated_strided_gate():
    """A head-major (non-contiguous) gate view gives the same result."""
    w = wl.custom(2, 130, 3, 128, 128, torch.bfloat16, init_state=True, gated=True)
    x = wl.generate(w, seed=27)
    g = to_dev(x)
    o_ref, s_ref = dn.gated_deltanet_fwd(g["q"], g["k"], g["v"], g["beta"], g["g"],
                                         g["initial_state"])
    gt = g["g"].permute(0, 2, 1).contiguous().permute(0, 2, 1)
    o, s = dn.gated_deltanet_fwd(g["q"], g["k"], g["v"], g["beta"], gt, g["initial_state"])
    assert torch.equal(o, o_ref) and torch.equal(s, s_ref)


# ---- full-size gated workloads: every output of a subset of heads ---------------

@pytest.mark.slow
def test_config_gdn_1p3b(margins):
    w = wl.WORKLOADS["gdn_1p3b"]
    check(w, wl.generate(w, 0), heads=(0, 4), log=margins, name="gdn_1p3b (heads 0-3)")


@pytest.mark.slow
def test_config_gdn_65k(margins):
    w = wl.WORKLOADS["gdn_65k"]
    check(w, wl.generate(w, 0), heads=(0, 2), log=margins, name="gdn_65k (heads 0-1)")
