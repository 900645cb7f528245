"""GPU parity of the Gated Delta Product ("Linear Attention, Visualized",
section "Gated Delta Product (GDP)"): gated_deltaproduct_fwd against the
float64 oracle's substep recurrence (decay once per token, n_h writes, then the
readout) on the same seeded inputs.  Bar as for DeltaNet: 1e-2 (bf16), 1e-4
(fp32) on max-normalised out and final_state.
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


def run_gpu(w, x, seg_chunks=0):
    g = to_dev(x)
    out, fs = dn.gated_deltaproduct_fwd(g["q"], g["k"], g["v"], g["beta"], g["g"], w.nh,
                                        g["initial_state"], g["cu_seqlens"],
                                        seg_chunks=seg_chunks)
    assert dn.get_error() == 0
    return out.cpu(), fs.cpu()


def check(w, x, seg_chunks=0, heads=None):
    out, fs = run_gpu(w, x, seg_chunks)
    ref_o, ref_s = oracle.token_recurrence(x["q"], x["k"], x["v"], x["beta"],
                                           x["initial_state"], x["cu_seqlens"], heads=heads,
                                           g=x["g"], n_sub=w.nh)
    h0, h1 = heads if heads else (0, w.H)
    eo = rel_err(out[:, :, h0:h1], ref_o[:, :, h0:h1])
    es = rel_err(fs[:, h0:h1], ref_s[:, h0:h1])
    tol = TOL[w.dtype]
    assert eo <= tol and es <= tol, (eo, es)


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dn.load()


@pytest.mark.parametrize("nh", [1, 2, 3])
@pytest.mark.parametrize("T", [1, 31, 64, 100])
def test_gdp_shapes_and_ragged_tails(nh, T):
    w = wl.custom(2, T, 3, 128, 128, torch.bfloat16, init_state=True, gated=True, nh=nh)
    check(w, wl.generate(w, seed=40 + T + nh))


@pytest.mark.parametrize("dk,dv,dtype", [(64, 64, torch.bfloat16), (128, 64, torch.bfloat16),
                                         (64, 64, torch.float32)])
def test_gdp_other_head_sizes(dk, dv, dtype):
    w = wl.custom(2, 90, 2, dk, dv, dtype, init_state=True, gated=True, nh=2)
    check(w, wl.generate(w, seed=41 + dk + dv))


@pytest.mark.parametrize("seg", [1, 3])
def test_gdp_forced_segmentation_is_exact(seg):
    """Runs of the virtual sequence may end inside a token's writes: the
    segment maps compose exactly all the same."""
    w = wl.custom(1, 64 * 5 - 7, 2, 128, 128, torch.bfloat16, init_state=True, gated=True, nh=3)
    check(w, wl.generate(w, seed=42), seg_chunks=seg)


@pytest.mark.parametrize("seg", [0, 1])
def test_gdp_varlen(seg):
    lens = [0, 1, 33, 100, 0, 65]
    w = wl.custom(1, 0, 2, 128, 128, torch.bfloat16, init_state=True, seqlens=lens, gated=True,
                  nh=3)
    check(w, wl.generate(w, seed=43), seg_chunks=seg)


def test_one_write_per_token_is_gdn():
    """n_h = 1 runs the same kernels as gated_deltanet_fwd: bit-identical."""
    w = wl.custom(2, 150, 2, 128, 128, torch.bfloat16, init_state=True, gated=True)
    x = wl.generate(w, seed=44)
    g = to_dev(x)
    o1, s1 = dn.gated_deltaproduct_fwd(g["q"], g["k"], g["v"], g["beta"], g["g"], 1,
                                       g["initial_state"])
    o2, s2 = dn.gated_deltanet_fwd(g["q"], g["k"], g["v"], g["beta"], g["g"], g["initial_state"])
    assert torch.equal(o1, o2) and torch.equal(s1, s2)


@pytest.mark.slow
def test_config_gdp_1p3b():
    w = wl.WORKLOADS["gdp_1p3b"]
    check(w, wl.generate(w, 0), heads=(0, 2))
