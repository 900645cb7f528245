"""The seeded input generator: deterministic, correctly shaped, normalised."""
import torch

from deltanet_chunkwise_delta_b200 import workloads as wl


def test_varlen_lengths_recipe():
    L = wl.varlen_lengths()
    assert len(L) == 32 and sum(L) == 222459 and min(L) == 129 and max(L) == 32264
    w = wl.WORKLOADS["varlen_32"]
    cu = w.cu_seqlens()
    assert cu[0] == 0 and cu[-1] == 222459 and cu.dtype == torch.int32


def test_generate_is_deterministic_and_normalised():
    w = wl.custom(2, 70, 3, 64, 32, torch.bfloat16, init_state=True)
    a = wl.generate(w, seed=3)
    b = wl.generate(w, seed=3)
    for key in ("q", "k", "v", "beta", "initial_state"):
        assert torch.equal(a[key], b[key])
    assert a["q"].shape == (2, 70, 3, 64) and a["v"].shape == (2, 70, 3, 32)
    assert a["initial_state"].shape == (2, 3, 64, 32)
    n = a["k"].float().norm(dim=-1)
    assert torch.allclose(n, torch.ones_like(n), atol=1e-2)
    assert (a["beta"] > 0).all() and (a["beta"] < 1).all()
    c = wl.generate(w, seed=4)
    assert not torch.equal(a["q"], c["q"])


def test_config_shapes():
    W = wl.WORKLOADS
    assert (W["layer_1p3b"].B, W["layer_1p3b"].T, W["layer_1p3b"].H) == (8, 2048, 16)
    assert (W["long_65k"].T, W["long_65k"].H, W["long_65k"].init_state) == (65536, 16, True)
    assert (W["ctx_1m"].T, W["ctx_1m"].H) == (1 << 20, 8)
    assert W["tiny_fp32"].dtype == torch.float32 and W["tiny_fp32"].dk == 64


def test_gate_recipe():
    """Gated workloads add g = logsigmoid(N(0,1) + 4) after the other draws, so
    their q, k, v, beta and initial state equal the plain workload's."""
    w = wl.custom(1, 4096, 2, 64, 64, torch.bfloat16, init_state=True, gated=True)
    a = wl.generate(w, seed=5)
    b = wl.generate(wl.custom(1, 4096, 2, 64, 64, torch.bfloat16, init_state=True), seed=5)
    for key in ("q", "k", "v", "beta", "initial_state"):
        assert torch.equal(a[key], b[key])
    assert b["g"] is None and a["g"].shape == (1, 4096, 2) and a["g"].dtype == torch.float32
    assert (a["g"] < 0).all()
    med = float(a["g"].exp().median())
    assert 0.97 < med < 0.99
    assert wl.WORKLOADS["gdn_65k"].gated and not wl.WORKLOADS["long_65k"].gated


def test_gdp_recipe():
    """Gated Delta Product workloads draw n_h key/value/beta rows per token."""
    w = wl.custom(2, 100, 3, 64, 32, torch.bfloat16, gated=True, nh=3)
    x = wl.generate(w, seed=6)
    assert x["q"].shape == (2, 100, 3, 64) and x["k"].shape == (2, 300, 3, 64)
    assert x["v"].shape == (2, 300, 3, 32) and x["beta"].shape == (2, 300, 3)
    assert x["g"].shape == (2, 100, 3)
    assert wl.WORKLOADS["gdp_1p3b"].nh == 2
