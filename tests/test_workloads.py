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
