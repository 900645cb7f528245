"""GPU parity of Kimi Delta Attention ("Linear Attention, Visualized", section
"Kimi Delta Attention (KDA)"): kda_fwd through the C ABI, on the tensor-core path
(d_k = d_v = 128, chains not split) and on the mma.sync chain kernels, against the
float64 oracle (a decay per key channel, S_t = (I - beta k^T k) Diag(a_t) S_{t-1} +
beta k^T v, o_t = q_t S_t) on the same seeded inputs.

Bar: max|x - x_ref| / max|x_ref| <= 1e-2 (bf16 inputs) on out and final_state.
"""
import pytest
import torch

import oracle
import deltanet_chunkwise_delta_b200 as dn
from deltanet_chunkwise_delta_b200 import workloads as wl

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")
TOL = 1e-2


def rel_err(x, ref):
    x, ref = x.double().cpu(), ref.double().cpu()
    m = ref.abs().max().item()
    return (x - ref).abs().max().item() / (m if m > 0 else 1.0)


def to_dev(x):
    return {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in x.items()}


def run_gpu(x, seg_chunks=0):
    g = to_dev(x)
    out, fs = dn.kda_fwd(g["q"], g["k"], g["v"], g["beta"], g["g"], g["initial_state"],
                         g["cu_seqlens"], seg_chunks=seg_chunks)
    assert dn.get_error() == 0
    return out.cpu(), fs.cpu()


def check(w, x, seg_chunks=0, heads=None, log=None, name=None):
    out, fs = run_gpu(x, seg_chunks)
    ref_o, ref_s = oracle.token_recurrence(x["q"], x["k"], x["v"], x["beta"], x["initial_state"],
                                           x["cu_seqlens"], heads=heads, g=x["g"])
    h0, h1 = heads if heads else (0, w.H)
    eo = rel_err(out[:, :, h0:h1], ref_o[:, :, h0:h1])
    es = rel_err(fs[:, h0:h1], ref_s[:, h0:h1])
    if log is not None:
        log.append((name or w.name, eo, es, TOL))
    assert eo <= TOL and es <= TOL, (eo, es)
    return eo, es


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dn.load()


@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 64), (128, 64), (64, 128)])
@pytest.mark.parametrize("T", [1, 63, 200, 333])
def test_kda_shapes_and_ragged_tails(dk, dv, T):
    w = wl.custom(2, T, 2, dk, dv, torch.bfloat16, init_state=True, kda=True)
    check(w, wl.generate(w, seed=T + dk + 3))


@pytest.mark.parametrize("seg", [1, 2, 3])
def test_kda_forced_segmentation(seg):
    """Runs composed through the segment maps (H_g, and P_g = the product of the
    channel-decayed transitions) equal the serial pass."""
    w = wl.custom(1, 64 * 9 - 7, 2, 128, 128, torch.bfloat16, init_state=True, kda=True)
    x = wl.generate(w, seed=70)
    check(w, x, seg_chunks=seg)


def test_kda_strong_channel_decays():
    """Log decays spread over [-2, 0] per channel (a state row keeps as little as
    e^-128 of itself across a chunk), so the within-chunk decay ratios matter."""
    w = wl.custom(2, 200, 2, 128, 128, torch.bfloat16, init_state=True, kda=True)
    x = wl.generate(w, seed=71)
    gen = torch.Generator().manual_seed(72)
    x["g"] = -2.0 * torch.rand(x["g"].shape, generator=gen)
    check(w, x, seg_chunks=2)


@pytest.mark.parametrize("seg", [0, 1])
def test_kda_packed_with_empty_and_tiny_sequences(seg):
    lens = [0, 1, 64, 200, 0, 129, 700, 63]
    w = wl.custom(1, 0, 2, 128, 128, torch.bfloat16, init_state=True, seqlens=lens, kda=True)
    check(w, wl.generate(w, seed=73), seg_chunks=seg)


def test_kda_equal_channel_gates_match_gated_deltanet():
    """One decay for every channel of a head is Gated DeltaNet: both entry points
    agree within the bar, and both match the oracle."""
    w = wl.custom(2, 150, 2, 128, 128, torch.bfloat16, init_state=True, gated=True)
    x = wl.generate(w, seed=74)
    g = to_dev(x)
    o_gdn, s_gdn = dn.gated_deltanet_fwd(g["q"], g["k"], g["v"], g["beta"], g["g"], g["initial_state"])
    gk = g["g"].unsqueeze(-1).expand(-1, -1, -1, 128).contiguous()
    o_kda, s_kda = dn.kda_fwd(g["q"], g["k"], g["v"], g["beta"], gk, g["initial_state"])
    assert dn.get_error() == 0
    assert rel_err(o_kda, o_gdn) <= TOL and rel_err(s_kda, s_gdn) <= TOL
    ref_o, ref_s = oracle.token_recurrence(x["q"], x["k"], x["v"], x["beta"], x["initial_state"],
                                           g=x["g"])
    assert rel_err(o_kda, ref_o) <= TOL and rel_err(s_kda, ref_s) <= TOL


def test_kda_beta_zero_is_pure_channel_decay():
    """beta = 0: no writes, every state row decays by the product of its channel's
    gates; out reads the decayed state."""
    w = wl.custom(1, 100, 2, 64, 64, torch.bfloat16, init_state=True, kda=True)
    x = wl.generate(w, seed=75, beta_mode="zero")
    out, fs = run_gpu(x)
    decay = torch.exp(x["g"][0].sum(0))  # [H, d_k]
    expect = x["initial_state"][0] * decay[:, :, None]
    assert rel_err(fs[0], expect) <= 1e-4
    check(w, x)


def test_kda_chained_calls_equal_one_call():
    """Two calls chained through the state equal one call bit for bit when both
    run the same chunk steps (no split)."""
    w = wl.custom(1, 64 * 6, 2, 128, 128, torch.bfloat16, init_state=True, kda=True)
    x = wl.generate(w, seed=76)
    g = to_dev(x)
    one = 1000
    o_full, s_full = dn.kda_fwd(g["q"], g["k"], g["v"], g["beta"], g["g"], g["initial_state"],
                                seg_chunks=one)
    c = 64 * 2
    sl = lambda t, a, b: t[:, a:b].contiguous()
    o1, s1 = dn.kda_fwd(sl(g["q"], 0, c), sl(g["k"], 0, c), sl(g["v"], 0, c), sl(g["beta"], 0, c),
                        sl(g["g"], 0, c), g["initial_state"], seg_chunks=one)
    o2, s2 = dn.kda_fwd(sl(g["q"], c, None), sl(g["k"], c, None), sl(g["v"], c, None),
                        sl(g["beta"], c, None), sl(g["g"], c, None), s1, seg_chunks=one)
    assert torch.equal(torch.cat([o1, o2], 1), o_full)
    assert torch.equal(s2, s_full)


# One run per chain (seg_chunks past the chain length): d_k = d_v = 128 then runs on the
# tensor-core path, its pre-pass and boundary kernel (two launches), instead of the
# mma.sync chain kernel (one launch).
ONE_RUN = 1 << 14


@pytest.mark.parametrize("T", [1, 63, 64, 200, 333])
def test_kda_tensor_core_path_shapes(T):
    w = wl.custom(2, T, 3, 128, 128, torch.bfloat16, init_state=True, kda=True)
    x = wl.generate(w, seed=80 + T)
    check(w, x, seg_chunks=ONE_RUN)
    assert dn.last_launches() == 2


def test_kda_tensor_core_path_strong_decays_no_initial_state():
    """Log decays down to -2 per channel and token, no initial state: the channel-decayed
    Gram blocks, K<-, K-> and the per-channel state decay of the tensor-core path."""
    w = wl.custom(2, 300, 2, 128, 128, torch.bfloat16, init_state=False, kda=True)
    x = wl.generate(w, seed=90)
    gen = torch.Generator().manual_seed(91)
    x["g"] = -2.0 * torch.rand(x["g"].shape, generator=gen)
    check(w, x, seg_chunks=ONE_RUN)
    assert dn.last_launches() == 2


def test_kda_tensor_core_path_equals_gdn_on_equal_channel_gates():
    """Equal gates on every channel: the KDA tensor-core path and Gated DeltaNet's agree
    within the bar."""
    w = wl.custom(2, 200, 2, 128, 128, torch.bfloat16, init_state=True, gated=True)
    x = wl.generate(w, seed=92)
    g = to_dev(x)
    o_gdn, s_gdn = dn.gated_deltanet_fwd(g["q"], g["k"], g["v"], g["beta"], g["g"], g["initial_state"])
    gk = g["g"].unsqueeze(-1).expand(-1, -1, -1, 128).contiguous()
    o_kda, s_kda = dn.kda_fwd(g["q"], g["k"], g["v"], g["beta"], gk, g["initial_state"], seg_chunks=ONE_RUN)
    assert dn.get_error() == 0
    assert rel_err(o_kda, o_gdn) <= TOL and rel_err(s_kda, s_gdn) <= TOL


@pytest.mark.slow
def test_config_kda_1p3b(margins):
    w = wl.WORKLOADS["kda_1p3b"]
    check(w, wl.generate(w, 0), heads=(0, 2), log=margins, name="kda_1p3b (heads 0-1)")
    assert dn.last_launches() == 2  # unsplit chains: the tensor-core pre-pass and boundary kernel
