"""GPU parity of the chunk-boundary states (the state entering every chunk,
which a backward pass reuses; "Linear Attention, Visualized", section
"Chunkwise algorithm"): deltanet_fwd_states against the float64 oracle run on
each chunk-aligned prefix, for DeltaNet and Gated DeltaNet, dense and packed,
with and without a split of the chains.  Bar: 1e-2 (bf16) on max-normalised
states, outputs and final states.
"""
import pytest
import torch

import oracle
import deltanet_chunkwise_delta_b200 as dn
from deltanet_chunkwise_delta_b200 import workloads as wl

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda:0")
C = 64


def rel_err(x, ref):
    x = x.double().cpu()
    ref = ref.double().cpu()
    m = ref.abs().max().item()
    return (x - ref).abs().max().item() / (m if m > 0 else 1.0)


def to_dev(x):
    return {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in x.items()}


def prefix_state(x, b, a, L, n, gated):
    """Oracle state of sequence n (batch row b, tokens a .. a+L-1 of that row)."""
    sl = lambda t: t[b:b + 1, a:a + L].contiguous()
    s0 = None if x["initial_state"] is None else x["initial_state"][n:n + 1]
    _, fs = oracle.token_recurrence(sl(x["q"]), sl(x["k"]), sl(x["v"]), sl(x["beta"]), s0,
                                    want_out=False, g=sl(x["g"]) if gated else None)
    return fs[0]


def expected_states(w, x, gated):
    """[rows, H, d_k, d_v]: row = global chunk index, chunks numbered per sequence in
    input order; the state before each chunk's tokens."""
    if w.seqlens is None:
        seqs = [(b, 0, w.T, b) for b in range(w.B)]
    else:
        cu = w.cu_seqlens().tolist()
        seqs = [(0, cu[n], cu[n + 1] - cu[n], n) for n in range(w.n_seq)]
    rows = []
    for b, a, L, n in seqs:
        for r in range((L + C - 1) // C):
            rows.append(prefix_state(x, b, a, r * C, n, gated))
    return torch.stack(rows)


def check(w, x, gated, seg_chunks=0):
    g = to_dev(x)
    out, fs, cs = dn.deltanet_fwd_states(g["q"], g["k"], g["v"], g["beta"],
                                         g["g"] if gated else None, g["initial_state"],
                                         g["cu_seqlens"], seg_chunks=seg_chunks)
    assert dn.get_error() == 0
    ref = expected_states(w, x, gated)
    assert rel_err(cs[:ref.shape[0]], ref) <= 1e-2
    assert torch.count_nonzero(cs[ref.shape[0]:]) == 0     # rows past the total untouched
    ref_o, ref_s = oracle.token_recurrence(x["q"], x["k"], x["v"], x["beta"],
                                           x["initial_state"], x["cu_seqlens"],
                                           g=x["g"] if gated else None)
    assert rel_err(out, ref_o) <= 1e-2 and rel_err(fs, ref_s) <= 1e-2
    return cs


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dn.load()


@pytest.mark.parametrize("gated", [False, True])
@pytest.mark.parametrize("seg", [0, 2])
def test_states_dense(gated, seg):
    w = wl.custom(2, 333, 2, 128, 128, torch.bfloat16, init_state=True, gated=True)
    x = wl.generate(w, seed=60)
    cs = check(w, x, gated, seg)
    # row 0 of each sequence is its initial state, exactly
    assert torch.equal(cs[0].cpu(), x["initial_state"][0])
    assert torch.equal(cs[6].cpu(), x["initial_state"][1])


@pytest.mark.parametrize("gated", [False, True])
def test_states_packed(gated):
    lens = [0, 1, 64, 130, 0, 200]
    w = wl.custom(1, 0, 2, 64, 64, torch.bfloat16, init_state=True, seqlens=lens, gated=True)
    x = wl.generate(w, seed=61)
    check(w, x, gated, seg_chunks=1)


@pytest.mark.parametrize("seg", [0, 1, 3])
def test_states_packed_tensor_core_shape(seg):
    """d_k = d_v = 128 bf16 DeltaNet: the tensor-core boundary kernel writes the
    states, packed input with empty and 1-token sequences, split or not."""
    lens = [0, 1, 64, 130, 0, 200, 700]
    w = wl.custom(1, 0, 2, 128, 128, torch.bfloat16, init_state=True, seqlens=lens)
    x = wl.generate(w, seed=62)
    check(w, x, False, seg_chunks=seg)
