"""The time-out path of the bounded device waits, on the GPU, with no fault.

Every wait of the tensor-core kernels on an mbarrier gives up after a time
limit: the CTA then stops issuing, waits for its copies and tensor-core
products already in flight, frees its tensor memory, exits and reports
DN_ERR_TIMEOUT through deltanet_get_error.  These tests make a wait run out
on purpose through the library's test hook (deltanet_test_set_wait): a short
limit and a wait, at a chosen chunk of every run, on a barrier that nothing
completes.  They then check that the error reaches the caller and that a
normal call on the same stream afterwards matches the float64 oracle.
"""
import pytest
import torch

import oracle
import deltanet_chunkwise_delta_b200 as dn
from deltanet_chunkwise_delta_b200 import _lib
from deltanet_chunkwise_delta_b200 import workloads as wl

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")
LIMIT_NS = 1_000_000  # 1 ms


def rel_err(x, ref):
    x, ref = x.double().cpu(), ref.double().cpu()
    m = ref.abs().max().item()
    return (x - ref).abs().max().item() / (m if m > 0 else 1.0)


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dn.load()
    yield
    dn.test_set_wait()


def _inputs(T, seed):
    w = wl.custom(2, T, 2, 128, 128, torch.bfloat16, init_state=True)
    x = wl.generate(w, seed=seed)
    g = {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
    return x, g


@pytest.mark.parametrize("stall_chunk,seg_chunks", [(1, 0), (3, 0), (2, 2)])
def test_stalled_wait_reports_timeout_then_next_call_is_exact(stall_chunk, seg_chunks):
    """A run whose chain issuer waits on a barrier nothing completes (before its
    first product, or after two chunks' products are in flight; one run per
    chain or runs of two chunks) ends with DN_ERR_TIMEOUT; the next normal call
    on the same stream equals the oracle within the bf16 bar."""
    x, g = _inputs(400, seed=stall_chunk)
    assert dn.get_error() == 0
    dn.test_set_wait(LIMIT_NS, stall_chunk)
    try:
        dn.deltanet_fwd(g["q"], g["k"], g["v"], g["beta"], g["initial_state"],
                        seg_chunks=seg_chunks)
        assert dn.get_error() == _lib.DN_ERR_TIMEOUT
    finally:
        dn.test_set_wait()
    assert dn.get_error() == 0   # read once, then cleared
    out, fs = dn.deltanet_fwd(g["q"], g["k"], g["v"], g["beta"], g["initial_state"],
                              seg_chunks=seg_chunks)
    assert dn.get_error() == 0
    ref_o, ref_s = oracle.token_recurrence(x["q"], x["k"], x["v"], x["beta"], x["initial_state"])
    eo, es = rel_err(out, ref_o), rel_err(fs, ref_s)
    print(f"after time-out: out {eo:.3e}, final_state {es:.3e}")
    assert eo <= 1e-2 and es <= 1e-2, (eo, es)


def test_short_limit_alone_does_not_fire():
    """A 1 ms limit with no stall: every wait of a normal call completes well
    within it, so the call reports no error and stays exact."""
    x, g = _inputs(700, seed=7)
    dn.test_set_wait(LIMIT_NS, 0)
    try:
        out, fs = dn.deltanet_fwd(g["q"], g["k"], g["v"], g["beta"], g["initial_state"],
                                  seg_chunks=3)
        assert dn.get_error() == 0
    finally:
        dn.test_set_wait()
    ref_o, ref_s = oracle.token_recurrence(x["q"], x["k"], x["v"], x["beta"], x["initial_state"])
    assert rel_err(out, ref_o) <= 1e-2 and rel_err(fs, ref_s) <= 1e-2
