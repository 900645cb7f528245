"""The entry point that allocates nothing (deltanet_fwd_noalloc).

Some callers cannot allocate device memory (host callbacks, plugins running
inside another runtime's allocator, graph-recording runtimes, memory-capped
processes).  deltanet_fwd_noalloc serves them from a fixed device array built
into the library.  This file is collected last on purpose: if it fails, a run
that stops at the first failure has already run every other test.
"""
import pytest
import torch

import deltanet_chunkwise_delta_b200 as dn
from deltanet_chunkwise_delta_b200 import _lib
from deltanet_chunkwise_delta_b200 import workloads as wl

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


def rel_err(x, ref):
    x, ref = x.double().cpu(), ref.double().cpu()
    m = ref.abs().max().item()
    return (x - ref).abs().max().item() / (m if m > 0 else 1.0)


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dn.load()


def test_noalloc_matches_allocating_entry_point_on_two_calls():
    """Two calls in a row (different inputs, same shared scratch) match the
    allocating entry point within the bf16 parity tolerance."""
    for seed in (1, 2):
        w = wl.custom(2, 300, 4, 128, 128, torch.bfloat16, init_state=True)
        x = wl.generate(w, seed=seed)
        g = {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
        o_ref, s_ref = dn.deltanet_fwd(g["q"], g["k"], g["v"], g["beta"], g["initial_state"])
        o, s = _lib.deltanet_fwd_noalloc(g["q"], g["k"], g["v"], g["beta"], g["initial_state"])
        torch.cuda.synchronize()
        assert rel_err(o, o_ref) <= 1e-2
        assert rel_err(s, s_ref) <= 1e-2


def test_noalloc_rejects_sizes_beyond_its_scratch():
    q = torch.zeros((1, 64 * 3073, 1, 128), dtype=torch.bfloat16, device=DEV)
    b = torch.zeros((1, 64 * 3073, 1), device=DEV)
    with pytest.raises(dn.DeltaNetError) as e:
        _lib.deltanet_fwd_noalloc(q, q, q, b)
    assert e.value.status == _lib.DN_ERR_WORKSPACE
