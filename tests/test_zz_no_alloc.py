"""The entry point that allocates nothing (deltanet_fwd_noalloc).

Some callers cannot allocate device memory: host callbacks and plugins that run
inside another runtime's allocator, graph-recording runtimes that forbid
allocation while they record, and processes whose device memory is capped and
owned by someone else.  deltanet_fwd_noalloc serves them from a fixed device
array built into the library.  These tests check it against the float64 oracle
and against the allocating entry point, at its largest accepted size, and that
its aliasing rules and device-side errors behave like deltanet_fwd's.  This file
is collected last on purpose: if it fails, a run that stops at the first failure
has already run every other test.
"""
import pytest
import torch

import oracle
import deltanet_chunkwise_delta_b200 as dn
from deltanet_chunkwise_delta_b200 import _lib
from deltanet_chunkwise_delta_b200 import workloads as wl

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")
TOL = 1e-2  # bf16 inputs: max|x - x_ref| / max|x_ref|


def rel_err(x, ref):
    x, ref = x.double().cpu(), ref.double().cpu()
    m = ref.abs().max().item()
    return (x - ref).abs().max().item() / (m if m > 0 else 1.0)


def to_dev(x):
    return {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in x.items()}


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dn.load()
    yield
    dn.test_set_wait()


def test_noalloc_matches_oracle_and_allocating_entry_point_on_two_calls():
    """Two calls in a row (different inputs, the same shared scratch, which the
    second call must rewrite): each matches the float64 oracle and the
    allocating entry point within the bf16 bar."""
    for seed in (1, 2):
        w = wl.custom(2, 300, 4, 128, 128, torch.bfloat16, init_state=True)
        x = wl.generate(w, seed=seed)
        g = to_dev(x)
        o, s = _lib.deltanet_fwd_noalloc(g["q"], g["k"], g["v"], g["beta"], g["initial_state"])
        assert dn.get_error() == 0
        o_a, s_a = dn.deltanet_fwd(g["q"], g["k"], g["v"], g["beta"], g["initial_state"])
        assert dn.get_error() == 0
        ref_o, ref_s = oracle.token_recurrence(x["q"], x["k"], x["v"], x["beta"], x["initial_state"])
        eo, es = rel_err(o, ref_o), rel_err(s, ref_s)
        print(f"noalloc call {seed} vs oracle: out {eo:.3e}, final_state {es:.3e}")
        assert eo <= TOL and es <= TOL, (eo, es)
        assert rel_err(o, o_a) <= TOL and rel_err(s, s_a) <= TOL


def test_noalloc_at_its_largest_size_without_initial_state():
    """B * ceil(T / 64) * H == 3072 (chunk, head) pairs, the limit: the last
    16 KiB unit of the array is written and read; no initial state."""
    w = wl.custom(2, 64 * 384, 4, 128, 128, torch.bfloat16, init_state=False)
    x = wl.generate(w, seed=3)
    g = to_dev(x)
    o, s = _lib.deltanet_fwd_noalloc(g["q"], g["k"], g["v"], g["beta"], None)
    assert dn.get_error() == 0
    ref_o, ref_s = oracle.token_recurrence(x["q"], x["k"], x["v"], x["beta"], None)
    eo, es = rel_err(o, ref_o), rel_err(s, ref_s)
    print(f"noalloc at 3072 units vs oracle: out {eo:.3e}, final_state {es:.3e}")
    assert eo <= TOL and es <= TOL, (eo, es)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    q = torch.zeros((1, 64 * 3073, 1, 128), dtype=torch.bfloat16, device=DEV)
    b = torch.zeros((1, 64 * 3073, 1), device=DEV)
    with pytest.raises(dn.DeltaNetError) as e:
        _lib.deltanet_fwd_noalloc(q, q, q, b)
    assert e.value.status == _lib.DN_ERR_WORKSPACE


def test_noalloc_rejects_aliasing_like_the_allocating_entry_point():
    """final_state on initial_state, and out on q, are refused before any work."""
    w = wl.custom(1, 64, 2, 128, 128, torch.bfloat16, init_state=True)
    g = to_dev(wl.generate(w, seed=4))
    s0 = g["initial_state"]
    with pytest.raises(dn.DeltaNetError) as e:
        _lib.deltanet_fwd_noalloc(g["q"], g["k"], g["v"], g["beta"], s0, final_state=s0)
    assert e.value.status == _lib.DN_ERR_ALIAS
    with pytest.raises(dn.DeltaNetError) as e:
        dn.deltanet_fwd(g["q"], g["k"], g["v"], g["beta"], s0, final_state=s0)
    assert e.value.status == _lib.DN_ERR_ALIAS
    with pytest.raises(dn.DeltaNetError) as e:
        _lib.deltanet_fwd_noalloc(g["q"], g["k"], g["v"], g["beta"], s0, out=g["q"])
    assert e.value.status == _lib.DN_ERR_ALIAS


def test_noalloc_device_timeout_reaches_the_caller():
    """A wait that runs out inside a no-alloc call (the library's test stall,
    1 ms limit) is reported by deltanet_get_error on that call's stream; the
    next no-alloc call clears the word and matches the oracle."""
    w = wl.custom(1, 256, 2, 128, 128, torch.bfloat16, init_state=True)
    x = wl.generate(w, seed=5)
    g = to_dev(x)
    assert dn.get_error() == 0
    dn.test_set_wait(1_000_000, 2)
    try:
        _lib.deltanet_fwd_noalloc(g["q"], g["k"], g["v"], g["beta"], g["initial_state"])
        assert dn.get_error() == _lib.DN_ERR_TIMEOUT
    finally:
        dn.test_set_wait()
    assert dn.get_error() == 0
    o, s = _lib.deltanet_fwd_noalloc(g["q"], g["k"], g["v"], g["beta"], g["initial_state"])
    assert dn.get_error() == 0
    ref_o, ref_s = oracle.token_recurrence(x["q"], x["k"], x["v"], x["beta"], x["initial_state"])
    assert rel_err(o, ref_o) <= TOL and rel_err(s, ref_s) <= TOL
