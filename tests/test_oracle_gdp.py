"""Pins for the Gated Delta Product oracle ("Linear Attention, Visualized",
section "Gated Delta Product (GDP)"): per token, S_{t,0} = a_t S_{t-1}, then n_h
delta-rule writes S_{t,j} = (I - b_{t,j} k_{t,j}^T k_{t,j}) S_{t,j-1} + b_{t,j} k_{t,j}^T v_{t,j},
then o_t = q_t S_{t,n_h}.  k, v and beta hold n_h rows per token, substep-major.

No value here comes from the CUDA path.  The C oracle states the substeps
directly; the pins are the page's own explicit-matrix update, its claim that
GDP is GDN over the virtual sequence (run through the independent numpy GDN
chunk form), n_h = 1 being GDN, and writes with beta = 0 dropping out.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import chunkwise as cw


def _t(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float64))


def f32(x):
    return np.asarray(x, dtype=np.float32).astype(np.float64)


def close(a, b, tol):
    scale = max(1.0, float(np.max(np.abs(b))))
    return float(np.max(np.abs(a - b))) <= tol * scale


def run(Q, K, V, beta, g, n_h, S0=None):
    n, dk = Q.shape
    dv = V.shape[1]
    q = _t(Q).reshape(1, n, 1, dk)
    k = _t(K).reshape(1, n * n_h, 1, dk)
    v = _t(V).reshape(1, n * n_h, 1, dv)
    b = torch.from_numpy(np.asarray(beta, dtype=np.float32)).reshape(1, n * n_h, 1)
    gg = torch.from_numpy(np.asarray(g, dtype=np.float32)).reshape(1, n, 1)
    s0 = None if S0 is None else _t(S0).reshape(1, 1, dk, dv)
    out, fs = oracle.token_recurrence(q, k, v, b, s0, n_threads=1, g=gg, n_sub=n_h)
    return out.reshape(n, dv).numpy(), fs.reshape(dk, dv).numpy()


def draw(rng, n, n_h, dk, dv):
    Q = rng.standard_normal((n, dk))
    K = rng.standard_normal((n * n_h, dk))
    K /= np.linalg.norm(K, axis=1, keepdims=True)
    V = rng.standard_normal((n * n_h, dv))
    b = f32(rng.uniform(0.05, 1.0, n * n_h))
    g = f32(rng.uniform(-0.5, 0.0, n))
    return Q, K, V, b, g


@pytest.mark.parametrize("n_h", [1, 2, 3])
def test_substeps_match_explicit_matrices(n_h):
    """The oracle's rank-one writes against the page's update with explicit
    transition matrices (decay once, then the n_h writes, then the readout)."""
    rng = np.random.default_rng(30 + n_h)
    Q, K, V, b, g = draw(rng, 17, n_h, 5, 4)
    S0 = rng.standard_normal((5, 4))
    o, s = run(Q, K, V, b, g, n_h, S0)
    Om, Sm = cw.gdp_substeps(Q, K, V, b, np.exp(g), n_h, S0)
    assert close(o, Om, 1e-12) and close(s, Sm, 1e-12)


@pytest.mark.parametrize("n_h,C", [(2, 1), (2, 16), (2, 64), (3, 7), (3, 64), (4, 32)])
def test_gdp_is_gdn_over_the_virtual_sequence(n_h, C):
    """The page's construction: flattening the substeps into virtual steps with
    the decay on the first and the query on the last gives the same outputs
    and final state (through the independent numpy GDN chunk form)."""
    rng = np.random.default_rng(40 + n_h + C)
    Q, K, V, b, g = draw(rng, 53, n_h, 6, 5)
    S0 = rng.standard_normal((6, 5))
    o, s = run(Q, K, V, b, g, n_h, S0)
    Ov, Sv = cw.gdp_chunkwise(Q, K, V, b, np.exp(g), n_h, S0, C)
    assert close(o, Ov, 1e-11) and close(s, Sv, 1e-11)


def test_one_substep_is_gdn():
    """n_h = 1 is Gated DeltaNet, bit for bit."""
    rng = np.random.default_rng(50)
    Q, K, V, b, g = draw(rng, 40, 1, 6, 3)
    S0 = rng.standard_normal((6, 3))
    o1, s1 = run(Q, K, V, b, g, 1, S0)
    n = Q.shape[0]
    o2, s2 = oracle.token_recurrence(_t(Q).reshape(1, n, 1, 6), _t(K).reshape(1, n, 1, 6),
                                     _t(V).reshape(1, n, 1, 3),
                                     torch.from_numpy(np.asarray(b, np.float32)).reshape(1, n, 1),
                                     _t(S0).reshape(1, 1, 6, 3), n_threads=1,
                                     g=torch.from_numpy(np.asarray(g, np.float32)).reshape(1, n, 1))
    assert np.array_equal(o1, o2.reshape(n, 3).numpy()) and np.array_equal(s1, s2.reshape(6, 3).numpy())


def test_zero_beta_substeps_drop_out():
    """Writes with beta = 0 are identities: GDP with the second substep's beta
    zeroed equals GDN on the first substeps alone."""
    rng = np.random.default_rng(51)
    n = 30
    Q, K, V, b, g = draw(rng, n, 2, 5, 4)
    b[1::2] = 0.0
    S0 = rng.standard_normal((5, 4))
    o2, s2 = run(Q, K, V, b, g, 2, S0)
    o1, s1 = run(Q, K[0::2], V[0::2], b[0::2], g, 1, S0)
    assert close(o2, o1, 1e-13) and close(s2, s1, 1e-13)


def test_gdp_rejects_mismatched_rows():
    q = torch.zeros(1, 4, 1, 2, dtype=torch.float64)
    k = torch.zeros(1, 8, 1, 2, dtype=torch.float64)
    with pytest.raises(ValueError):
        oracle.token_recurrence(q, k, k, torch.zeros(1, 8, 1), g=torch.zeros(1, 4, 1), n_sub=3)


def _mutant(kind, Q, K, V, beta, a, n_h, S0):
    S = S0.copy()
    O = np.zeros((Q.shape[0], V.shape[1]))
    for t in range(Q.shape[0]):
        if kind != "decay_every_substep":
            S = a[t] * S
        for j in range(n_h):
            m = t * n_h + j
            if kind == "decay_every_substep":
                S = a[t] * S
            S = S + np.outer(K[m], beta[m] * (V[m] - K[m] @ S))
            if kind == "read_after_first" and j == 0:
                O[t] = Q[t] @ S
        if kind != "read_after_first":
            O[t] = Q[t] @ S
    return O, S


@pytest.mark.parametrize("kind", ["decay_every_substep", "read_after_first"])
def test_planted_gdp_mistakes_are_caught(kind):
    rng = np.random.default_rng(52)
    Q, K, V, b, g = draw(rng, 12, 3, 5, 4)
    a = np.exp(g)
    S0 = rng.standard_normal((5, 4))
    O, S = cw.gdp_substeps(Q, K, V, b, a, 3, S0)
    Om, Sm = _mutant(kind, Q, K, V, b, a, 3, S0)
    assert not (close(Om, O, 1e-6) and close(Sm, S, 1e-6))
    On, Sn = _mutant("none", Q, K, V, b, a, 3, S0)
    assert close(On, O, 1e-12) and close(Sn, S, 1e-12)
