"""Pins for the Gated DeltaNet oracle ("Linear Attention, Visualized", section
"Gated DeltaNet (GDN)"): S_t = a_t (I - beta_t k_t^T k_t) S_{t-1} + beta_t k_t^T v_t,
o_t = q_t S_t, with the decay a_t given to the oracle as g_t = ln a_t.

No value here comes from the CUDA path.  The pins are what the page and the
mathematics fix: all gates 1 is plain DeltaNet; beta = 0 leaves pure decay;
orthonormal keys with beta = 1 give the page's Mamba-2 form with V in place of
Z; the recurrence multiplied out with explicit d x d transition matrices; and
the page's per-chunk algorithm (Gamma mask, left- and right-decayed rows) at
every chunk size.  ``test_planted_gate_mistakes_are_caught`` plants gate
mistakes in copies of the recurrence and checks that the pins reject them.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import chunkwise as cw

RTOL = 1e-12


def _t(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float64))


def f32(x):
    """beta and g travel as fp32; draw them there so both sides use the same value."""
    return np.asarray(x, dtype=np.float32).astype(np.float64)


def run(Q, K, V, beta, g, S0=None):
    """Gated token recurrence (C oracle) for one (sequence, head)."""
    n, dk = K.shape
    dv = V.shape[1]
    b = torch.from_numpy(np.asarray(beta, dtype=np.float32)).reshape(1, n, 1)
    gg = None if g is None else torch.from_numpy(np.asarray(g, dtype=np.float32)).reshape(1, n, 1)
    s0 = None if S0 is None else _t(S0).reshape(1, 1, dk, dv)
    out, fs = oracle.token_recurrence(_t(Q).reshape(1, n, 1, dk), _t(K).reshape(1, n, 1, dk),
                                      _t(V).reshape(1, n, 1, dv), b, s0, n_threads=1, g=gg)
    return out.reshape(n, dv).numpy(), fs.reshape(dk, dv).numpy()


def unit_rows(rng, n, d):
    x = rng.standard_normal((n, d))
    return x / np.linalg.norm(x, axis=1, keepdims=True)


def close(a, b, tol=RTOL):
    scale = max(1.0, float(np.max(np.abs(b))))
    return float(np.max(np.abs(a - b))) <= tol * scale


def draw(rng, n, dk, dv, g_lo=-0.5, g_hi=0.0):
    Q = rng.standard_normal((n, dk))
    K = unit_rows(rng, n, dk)
    V = rng.standard_normal((n, dv))
    b = f32(rng.uniform(0.05, 1.0, n))
    g = f32(rng.uniform(g_lo, g_hi, n))
    return Q, K, V, b, g


def matrix_form(Q, K, V, beta, a, S0):
    """The GDN recurrence as the page writes it, with explicit d_k x d_k
    transition matrices: S_t = a_t (I - beta_t k_t^T k_t) S_{t-1} + beta_t k_t^T v_t."""
    S = S0.copy()
    O = np.zeros((K.shape[0], V.shape[1]))
    for t in range(K.shape[0]):
        A = a[t] * (np.eye(K.shape[1]) - beta[t] * np.outer(K[t], K[t]))
        S = A @ S + beta[t] * np.outer(K[t], V[t])
        O[t] = Q[t] @ S
    return O, S


def test_unit_gates_are_plain_deltanet():
    """a_t = 1 (g_t = 0) removes the decay: the result is DeltaNet's, bit for bit."""
    rng = np.random.default_rng(1)
    Q, K, V, b, _ = draw(rng, 40, 6, 5)
    S0 = rng.standard_normal((6, 5))
    o1, s1 = run(Q, K, V, b, np.zeros(40), S0)
    o2, s2 = run(Q, K, V, b, None, S0)
    assert np.array_equal(o1, o2) and np.array_equal(s1, s2)


def test_zero_beta_is_pure_decay():
    """beta = 0 writes nothing: S_t = (prod_{s<=t} a_s) S_0 and o_t = q_t S_t."""
    rng = np.random.default_rng(2)
    n, dk, dv = 25, 4, 3
    Q, K, V, _, g = draw(rng, n, dk, dv, -1.0, 0.0)
    S0 = rng.standard_normal((dk, dv))
    o, s = run(Q, K, V, np.zeros(n), g, S0)
    lam = np.cumprod(np.exp(g))
    assert close(s, lam[-1] * S0)
    assert close(o, lam[:, None] * (Q @ S0))


def test_orthonormal_keys_give_decayed_linear_attention():
    """Orthonormal keys, beta = 1, S_0 = 0: each write lands on a direction no
    other key reads, so GDN is linear attention with scalar decay (the page's
    Mamba-2 row with V in place of Z): O = (Q K^T o D) V, D[t, s] = lambda[s+1:t]."""
    rng = np.random.default_rng(3)
    n, dk, dv = 12, 16, 5
    K = np.linalg.qr(rng.standard_normal((dk, dk)))[0][:n]
    Q = rng.standard_normal((n, dk))
    V = rng.standard_normal((n, dv))
    g = f32(rng.uniform(-0.7, 0.0, n))
    o, s = run(Q, K, V, np.ones(n), g)
    a = np.exp(g)
    assert close(o, cw.decayed_linear_attention(Q, K, V, a), 1e-12)
    lam = cw.decay_products(a)
    S_ref = sum(lam(t + 2, n) * np.outer(K[t], V[t]) for t in range(n))
    assert close(s, S_ref, 1e-12)


def test_matrix_form_brute_force():
    """The rank-one update of the oracle against the explicit transition matrices."""
    rng = np.random.default_rng(4)
    n, dk, dv = 30, 5, 7
    Q, K, V, b, g = draw(rng, n, dk, dv, -0.4, 0.0)
    K = K * rng.uniform(0.5, 1.5, (n, 1))  # keys off the unit sphere too
    S0 = rng.standard_normal((dk, dv))
    o, s = run(Q, K, V, b, g, S0)
    Om, Sm = matrix_form(Q, K, V, b, np.exp(g), S0)
    assert close(o, Om, 1e-12) and close(s, Sm, 1e-12)


@pytest.mark.parametrize("C", [1, 2, 5, 16, 64, 1000])
def test_gated_chunk_form_equals_recurrence(C):
    """The GDN "Complete per-chunk algorithm" at any chunk size (C = 1 is the
    recurrence itself, C >= n one chunk) equals the token recurrence."""
    rng = np.random.default_rng(5)
    n, dk, dv = 150, 8, 6
    Q, K, V, b, g = draw(rng, n, dk, dv, -0.3, 0.0)
    S0 = rng.standard_normal((dk, dv))
    o, s = run(Q, K, V, b, g, S0)
    Oc, Sc = cw.gated_chunkwise(Q, K, V, b, np.exp(g), S0, C)
    assert close(Oc, o, 1e-11) and close(Sc, s, 1e-11)


def test_gated_chunk_form_with_strong_decay():
    """Decays down to a = e^-4 per token: within-chunk products reach e^-250."""
    rng = np.random.default_rng(6)
    n, dk, dv = 130, 6, 6
    Q, K, V, b, g = draw(rng, n, dk, dv, -4.0, 0.0)
    S0 = rng.standard_normal((dk, dv))
    o, s = run(Q, K, V, b, g, S0)
    Oc, Sc = cw.gated_chunkwise(Q, K, V, b, np.exp(g), S0, 64)
    assert close(Oc, o, 1e-11) and close(Sc, s, 1e-11)


def test_gated_chunk_transition_brute_force():
    """One chunk's transition lambda[1:C] I - K->^T W<- equals the ordered
    product of a_l (I - beta_l k_l^T k_l), and K->^T U the zero-start writes."""
    rng = np.random.default_rng(7)
    c, d = 7, 5
    _, K, V, b, g = draw(rng, c, d, 3, -0.6, 0.0)
    a = np.exp(g)
    f = cw.gated_chunk_factors(K, V, b, a)
    P = np.eye(d)
    for t in range(c):
        P = a[t] * (np.eye(d) - b[t] * np.outer(K[t], K[t])) @ P
    assert close(f["lamC"] * np.eye(d) - f["Kr"].T @ f["W"], P, 1e-13)
    _, Hz = matrix_form(np.zeros((c, d)), K, V, b, a, np.zeros((d, 3)))
    assert close(f["Kr"].T @ f["U"], Hz, 1e-13)


@pytest.mark.parametrize("G", [2, 3, 7])
def test_gated_segmented_scan_equals_serial(G):
    """Composing the GDN segment maps (P_g, H_g) reproduces the serial pass."""
    rng = np.random.default_rng(8)
    n, dk, dv = 64 * 7 + 11, 6, 5
    Q, K, V, b, g = draw(rng, n, dk, dv, -0.2, 0.0)
    S0 = rng.standard_normal((dk, dv))
    o, s = run(Q, K, V, b, g, S0)
    Op, Sp = cw.gated_context_parallel(Q, K, V, b, np.exp(g), S0, 64, G)
    assert close(Op, o, 1e-10) and close(Sp, s, 1e-10)


def test_gated_varlen_packing_equals_separate_calls():
    """Sequences in one packed call restart from their own state and gates."""
    gen = torch.Generator().manual_seed(9)
    lens = [5, 0, 17, 9]
    H, dk, dv = 2, 4, 3
    T = sum(lens)
    q = torch.randn(1, T, H, dk, generator=gen, dtype=torch.float64)
    k = torch.randn(1, T, H, dk, generator=gen, dtype=torch.float64)
    v = torch.randn(1, T, H, dv, generator=gen, dtype=torch.float64)
    beta = torch.rand(1, T, H, generator=gen)
    g = -torch.rand(1, T, H, generator=gen)
    s0 = torch.randn(len(lens), H, dk, dv, generator=gen, dtype=torch.float64)
    cu = torch.tensor([0] + np.cumsum(lens).tolist(), dtype=torch.int32)
    out, fs = oracle.token_recurrence(q, k, v, beta, s0, cu, g=g)
    for n, (a0, L) in enumerate(zip(cu[:-1].tolist(), lens)):
        for h in range(H):
            o_n, f_n = run(q[0, a0:a0 + L, h].numpy(), k[0, a0:a0 + L, h].numpy(),
                           v[0, a0:a0 + L, h].numpy(), beta[0, a0:a0 + L, h].numpy(),
                           g[0, a0:a0 + L, h].numpy(), s0[n, h].numpy())
            assert np.array_equal(out[0, a0:a0 + L, h].numpy(), o_n)
            assert np.array_equal(fs[n, h].numpy(), f_n)


def test_gate_shape_is_checked():
    q = torch.zeros(1, 4, 1, 2, dtype=torch.float64)
    with pytest.raises(ValueError):
        oracle.token_recurrence(q, q, q, torch.zeros(1, 4, 1), g=torch.zeros(1, 3, 1))


# --- the pins reject plausible gate mistakes -------------------------------------

def _mutant(kind, Q, K, V, beta, a, S0):
    """A deliberately wrong gated recurrence (numpy), one mistake per kind."""
    S = S0.copy()
    O = np.zeros((K.shape[0], V.shape[1]))
    for t in range(K.shape[0]):
        if kind == "decay_after_write":
            u = beta[t] * (V[t] - K[t] @ S)
            S = a[t] * (S + np.outer(K[t], u))
        elif kind == "undecayed_prediction":
            u = beta[t] * (V[t] - K[t] @ S)
            S = a[t] * S + np.outer(K[t], u)
        elif kind == "decay_on_read_only":
            u = beta[t] * (V[t] - K[t] @ S)
            S = S + np.outer(K[t], u)
        else:
            Sd = a[t] * S
            S = Sd + np.outer(K[t], beta[t] * (V[t] - K[t] @ Sd))
        O[t] = (a[t] if kind == "decay_on_read_only" else 1.0) * (Q[t] @ S)
    return O, S


@pytest.mark.parametrize("kind", ["decay_after_write", "undecayed_prediction",
                                  "decay_on_read_only"])
def test_planted_gate_mistakes_are_caught(kind):
    """The matrix form and the chunk form reject each planted mistake; the
    correct restatement passes them."""
    rng = np.random.default_rng(10)
    n, dk, dv = 20, 5, 4
    Q, K, V, b, g = draw(rng, n, dk, dv, -0.5, -0.05)
    a = np.exp(g)
    S0 = rng.standard_normal((dk, dv))
    O, S = matrix_form(Q, K, V, b, a, S0)
    Oc, Sc = cw.gated_chunkwise(Q, K, V, b, a, S0, 8)
    Om, Sm = _mutant(kind, Q, K, V, b, a, S0)
    assert not (close(Om, O, 1e-6) and close(Sm, S, 1e-6))
    assert not (close(Om, Oc, 1e-6) and close(Sm, Sc, 1e-6))
    On, Sn = _mutant("none", Q, K, V, b, a, S0)
    assert close(On, O, 1e-12) and close(Sn, S, 1e-12)
