"""Pins for the Kimi Delta Attention oracle ("Linear Attention, Visualized",
section "Kimi Delta Attention (KDA)"): S_t = Diag(a_t) S_{t-1} +
beta_t k_t^T (v_t - k_t Diag(a_t) S_{t-1}), o_t = q_t S_t, with a_t in (0, 1]^{d_k}
given as g = ln a [B, T, H, d_k].

No value here comes from a CUDA path.  The pins: equal channel gates are GDN
(bit for bit); beta = 0 is pure channelwise decay; one-hot keys on distinct
channels with beta = 1 make the correction vanish, leaving GLA, checked
against the page's GLA chunk form; the page's first (matrix) line of the
update; its complete per-chunk algorithm at every chunk size; the segment
maps; and planted mistakes.
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


def run(Q, K, V, beta, G, S0=None):
    """C oracle, one (sequence, head); G [n, d_k] log decays (or [n] scalar)."""
    n, dk = K.shape
    dv = V.shape[1]
    b = torch.from_numpy(np.asarray(beta, np.float32)).reshape(1, n, 1)
    gt = torch.from_numpy(np.asarray(G, np.float32))
    gt = gt.reshape(1, n, 1, dk) if gt.dim() == 2 else gt.reshape(1, n, 1)
    s0 = None if S0 is None else _t(S0).reshape(1, 1, dk, dv)
    out, fs = oracle.token_recurrence(_t(Q).reshape(1, n, 1, dk), _t(K).reshape(1, n, 1, dk),
                                      _t(V).reshape(1, n, 1, dv), b, s0, n_threads=1, g=gt)
    return out.reshape(n, dv).numpy(), fs.reshape(dk, dv).numpy()


def draw(rng, n, dk, dv, lo=-0.5):
    Q = rng.standard_normal((n, dk))
    K = rng.standard_normal((n, dk))
    K /= np.linalg.norm(K, axis=1, keepdims=True)
    V = rng.standard_normal((n, dv))
    b = f32(rng.uniform(0.05, 1.0, n))
    G = f32(rng.uniform(lo, 0.0, (n, dk)))
    return Q, K, V, b, G


def matrix_form(Q, K, V, beta, A, S0):
    """The page's first line: S_t = (I - beta k^T k) Diag(a_t) S_{t-1} + beta k^T v."""
    S = S0.copy()
    O = np.zeros((K.shape[0], V.shape[1]))
    for t in range(K.shape[0]):
        S = (np.eye(K.shape[1]) - beta[t] * np.outer(K[t], K[t])) @ np.diag(A[t]) @ S \
            + beta[t] * np.outer(K[t], V[t])
        O[t] = Q[t] @ S
    return O, S


def test_equal_channel_gates_are_gdn():
    """a_t = a_t 1 is GDN, bit for bit."""
    rng = np.random.default_rng(70)
    Q, K, V, b, G = draw(rng, 40, 6, 4)
    g = G[:, 0]
    S0 = rng.standard_normal((6, 4))
    o1, s1 = run(Q, K, V, b, np.repeat(g[:, None], 6, axis=1), S0)
    o2, s2 = run(Q, K, V, b, g, S0)
    assert np.array_equal(o1, o2) and np.array_equal(s1, s2)


def test_zero_beta_is_channelwise_decay():
    rng = np.random.default_rng(71)
    n, dk, dv = 20, 5, 3
    Q, K, V, _, G = draw(rng, n, dk, dv, -1.0)
    S0 = rng.standard_normal((dk, dv))
    o, s = run(Q, K, V, np.zeros(n), G, S0)
    lam = np.cumprod(np.exp(G), axis=0)               # [n, dk]
    assert close(s, lam[-1][:, None] * S0, 1e-12)
    assert close(o, np.stack([Q[t] @ (lam[t][:, None] * S0) for t in range(n)]), 1e-12)


def test_one_hot_keys_reduce_to_gla():
    """Keys on distinct basis channels with beta = 1 and S_0 = 0: a key never reads
    another write's channel, so the correction vanishes and KDA is GLA,
    S_t = Diag(a_t) S_{t-1} + k_t^T v_t, checked against the page's GLA chunk form."""
    rng = np.random.default_rng(72)
    n, dk, dv = 12, 16, 5
    K = np.eye(dk)[rng.permutation(dk)[:n]]
    Q = rng.standard_normal((n, dk))
    V = rng.standard_normal((n, dv))
    G = f32(rng.uniform(-0.6, 0.0, (n, dk)))
    o, s = run(Q, K, V, np.ones(n), G)
    for C in (n, 5):
        Og, Sg = cw.gla_chunkwise(Q, K, V, np.exp(G), None, C)
        assert close(o, Og, 1e-12) and close(s, Sg, 1e-12)


def test_matrix_form_brute_force():
    rng = np.random.default_rng(73)
    Q, K, V, b, G = draw(rng, 25, 5, 6)
    K = K * rng.uniform(0.5, 1.5, (25, 1))
    S0 = rng.standard_normal((5, 6))
    o, s = run(Q, K, V, b, G, S0)
    Om, Sm = matrix_form(Q, K, V, b, np.exp(G), S0)
    assert close(o, Om, 1e-12) and close(s, Sm, 1e-12)


@pytest.mark.parametrize("C", [1, 3, 16, 64, 1000])
def test_kda_chunk_form_equals_recurrence(C):
    rng = np.random.default_rng(74)
    Q, K, V, b, G = draw(rng, 100, 6, 5, -0.3)
    S0 = rng.standard_normal((6, 5))
    o, s = run(Q, K, V, b, G, S0)
    Oc, Sc = cw.kda_chunkwise(Q, K, V, b, np.exp(G), S0, C)
    assert close(Oc, o, 1e-11) and close(Sc, s, 1e-11)


@pytest.mark.parametrize("G_", [2, 3])
def test_kda_segment_maps_compose(G_):
    """Composing the KDA segment maps from S_0 reproduces the serial final state."""
    rng = np.random.default_rng(75)
    n, C = 64 * 5 + 9, 64
    _, K, V, b, G = draw(rng, n, 5, 4, -0.2)
    S0 = rng.standard_normal((5, 4))
    _, s = run(np.zeros((n, 5)), K, V, b, G, S0)
    chunks = cw.chunk_bounds(n, C)
    edges = [round(g * len(chunks) / G_) for g in range(G_ + 1)]
    S = S0.copy()
    for g in range(G_):
        a, e = chunks[edges[g]][0], chunks[edges[g + 1] - 1][1]
        P, H = cw.kda_segment_map(K[a:e], V[a:e], b[a:e], np.exp(G[a:e]), C)
        S = P @ S + H
    assert close(S, s, 1e-10)


def _mutant(kind, Q, K, V, beta, A, S0):
    S = S0.copy()
    O = np.zeros((K.shape[0], V.shape[1]))
    for t in range(K.shape[0]):
        if kind == "decay_value_channels":
            Sd = S * A[t][: S.shape[1]][None, :]
        elif kind == "decay_after_correction":
            Sd = S
        else:
            Sd = A[t][:, None] * S
        S = Sd + np.outer(K[t], beta[t] * (V[t] - K[t] @ Sd))
        if kind == "decay_after_correction":
            S = A[t][:, None] * S
        O[t] = Q[t] @ S
    return O, S


@pytest.mark.parametrize("kind", ["decay_value_channels", "decay_after_correction"])
def test_planted_kda_mistakes_are_caught(kind):
    rng = np.random.default_rng(76)
    Q, K, V, b, G = draw(rng, 15, 6, 6, -0.6)
    A = np.exp(G)
    S0 = rng.standard_normal((6, 6))
    O, S = matrix_form(Q, K, V, b, A, S0)
    Om, Sm = _mutant(kind, Q, K, V, b, A, S0)
    assert not (close(Om, O, 1e-6) and close(Sm, S, 1e-6))
    On, Sn = _mutant("none", Q, K, V, b, A, S0)
    assert close(On, O, 1e-12) and close(Sn, S, 1e-12)
