"""Pins for the oracle: checks against what the pages and the mathematics fix.

No value here comes from the CUDA path.  Each test names the passage it
follows.  A plausible mistake in the oracle (readout before the write, a
dropped beta, a transposed state, a wrong mask or sign) fails at least one:
``test_planted_mistakes_are_caught`` plants several in copies of the oracle's
steps and checks that the pins reject them.
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import chunkwise as cw

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
RTOL = 1e-12


def _t(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float64))


def run(Q, K, V, beta, S0=None):
    """Token recurrence for one (sequence, head) in float64 numpy arrays."""
    n, dk = K.shape
    dv = V.shape[1]
    q = _t(Q).reshape(1, n, 1, dk)
    k = _t(K).reshape(1, n, 1, dk)
    v = _t(V).reshape(1, n, 1, dv)
    b = torch.from_numpy(np.asarray(beta, dtype=np.float32)).reshape(1, n, 1)
    s0 = None if S0 is None else _t(S0).reshape(1, 1, dk, dv)
    out, fs = oracle.token_recurrence(q, k, v, b, s0, n_threads=1)
    return out.reshape(n, dv).numpy(), fs.reshape(dk, dv).numpy()


def unit_rows(rng, n, d):
    x = rng.standard_normal((n, d))
    return x / np.linalg.norm(x, axis=1, keepdims=True)


def f32(x):
    """beta travels as fp32; draw it there so both sides use the same value."""
    return np.asarray(x, dtype=np.float32).astype(np.float64)


def close(a, b, tol=RTOL):
    scale = max(1.0, float(np.max(np.abs(b))))
    return float(np.max(np.abs(a - b))) <= tol * scale


# --- "Recurrent form" and "The triangular correction system" -----------------

def test_hand_expanded_three_tokens():
    """u_1 = b1 v1, u_2 = b2 (v2 - (k2 k1^T) u1),
    u_3 = b3 (v3 - (k3 k1^T) u1 - (k3 k2^T) u2); S_t = sum_{i<=t} k_i^T u_i;
    o_t = q_t S_t.  d_k != d_v so a transposed state cannot pass."""
    rng = np.random.default_rng(1)
    Q = rng.standard_normal((3, 5))
    K = rng.standard_normal((3, 5))
    V = rng.standard_normal((3, 4))
    b = f32(rng.uniform(0.1, 0.9, 3))
    u1 = b[0] * V[0]
    u2 = b[1] * (V[1] - (K[1] @ K[0]) * u1)
    u3 = b[2] * (V[2] - (K[2] @ K[0]) * u1 - (K[2] @ K[1]) * u2)
    S1 = np.outer(K[0], u1)
    S2 = S1 + np.outer(K[1], u2)
    S3 = S2 + np.outer(K[2], u3)
    O = np.stack([Q[0] @ S1, Q[1] @ S2, Q[2] @ S3])
    out, fs = run(Q, K, V, b)
    assert close(out, O) and close(fs, S3)


def test_alice_bob_golden():
    """Worked example of subsection "An intuitive example" (golden fixture)."""
    with open(os.path.join(GOLDEN, "alice_bob.json")) as f:
        g = json.load(f)
    out, fs = run(np.array(g["q"], float), np.array(g["k"], float),
                  np.array(g["v"], float), f32(g["beta"]))
    assert np.array_equal(out, np.array(g["expected_out"], float))
    assert np.array_equal(fs, np.array(g["expected_final_state"], float))


def test_unit_key_read_back():
    """For ||k_t|| = 1: k_t S_t = (1 - b_t) vhat_t + b_t v_t with vhat_t = k_t S_{t-1}."""
    rng = np.random.default_rng(2)
    n, dk, dv = 7, 6, 3
    Q = rng.standard_normal((n, dk))
    K = unit_rows(rng, n, dk)
    V = rng.standard_normal((n, dv))
    b = f32(rng.uniform(0.05, 1.0, n))
    S0 = 0.3 * rng.standard_normal((dk, dv))
    prev = S0
    for t in range(1, n + 1):
        _, St = run(Q[:t], K[:t], V[:t], b[:t], S0)
        want = (1 - b[t - 1]) * (K[t - 1] @ prev) + b[t - 1] * V[t - 1]
        assert close(K[t - 1] @ St, want, 1e-12)
        prev = St


def test_beta_one_writes_value_exactly():
    """beta_t = 1 and unit key: the read at k_t returns v_t (S_t k_t = v_t in the
    column convention)."""
    rng = np.random.default_rng(3)
    n, dk, dv = 9, 8, 5
    K = unit_rows(rng, n, dk)
    V = rng.standard_normal((n, dv))
    S0 = rng.standard_normal((dk, dv))
    for t in range(1, n + 1):
        _, St = run(K[:t], K[:t], V[:t], np.ones(t), S0)
        assert close(K[t - 1] @ St, V[t - 1], 1e-12)


def test_beta_zero_leaves_state_unchanged():
    """beta = 0: no write, so S_t = S_0 and o_t = q_t S_0."""
    rng = np.random.default_rng(4)
    n, dk, dv = 11, 4, 6
    Q = rng.standard_normal((n, dk))
    K = rng.standard_normal((n, dk))
    V = rng.standard_normal((n, dv))
    S0 = rng.standard_normal((dk, dv))
    out, fs = run(Q, K, V, np.zeros(n), S0)
    assert np.array_equal(fs, S0)
    assert close(out, Q @ S0)


def test_first_token_output():
    """o_1 = q_1 (S_0 + b_1 k_1^T (v_1 - k_1 S_0))."""
    rng = np.random.default_rng(5)
    dk, dv = 5, 7
    Q = rng.standard_normal((1, dk)); K = rng.standard_normal((1, dk))
    V = rng.standard_normal((1, dv)); S0 = rng.standard_normal((dk, dv))
    b = f32([0.37])
    out, _ = run(Q, K, V, b, S0)
    want = Q[0] @ (S0 + b[0] * np.outer(K[0], V[0] - K[0] @ S0))
    assert close(out[0], want)


# --- reduction to linear attention ("Why additive writes collide") ------------

def test_orthonormal_keys_reduce_to_linear_attention():
    """Orthogonal unit keys remove cross-talk; with beta = 1 and S_0 = 0 every
    prediction is zero, so DeltaNet equals causal linear attention
    (Q K^T o M) V exactly."""
    rng = np.random.default_rng(6)
    n, dk, dv = 12, 16, 5
    basis, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
    K = basis[:n]
    Q = rng.standard_normal((n, dk))
    V = rng.standard_normal((n, dv))
    out, _ = run(Q, K, V, np.ones(n))
    assert close(out, cw.linear_attention(Q, K, V), 1e-13)


def test_small_beta_limit_is_additive():
    """As beta -> 0 the correction u_t -> beta v_t (the additive update), so
    O / beta -> (Q K^T o M) V with an O(beta) gap."""
    rng = np.random.default_rng(7)
    n, dk, dv = 20, 8, 4
    Q = rng.standard_normal((n, dk)); K = unit_rows(rng, n, dk)
    V = rng.standard_normal((n, dv))
    beta = 1e-6
    out, _ = run(Q, K, V, f32(np.full(n, beta)))
    b = float(np.float32(beta))
    ref = cw.linear_attention(Q, K, V)
    err = np.max(np.abs(out / b - ref)) / np.max(np.abs(ref))
    assert err < 1e-4


# --- full-sequence closed form ("Solving for U", "Parallel output") -----------

@pytest.mark.parametrize("with_state", [False, True])
def test_closed_form_full_sequence(with_state):
    rng = np.random.default_rng(8)
    n, dk, dv = 40, 6, 5
    Q = rng.standard_normal((n, dk)); K = unit_rows(rng, n, dk)
    V = rng.standard_normal((n, dv)); b = f32(rng.uniform(0, 1, n))
    S0 = rng.standard_normal((dk, dv)) if with_state else None
    O, S, _ = cw.full_sequence(Q, K, V, b, S0)
    out, fs = run(Q, K, V, b, S0)
    assert close(out, O, 1e-11) and close(fs, S, 1e-11)


# --- chunk form ("Chunkwise algorithm" .. "Complete per-chunk algorithm") -----

@pytest.mark.parametrize("C", [1, 2, 3, 16, 64, 100])
def test_chunkwise_equals_recurrence(C):
    """Every chunk size is exact; 100 tokens leaves a ragged last chunk."""
    rng = np.random.default_rng(9)
    n, dk, dv = 100, 8, 6
    Q = rng.standard_normal((n, dk)); K = unit_rows(rng, n, dk)
    V = rng.standard_normal((n, dv)); b = f32(rng.uniform(0, 1, n))
    S0 = rng.standard_normal((dk, dv))
    O, S = cw.chunkwise(Q, K, V, b, S0, C)
    out, fs = run(Q, K, V, b, S0)
    assert close(O, out, 1e-11) and close(S, fs, 1e-11)


def test_wy_rows_match_hand_expansion_and_triangular_solve():
    """w_1 = b1 k1, w_2 = b2 (k2 - (k2 k1^T) w1),
    w_3 = b3 (k3 - (k3 k1^T) w1 - (k3 k2^T) w2); stacked: (I + B L) W = B K."""
    rng = np.random.default_rng(10)
    K = rng.standard_normal((6, 5)); b = rng.uniform(0.1, 1, 6)
    W = cw.wy_rows(K, b)
    w1 = b[0] * K[0]
    w2 = b[1] * (K[1] - (K[1] @ K[0]) * w1)
    w3 = b[2] * (K[2] - (K[2] @ K[0]) * w1 - (K[2] @ K[1]) * w2)
    assert close(W[:3], np.stack([w1, w2, w3]))
    _, _, Wt, _ = cw.chunk_factors(K, None, b)
    assert close(W, Wt)


@pytest.mark.parametrize("c,d", [(1, 3), (4, 4), (8, 8), (7, 5)])
def test_wy_transition_product_brute_force(c, d):
    """Lambda[1:C] = I - K^T W against the ordered product of I - b k^T k."""
    rng = np.random.default_rng(11 + c)
    K = rng.standard_normal((c, d)); b = rng.uniform(0, 1, c)
    _, _, W, _ = cw.chunk_factors(K, None, b)
    assert close(np.eye(d) - K.T @ W, cw.ordered_product(K, b), 1e-12)


def test_local_writes_are_zero_start_state():
    """H_r = K_r^T U_r equals the state one chunk writes from a zero state."""
    rng = np.random.default_rng(12)
    c, dk, dv = 16, 8, 5
    K = unit_rows(rng, c, dk); V = rng.standard_normal((c, dv)); b = f32(rng.uniform(0, 1, c))
    _, _, _, U = cw.chunk_factors(K, V, b)
    _, fs = run(np.zeros((c, dk)), K, V, b)
    assert close(K.T @ U, fs)


# --- context parallelism ("Context Parallelism for DeltaNet", section 3) ------

@pytest.mark.parametrize("G", [1, 2, 3, 7, 13])
def test_segmented_scan_equals_serial(G):
    rng = np.random.default_rng(13)
    n, dk, dv, C = 13 * 8 - 3, 8, 6, 8
    Q = rng.standard_normal((n, dk)); K = unit_rows(rng, n, dk)
    V = rng.standard_normal((n, dv)); b = f32(rng.uniform(0, 1, n))
    S0 = rng.standard_normal((dk, dv))
    O, S, starts = cw.context_parallel(Q, K, V, b, S0, C, G)
    out, fs = run(Q, K, V, b, S0)
    assert close(O, out, 1e-11) and close(S, fs, 1e-11)


def test_segment_map_brute_force():
    """(P, H) of a segment: P is the ordered product of every token transition
    and H is the zero-start state."""
    rng = np.random.default_rng(14)
    n, dk, dv = 21, 5, 3
    K = rng.standard_normal((n, dk)) * 0.5; V = rng.standard_normal((n, dv))
    b = f32(rng.uniform(0, 1, n))
    P, H = cw.segment_map(K, V, b, C=4)
    assert close(P, cw.ordered_product(K, b), 1e-12)
    _, fs = run(np.zeros((n, dk)), K, V, b)
    assert close(H, fs, 1e-12)


def test_final_state_affine_in_initial_state():
    """F(a S + b S') = a F(S) + b F(S') + (1 - a - b) F(0)."""
    rng = np.random.default_rng(15)
    n, dk, dv = 30, 6, 4
    Q = rng.standard_normal((n, dk)); K = unit_rows(rng, n, dk)
    V = rng.standard_normal((n, dv)); b = f32(rng.uniform(0, 1, n))
    Sa = rng.standard_normal((dk, dv)); Sb = rng.standard_normal((dk, dv))
    x, y = 0.7, -1.3
    _, F = run(Q, K, V, b, x * Sa + y * Sb)
    _, Fa = run(Q, K, V, b, Sa)
    _, Fb = run(Q, K, V, b, Sb)
    _, F0 = run(Q, K, V, b, None)
    assert close(F, x * Fa + y * Fb + (1 - x - y) * F0, 1e-11)


def test_transition_is_contractive():
    """Each factor I - b k^T k (unit k, 0 <= b <= 1) has eigenvalues 1 and 1 - b,
    so the segment transition has spectral norm <= 1."""
    rng = np.random.default_rng(16)
    K = unit_rows(rng, 200, 8); b = rng.uniform(0, 1, 200)
    P, _ = cw.segment_map(K, np.zeros((200, 1)), b, C=16)
    assert np.linalg.norm(P, 2) <= 1 + 1e-12


# --- plumbing of the C oracle --------------------------------------------------

def test_varlen_packing_equals_separate_calls():
    """Each packed sequence restarts from its own initial state."""
    rng = np.random.default_rng(17)
    lens = [5, 0, 17, 1, 9]
    H, dk, dv = 2, 6, 4
    T = sum(lens)
    q = torch.randn(1, T, H, dk, dtype=torch.float64)
    k = torch.nn.functional.normalize(torch.randn(1, T, H, dk, dtype=torch.float64), dim=-1)
    v = torch.randn(1, T, H, dv, dtype=torch.float64)
    beta = torch.rand(1, T, H)
    s0 = torch.randn(len(lens), H, dk, dv, dtype=torch.float64)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32)
    out, fs = oracle.token_recurrence(q, k, v, beta, s0, cu)
    for n, (a, L) in enumerate(zip(cu[:-1].tolist(), lens)):
        for h in range(H):
            o_n, f_n = run(q[0, a:a + L, h].numpy(), k[0, a:a + L, h].numpy(),
                           v[0, a:a + L, h].numpy(), beta[0, a:a + L, h].numpy(),
                           s0[n, h].numpy())
            assert np.array_equal(out[0, a:a + L, h].numpy(), o_n)
            assert np.array_equal(fs[n, h].numpy(), f_n)


def test_bf16_inputs_are_widened_exactly():
    g = torch.Generator().manual_seed(0)
    q = torch.randn(2, 33, 3, 8, generator=g).to(torch.bfloat16)
    k = torch.randn(2, 33, 3, 8, generator=g).to(torch.bfloat16)
    v = torch.randn(2, 33, 3, 4, generator=g).to(torch.bfloat16)
    beta = torch.rand(2, 33, 3, generator=g)
    o1, f1 = oracle.token_recurrence(q, k, v, beta)
    o2, f2 = oracle.token_recurrence(q.double(), k.double(), v.double(), beta)
    assert torch.equal(o1, o2) and torch.equal(f1, f2)


def test_head_subset_and_fp32_output():
    g = torch.Generator().manual_seed(1)
    q = torch.randn(1, 20, 4, 8, generator=g)
    k = torch.randn(1, 20, 4, 8, generator=g)
    v = torch.randn(1, 20, 4, 8, generator=g)
    beta = torch.rand(1, 20, 4, generator=g)
    o_all, f_all = oracle.token_recurrence(q, k, v, beta)
    o_sub, f_sub = oracle.token_recurrence(q, k, v, beta, heads=(1, 3), out_dtype=torch.float32)
    assert torch.equal(o_sub[:, :, 1:3], o_all[:, :, 1:3].float())
    assert torch.equal(f_sub[:, 1:3], f_all[:, 1:3])
    assert torch.isnan(o_sub[:, :, 0]).all() and torch.isnan(f_sub[:, 3]).all()


def test_oracle_rejects_bad_seqlens():
    q = torch.zeros(1, 4, 1, 2, dtype=torch.float64)
    with pytest.raises(ValueError):
        oracle.token_recurrence(q, q, q, torch.zeros(1, 4, 1),
                                cu_seqlens=torch.tensor([0, 3, 2, 4], dtype=torch.int32))


# --- the pins reject plausible mistakes ----------------------------------------

def _mutant(kind, Q, K, V, beta, S0=None):
    """A deliberately wrong token recurrence (numpy), one mistake per kind."""
    n, dk = K.shape
    S = np.zeros((dk, V.shape[1])) if S0 is None else S0.copy()
    O = np.zeros((n, V.shape[1]))
    for t in range(n):
        vhat = K[t] @ S
        b = 1.0 if kind == "drop_beta" else beta[t]
        u = b * (V[t] + vhat) if kind == "sign" else b * (V[t] - vhat)
        if kind == "read_before_write":
            O[t] = Q[t] @ S
        S = S + np.outer(K[t], u)
        if kind != "read_before_write":
            O[t] = (K[t] if kind == "key_readout" else Q[t]) @ S
    return O, S


@pytest.mark.parametrize("kind", ["drop_beta", "sign", "read_before_write", "key_readout"])
def test_planted_mistakes_are_caught(kind):
    """The closed form and the hand expansion reject each planted mistake."""
    rng = np.random.default_rng(18)
    n, dk, dv = 10, 6, 4
    Q = rng.standard_normal((n, dk)); K = unit_rows(rng, n, dk)
    V = rng.standard_normal((n, dv)); b = f32(rng.uniform(0.1, 0.9, n))
    O, S, _ = cw.full_sequence(Q, K, V, b)
    Om, Sm = _mutant(kind, Q, K, V, b)
    assert not (close(Om, O, 1e-6) and close(Sm, S, 1e-6))
    Oc, Sc = _mutant("none", Q, K, V, b)
    assert close(Oc, O, 1e-11) and close(Sc, S, 1e-11)
