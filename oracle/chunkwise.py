"""Float64 numpy statements of DeltaNet's chunk form, for tiny inputs.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).  These functions are a
second, independent oracle: they follow the algebra of "Linear Attention,
Visualized" (section "DeltaNet: correcting memory collisions") step by step,
one (sequence, head) at a time, in the page's row-vector convention:
S is d_k x d_v, reads are ``k S`` and ``q S``.  Library primitives used as
steps: matrix products and a triangular solve.

Every function takes K, Q as [n, d_k], V as [n, d_v], beta as [n], S0 as
[d_k, d_v] (all float64 numpy arrays).
"""
from __future__ import annotations

import numpy as np
from scipy.linalg import solve_triangular


def causal_masks(n: int):
    """Inclusive causal mask M and its strict part M^- = M - I (section
    "The triangular correction system")."""
    M = np.tril(np.ones((n, n)))
    return M, M - np.eye(n)


def full_sequence(Q, K, V, beta, S0=None):
    """Full-sequence parallel form (subsections "The triangular correction
    system", "Solving for U" and "Parallel output").

    L = (K K^T) o M^-, (I + B L) U = B V, O = (Q K^T o M) U.  The page starts from
    S0 = 0; with a nonzero incoming state the prediction gains the term k_t S0,
    so the right-hand side becomes B (V - K S0), the readout gains Q S0 and the
    final state is S0 + K^T U (the same substitution the page makes for a chunk
    in "Correct the incoming state").
    Returns (O, S_final, U).
    """
    n, dk = K.shape
    dv = V.shape[1]
    if S0 is None:
        S0 = np.zeros((dk, dv))
    M, Mm = causal_masks(n)
    Bm = np.diag(beta)
    L = (K @ K.T) * Mm
    A = np.eye(n) + Bm @ L                      # unit lower triangular
    R = Bm @ (V - K @ S0)
    U = solve_triangular(A, R, lower=True, unit_diagonal=True)
    O = Q @ S0 + ((Q @ K.T) * M) @ U
    return O, S0 + K.T @ U, U


def chunk_factors(Kc, Vc, bc):
    """Per-chunk factors of the "Complete per-chunk algorithm":
    L_r = (K_r K_r^T) o M_c^-, (I + B_r L_r) T_r = B_r, W_r = T_r K_r, U_r = T_r V_r.
    Returns (L, T, W, U)."""
    c = Kc.shape[0]
    _, Mm = causal_masks(c)
    Bm = np.diag(bc)
    L = (Kc @ Kc.T) * Mm
    T = solve_triangular(np.eye(c) + Bm @ L, Bm, lower=True, unit_diagonal=True)
    return L, T, T @ Kc, (T @ Vc if Vc is not None else None)


def chunk_step(Qc, Kc, Vc, bc, S):
    """One chunk of the boundary pass: Z = U - W S, O = Q S + (Q K^T o M_c) Z,
    S' = S + K^T Z.  Returns (O_chunk, S')."""
    M, _ = causal_masks(Kc.shape[0])
    _, _, W, U = chunk_factors(Kc, Vc, bc)
    Z = U - W @ S
    O = Qc @ S + ((Qc @ Kc.T) * M) @ Z
    return O, S + Kc.T @ Z


def chunk_bounds(n: int, C: int):
    """Chunks start at the sequence start; the last one may be shorter (a
    chunk of any size is exact, subsection "Cost")."""
    return [(s, min(n, s + C)) for s in range(0, n, C)]


def chunkwise(Q, K, V, beta, S0=None, C: int = 64):
    """The per-chunk algorithm threaded over all chunks from S0.
    Returns (O, S_final)."""
    n, dk = K.shape
    dv = V.shape[1]
    S = np.zeros((dk, dv)) if S0 is None else S0.copy()
    O = np.zeros((n, dv))
    for s, e in chunk_bounds(n, C):
        O[s:e], S = chunk_step(Q[s:e], K[s:e], V[s:e], beta[s:e], S)
    return O, S


def token_transition(k, b):
    """A_{r,l} = I - beta k^T k (subsection "One chunk as an affine recurrence")."""
    return np.eye(k.shape[0]) - b * np.outer(k, k)


def ordered_product(K, beta):
    """Lambda[1:n] = A_n ... A_1, multiplied out explicitly (later tokens on the
    left, since S^(l) = A_l S^(l-1) + X_l)."""
    P = np.eye(K.shape[1])
    for t in range(K.shape[0]):
        P = token_transition(K[t], beta[t]) @ P
    return P


def wy_rows(K, beta):
    """Rows of W_r built one transition at a time (subsection "Compact the
    transition product with WY"):
    w_l = beta_l (k_l - sum_{i<l} (k_l k_i^T) w_i)."""
    W = np.zeros_like(K)
    for l in range(K.shape[0]):
        acc = K[l].copy()
        for i in range(l):
            acc -= (K[l] @ K[i]) * W[i]
        W[l] = beta[l] * acc
    return W


def segment_map(K, V, beta, C: int = 64):
    """Affine map of a run of chunks: S_end = P S_start + H.

    The pages state the one-chunk case, S_{r+1} = Lambda_r[1:C] S_r + H_r with
    Lambda_r[1:C] = I - K_r^T W_r and H_r the zero-start local writes.  Composing
    two affine maps gives (P2, H2) o (P1, H1) = (P2 P1, P2 H1 + H2); a segment is
    the composition of its chunks, taken in chunk order.
    Returns (P [d_k, d_k], H [d_k, d_v]).
    """
    dk = K.shape[1]
    dv = V.shape[1]
    P = np.eye(dk)
    H = np.zeros((dk, dv))
    for s, e in chunk_bounds(K.shape[0], C):
        _, _, W, U = chunk_factors(K[s:e], V[s:e], beta[s:e])
        Lam = np.eye(dk) - K[s:e].T @ W
        Hr = K[s:e].T @ U
        P, H = Lam @ P, Lam @ H + Hr
    return P, H


def context_parallel(Q, K, V, beta, S0=None, C: int = 64, n_segments: int = 2):
    """Context parallelism over chunk segments ("Context Parallelism for
    DeltaNet", section 3): each segment summarises itself as (P_g, H_g), a short
    scan composes the true segment-start states, then every segment reruns its
    chunks from its own start state.  Exact, so it must equal ``chunkwise``.
    Returns (O, S_final, starts)."""
    n, dk = K.shape
    dv = V.shape[1]
    chunks = chunk_bounds(n, C)
    nc = len(chunks)
    n_segments = max(1, min(n_segments, nc))
    edges = [round(g * nc / n_segments) for g in range(n_segments + 1)]
    segs = [(chunks[edges[g]][0], chunks[edges[g + 1] - 1][1]) for g in range(n_segments)]
    maps = [segment_map(K[s:e], V[s:e], beta[s:e], C) for s, e in segs]
    starts = [np.zeros((dk, dv)) if S0 is None else S0.copy()]
    for P, H in maps[:-1]:
        starts.append(P @ starts[-1] + H)
    O = np.zeros((n, dv))
    S = None
    for (s, e), Sg in zip(segs, starts):
        O[s:e], S = chunkwise(Q[s:e], K[s:e], V[s:e], beta[s:e], Sg, C)
    return O, S, starts


def linear_attention(Q, K, V):
    """Causal linear attention, parallel form (Q K^T o M) V."""
    M, _ = causal_masks(K.shape[0])
    return ((Q @ K.T) * M) @ V


# --- Gated DeltaNet ("Linear Attention, Visualized", section "Gated DeltaNet (GDN)") ---
#
# Every function below takes the per-token decays a (shape [n], 0 < a <= 1)
# next to beta; the recurrence is S_t = a_t (I - beta_t k_t^T k_t) S_{t-1}
# + beta_t k_t^T v_t.

def decay_products(a):
    """lambda[i:j] = prod_{s=i}^{j} a_s with 1-based inclusive bounds, and 1 when
    i > j ("Complete per-chunk algorithm" of the GDN section)."""
    def lam(i, j):
        return float(np.prod(a[i - 1:j])) if i <= j else 1.0
    return lam


def gated_chunk_factors(Kc, Vc, bc, ac):
    """Per-chunk quantities of the GDN chunk algorithm, taken as the page
    defines them:
      Gamma[l, i] = lambda[i+1:l] for i <= l, else 0 (1-based l, i);
      left-decayed rows  q<-_l = lambda[1:l] q_l,  k<-_l = lambda[1:l] k_l;
      right-decayed rows k->_l = lambda[l+1:C] k_l;
      L = (K K^T o Gamma) o M_c^-, (I + B L) T = B, U = T V, W<- = T K<-.
    Returns a dict with Gamma, L, T, U, W (= W<-), Kl (= K<-), Kr (= K->),
    left (the lambda[1:l] column) and lamC (= lambda[1:C])."""
    c = Kc.shape[0]
    lam = decay_products(ac)
    Gam = np.zeros((c, c))
    for l in range(c):
        for i in range(l + 1):
            Gam[l, i] = lam(i + 2, l + 1)
    left = np.array([lam(1, l + 1) for l in range(c)])
    right = np.array([lam(l + 2, c) for l in range(c)])
    _, Mm = causal_masks(c)
    Bm = np.diag(bc)
    L = ((Kc @ Kc.T) * Gam) * Mm
    T = solve_triangular(np.eye(c) + Bm @ L, Bm, lower=True, unit_diagonal=True)
    Kl = left[:, None] * Kc
    Kr = right[:, None] * Kc
    return {"Gamma": Gam, "L": L, "T": T, "U": (T @ Vc if Vc is not None else None),
            "W": T @ Kl, "Kl": Kl, "Kr": Kr, "left": left, "lamC": lam(1, c)}


def gated_chunk_step(Qc, Kc, Vc, bc, ac, S):
    """One chunk of the GDN boundary pass: Z = U - W<- S,
    O = Q<- S + (Q K^T o Gamma) Z, S' = lambda[1:C] S + K->^T Z.
    Returns (O_chunk, S')."""
    f = gated_chunk_factors(Kc, Vc, bc, ac)
    Z = f["U"] - f["W"] @ S
    O = (f["left"][:, None] * Qc) @ S + ((Qc @ Kc.T) * f["Gamma"]) @ Z
    return O, f["lamC"] * S + f["Kr"].T @ Z


def gated_chunkwise(Q, K, V, beta, a, S0=None, C: int = 64):
    """The GDN per-chunk algorithm threaded over all chunks from S0.
    Returns (O, S_final)."""
    n, dk = K.shape
    dv = V.shape[1]
    S = np.zeros((dk, dv)) if S0 is None else S0.copy()
    O = np.zeros((n, dv))
    for s, e in chunk_bounds(n, C):
        O[s:e], S = gated_chunk_step(Q[s:e], K[s:e], V[s:e], beta[s:e], a[s:e], S)
    return O, S


def gated_segment_map(K, V, beta, a, C: int = 64):
    """Affine map S_end = P S_start + H of a run of chunks under GDN: one chunk
    is S' = (lambda[1:C] I - K->^T W<-) S + K->^T U, and chunks compose in order
    as in ``segment_map``.  Returns (P, H)."""
    dk = K.shape[1]
    P = np.eye(dk)
    H = np.zeros((dk, V.shape[1]))
    for s, e in chunk_bounds(K.shape[0], C):
        f = gated_chunk_factors(K[s:e], V[s:e], beta[s:e], a[s:e])
        Lam = f["lamC"] * np.eye(dk) - f["Kr"].T @ f["W"]
        Hr = f["Kr"].T @ f["U"]
        P, H = Lam @ P, Lam @ H + Hr
    return P, H


def gated_context_parallel(Q, K, V, beta, a, S0=None, C: int = 64, n_segments: int = 2):
    """``context_parallel`` with the GDN chunk maps.  Returns (O, S_final)."""
    n, dk = K.shape
    dv = V.shape[1]
    chunks = chunk_bounds(n, C)
    nc = len(chunks)
    n_segments = max(1, min(n_segments, nc))
    edges = [round(g * nc / n_segments) for g in range(n_segments + 1)]
    segs = [(chunks[edges[g]][0], chunks[edges[g + 1] - 1][1]) for g in range(n_segments)]
    maps = [gated_segment_map(K[s:e], V[s:e], beta[s:e], a[s:e], C) for s, e in segs]
    starts = [np.zeros((dk, dv)) if S0 is None else S0.copy()]
    for P, H in maps[:-1]:
        starts.append(P @ starts[-1] + H)
    O = np.zeros((n, dv))
    S = None
    for (s, e), Sg in zip(segs, starts):
        O[s:e], S = gated_chunkwise(Q[s:e], K[s:e], V[s:e], beta[s:e], a[s:e], Sg, C)
    return O, S


def decayed_linear_attention(Q, K, V, a):
    """Linear attention with scalar decay (the Mamba-2 row of the page's table,
    one chunk spanning the sequence, zero start): O = (Q K^T o D) V with
    D[t, s] = lambda[s+1:t] for s <= t."""
    n = K.shape[0]
    lam = decay_products(a)
    D = np.zeros((n, n))
    for t in range(n):
        for s in range(t + 1):
            D[t, s] = lam(s + 2, t + 1)
    return ((Q @ K.T) * D) @ V


# --- Gated Delta Product ("Linear Attention, Visualized", section "Gated Delta Product (GDP)") ---

def gdp_virtual_sequence(Q, K, V, beta, a, n_h: int):
    """The page's "GDP as GDN over a virtual sequence": token t's n_h substeps
    become virtual steps m = n_h (t - 1) + j; k, v, beta move over unchanged,
    the decay sits on the first substep (1 elsewhere) and the query on the last
    (0 elsewhere).  K, V, beta hold n_h rows per token (substep-major), Q and a
    one per token.  Returns (Qv, Kv, Vv, beta_v, a_v)."""
    n = Q.shape[0]
    Qv = np.zeros((n * n_h, Q.shape[1]))
    Qv[n_h - 1::n_h] = Q
    av = np.ones(n * n_h)
    av[0::n_h] = a
    return Qv, K, V, beta, av


def gdp_chunkwise(Q, K, V, beta, a, n_h: int, S0=None, C: int = 64):
    """GDP evaluated as the GDN chunk algorithm over the virtual sequence,
    keeping every n_h-th output.  Returns (O [n, d_v], S_final)."""
    Qv, Kv, Vv, bv, av = gdp_virtual_sequence(Q, K, V, beta, a, n_h)
    Ov, S = gated_chunkwise(Qv, Kv, Vv, bv, av, S0, C)
    return Ov[n_h - 1::n_h], S


def gdp_substeps(Q, K, V, beta, a, n_h: int, S0):
    """GDP's token update as the page writes it, with explicit d_k x d_k
    matrices: S_{t,0} = a_t S_{t-1}, S_{t,j} = A_{t,j} S_{t,j-1} + X_{t,j}
    (A = I - beta k^T k, X = beta k^T v), o_t = q_t S_{t,n_h}."""
    S = S0.copy()
    O = np.zeros((Q.shape[0], V.shape[1]))
    for t in range(Q.shape[0]):
        S = a[t] * S
        for j in range(n_h):
            m = t * n_h + j
            A = np.eye(K.shape[1]) - beta[m] * np.outer(K[m], K[m])
            S = A @ S + beta[m] * np.outer(K[m], V[m])
        O[t] = Q[t] @ S
    return O, S


# --- Gated Linear Attention and Kimi Delta Attention ("Linear Attention, Visualized",
#     sections "Gated Linear Attention (GLA)" and "Kimi Delta Attention (KDA)") ---
#
# Here the decay is a vector per token, A [n, d_k] with entries in (0, 1]: it
# scales row c of the state (key channel c) by A[t, c].

def channel_decay_products(A):
    """lambda[i:j] = a_i o ... o a_j (elementwise, 1-based inclusive), the ones
    vector when i > j."""
    def lam(i, j):
        return np.prod(A[i - 1:j], axis=0) if i <= j else np.ones(A.shape[1])
    return lam


def kda_chunk_factors(Qc, Kc, Vc, bc, Ac):
    """The KDA "Complete per-chunk algorithm", quantities as the page defines them:
      q<-_l = lambda[1:l] o q_l, k<-_l = lambda[1:l] o k_l, k->_l = lambda[l+1:C] o k_l;
      A[l, m] = q_l (lambda[m+1:l] o k_m)^T for m <= l; L[l, m] = k_l (lambda[m+1:l] o k_m)^T
      for m < l; (I + B L) T = B, U = T V, W<- = T K<-.
    Qc may be None (no readout)."""
    c = Kc.shape[0]
    lam = channel_decay_products(Ac)
    Ql = None if Qc is None else np.stack([lam(1, l + 1) * Qc[l] for l in range(c)])
    Kl = np.stack([lam(1, l + 1) * Kc[l] for l in range(c)])
    Kr = np.stack([lam(l + 2, c) * Kc[l] for l in range(c)])
    Am = np.zeros((c, c))
    L = np.zeros((c, c))
    for l in range(c):
        for m in range(l + 1):
            km = lam(m + 2, l + 1) * Kc[m]
            if Qc is not None:
                Am[l, m] = Qc[l] @ km
            if m < l:
                L[l, m] = Kc[l] @ km
    Bm = np.diag(bc)
    T = solve_triangular(np.eye(c) + Bm @ L, Bm, lower=True, unit_diagonal=True)
    return {"Ql": Ql, "Kl": Kl, "Kr": Kr, "A": Am, "L": L, "T": T,
            "U": (T @ Vc if Vc is not None else None), "W": T @ Kl, "lamC": lam(1, c)}


def kda_chunkwise(Q, K, V, beta, A, S0=None, C: int = 64):
    """KDA threaded over the chunks: Z = U - W<- S, O = Q<- S + A Z,
    S' = Diag(lambda[1:C]) S + K->^T Z.  Returns (O, S_final)."""
    n, dk = K.shape
    dv = V.shape[1]
    S = np.zeros((dk, dv)) if S0 is None else S0.copy()
    O = np.zeros((n, dv))
    for s, e in chunk_bounds(n, C):
        f = kda_chunk_factors(Q[s:e], K[s:e], V[s:e], beta[s:e], A[s:e])
        Z = f["U"] - f["W"] @ S
        O[s:e] = f["Ql"] @ S + f["A"] @ Z
        S = f["lamC"][:, None] * S + f["Kr"].T @ Z
    return O, S


def kda_segment_map(K, V, beta, A, C: int = 64):
    """S_end = P S_start + H of a run of chunks under KDA: one chunk is
    S' = (Diag(lambda[1:C]) - K->^T W<-) S + K->^T U; chunks compose in order."""
    dk = K.shape[1]
    P = np.eye(dk)
    H = np.zeros((dk, V.shape[1]))
    for s, e in chunk_bounds(K.shape[0], C):
        f = kda_chunk_factors(None, K[s:e], V[s:e], beta[s:e], A[s:e])
        Lam = np.diag(f["lamC"]) - f["Kr"].T @ f["W"]
        P, H = Lam @ P, Lam @ H + f["Kr"].T @ f["U"]
    return P, H


def gla_chunkwise(Q, K, V, A, S0=None, C: int = 64):
    """GLA's chunk form: O = Q<- S + A V, S' = Diag(lambda[1:C]) S + K->^T V."""
    n, dk = K.shape
    dv = V.shape[1]
    S = np.zeros((dk, dv)) if S0 is None else S0.copy()
    O = np.zeros((n, dv))
    for s, e in chunk_bounds(n, C):
        f = kda_chunk_factors(Q[s:e], K[s:e], V[s:e], np.zeros(e - s), A[s:e])
        O[s:e] = f["Ql"] @ S + f["A"] @ V[s:e]
        S = f["lamC"][:, None] * S + f["Kr"].T @ V[s:e]
    return O, S
