"""The algebra the two-pass path uses for the truncated Neumann inverse at chunk
128: the chunk run as two 64-token halves, each with its own factor, the second
half's E corrected by Y E1 with Y = Atil21 Atil11^{-1} + Atil22 Ntil21 (Atil the
series of Ntil = diag(beta) G, beta on the rows).  Checked in float64 numpy on
small random chunks (here halves of h tokens) against one step of the whole
chunk with the same truncated inverse; no oracle or kernel code is involved."""
import numpy as np
import pytest


def neumann(N, order, resid):
    """Order-`order` Neumann series of (I + N)^{-1} by Horner's rule, then `resid`
    Newton steps X <- X + X (I - (I + N) X)."""
    n = N.shape[0]
    I = np.eye(n)
    X = I.copy()
    for _ in range(order):
        X = I - N @ X
    for _ in range(resid):
        X = X + X @ (I - (I + N) @ X)
    return X


def one_step_neumann(M, blk):
    """1-Step Neumann approximation of (I + M)^{-1}: with D the block-diagonal part
    of I + M in blocks of `blk` rows, D^{-1} - D^{-1} M_off D^{-1}."""
    n = M.shape[0]
    D = np.eye(n)
    for b0 in range(0, n, blk):
        s = slice(b0, min(n, b0 + blk))
        D[s, s] += M[s, s]
    Dinv = np.linalg.inv(D)
    return Dinv - Dinv @ (M - (D - np.eye(n))) @ Dinv


def chunk_step(q, k, v, lam, beta, S, A_of):
    """One chunk of the chunkwise form: decays relative to the chunk start
    (lam[t] = Lambda_t per channel, lam[-1] the chunk end), T = diag(beta) A(M)."""
    C = k.shape[0]
    Kbar = k * np.exp(lam)
    Khat = k * np.exp(lam[-1] - lam)
    Qbar = q * np.exp(lam)
    G = np.zeros((C, C))
    L = np.zeros((C, C))
    for t in range(C):
        for j in range(t + 1):
            d = np.exp(lam[t] - lam[j])
            if j < t:
                G[t, j] = np.sum(k[t] * k[j] * d)
            L[t, j] = np.sum(q[t] * k[j] * d)
    M = G * beta[None, :]
    T = beta[:, None] * A_of(M)
    E = T @ (v - Kbar @ S)
    O = Qbar @ S + L @ E
    S_new = np.exp(lam[-1])[:, None] * S + Khat.T @ E
    return O, S_new, E, G


@pytest.mark.parametrize("h,order,resid,seed", [(8, 4, 1, 0), (8, 2, 0, 1), (6, 3, 2, 2),
                                                (16, 4, 1, 3), (5, 0, 1, 4), (8, -1, 4, 5),
                                                (12, -1, 4, 6)])
def test_pair_correction_reproduces_the_whole_chunk(h, order, resid, seed):
    """order >= 0: truncated Neumann of that order with `resid` Newton steps;
    order -1: 1-Step Neumann in blocks of `resid` rows (blocks inside each half)."""
    rng = np.random.default_rng(seed)
    dk, dv, C = 6, 5, 2 * h
    q = rng.standard_normal((C, dk))
    k = rng.standard_normal((C, dk))
    k /= np.linalg.norm(k, axis=1, keepdims=True)
    v = rng.standard_normal((C, dv))
    g = -np.log1p(np.exp(rng.standard_normal((C, dk))))      # -softplus, per channel
    beta = 1 / (1 + np.exp(-rng.standard_normal(C)))
    S = 0.3 * rng.standard_normal((dk, dv))
    A_of = ((lambda M: neumann(M, order, resid)) if order >= 0
            else (lambda M: one_step_neumann(M, resid)))
    lam = np.cumsum(g, axis=0)
    O_ref, S_ref, _, G = chunk_step(q, k, v, lam, beta, S, A_of)

    # the halves, each with decays relative to its own start
    a, b = slice(0, h), slice(h, C)
    lam1 = np.cumsum(g[a], axis=0)
    lam2 = np.cumsum(g[b], axis=0)
    O1, S_mid, E1, _ = chunk_step(q[a], k[a], v[a], lam1, beta[a], S, A_of)
    # the correction from the 2h-token series in the beta-on-rows form
    Ntil = beta[:, None] * G
    Atil = A_of(Ntil)
    Y = Atil[b, a] @ np.linalg.inv(Atil[a, a]) + Atil[b, b] @ Ntil[b, a]
    # half 2 as the state pass runs it: its own factors from S_mid, plus Y E1 in E
    Kbar2 = k[b] * np.exp(lam2)
    Khat2 = k[b] * np.exp(lam2[-1] - lam2)
    Qbar2 = q[b] * np.exp(lam2)
    G2 = G[b, b]
    L2 = np.zeros((h, h))
    for t in range(h):
        for j in range(t + 1):
            L2[t, j] = np.sum(q[h + t] * k[h + j] * np.exp(lam2[t] - lam2[j]))
    T2 = beta[b][:, None] * A_of(G2 * beta[b][None, :])
    E2 = T2 @ (v[b] - Kbar2 @ S_mid) + Y @ E1
    O2 = Qbar2 @ S_mid + L2 @ E2
    S_end = np.exp(lam2[-1])[:, None] * S_mid + Khat2.T @ E2
    O = np.concatenate([O1, O2])
    assert np.abs(O - O_ref).max() <= 1e-10 * np.abs(O_ref).max()
    assert np.abs(S_end - S_ref).max() <= 1e-10 * np.abs(S_ref).max()
    # and the correction is not trivially zero when the series is truncated
    if 0 <= order < C - 1 and resid == 0:
        assert np.abs(Y @ E1).max() > 1e-8


def test_exact_inverse_needs_no_correction():
    rng = np.random.default_rng(9)
    C, h, dk = 12, 6, 4
    k = rng.standard_normal((C, dk))
    g = -np.log1p(np.exp(rng.standard_normal((C, dk))))
    beta = 1 / (1 + np.exp(-rng.standard_normal(C)))
    lam = np.cumsum(g, axis=0)
    G = np.zeros((C, C))
    for t in range(C):
        for j in range(t):
            G[t, j] = np.sum(k[t] * k[j] * np.exp(lam[t] - lam[j]))
    Ntil = beta[:, None] * G
    Atil = np.linalg.inv(np.eye(C) + Ntil)
    a, b = slice(0, h), slice(h, C)
    Y = Atil[b, a] @ np.linalg.inv(Atil[a, a]) + Atil[b, b] @ Ntil[b, a]
    assert np.abs(Y).max() < 1e-12
