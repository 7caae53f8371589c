"""Pins for the fp64 oracle: checks against values and identities that the
pages and plain mathematics fix, never against the oracle itself retyped.

Each pin returns the largest error it saw (0 when the oracle is right up to
fp64 rounding).  tests/test_oracle_pins.py asserts each one, and
tests/test_oracle_mutants.py re-runs the whole list on deliberately broken
builds of the oracle to show that every planted mistake trips at least one.
"""
from __future__ import annotations

import json
import os

import numpy as np

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden",
                      "hand_worked_delta.json")


def _rel(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    den = max(np.abs(b).max(), 1e-300) if b.size else 1.0
    return float(np.abs(a - b).max() / den) if a.size else 0.0


def rand_inputs(rng, B, T, Hk, Hv, dk, dv, G, s0=True, decay=1.0, beta_scale=1.0):
    q = rng.standard_normal((B, Hk, T, dk))
    k = rng.standard_normal((B, Hk, T, dk))
    q /= np.linalg.norm(q, axis=-1, keepdims=True)
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, Hv, T, dv))
    g = -np.logaddexp(0.0, rng.standard_normal((B, Hk, T, G))) * decay
    beta = beta_scale / (1.0 + np.exp(-rng.standard_normal((B, Hk, T))))
    S0 = rng.standard_normal((B, Hv, dk, dv)) * 0.5 if s0 else None
    return q, k, v, g, beta, S0


def _both_forms(q, k, v, g, beta, S0, chunks=(1, 2, 3, 64)):
    """Yield (label, o, S_final) for the token recurrence and chunked forms."""
    yield ("recurrent",) + oracle.recurrent(q, k, v, g, beta, S0)
    for C in chunks:
        yield ("chunked C=%d" % C,) + oracle.chunked(q, k, v, g, beta, S0, chunk=C)


# ---------------------------------------------------------------------------
# P0: hand-worked examples (tests/golden), both oracle forms.
def pin_golden_examples():
    with open(GOLDEN) as f:
        gold = json.load(f)
    worst = 0.0
    for case in gold["cases"]:
        arr = {n: (None if case[n] is None else np.array(case[n], np.float64))
               for n in ("q", "k", "v", "g", "beta", "S0", "o", "S_final")}
        for _, o, Sf in _both_forms(arr["q"], arr["k"], arr["v"], arr["g"], arr["beta"],
                                    arr["S0"], chunks=(1, 2, 4)):
            worst = max(worst, np.abs(o - arr["o"]).max(), np.abs(Sf - arr["S_final"]).max())
    return worst


def pin_golden_inverse():
    with open(GOLDEN) as f:
        gold = json.load(f)
    worst = 0.0
    for case in gold["inverse_cases"]:
        N = np.array(case["N"], np.float64)
        worst = max(worst, np.abs(oracle.tril_inverse(N) - case["inverse"]).max())
        worst = max(worst, np.abs(oracle.neumann_inverse(N, order=1, resid=0)
                                  - case["order1_no_resid"]).max())
        worst = max(worst, np.abs(oracle.neumann_inverse(N, order=1, resid=1)
                                  - case["inverse"]).max())
        worst = max(worst, np.abs(oracle.neumann_inverse(N, order=2, resid=0)
                                  - case["inverse"]).max())
    return worst


# ---------------------------------------------------------------------------
# P2/P3: beta = 0 leaves only the decay of S0 ("pure decay"):
#   S_T = diag(exp(Lam_T)) S0,  o_t = S0^T (exp(Lam_t) * q_t),  Lam_t = cumsum g.
def pin_pure_decay(seed=1):
    rng = np.random.default_rng(seed)
    worst = 0.0
    for (dk, G) in ((8, 1), (8, 2), (8, 8)):
        B, T, Hk, Hv, dv = 2, 11, 2, 4, 3
        q, k, v, g, beta, S0 = rand_inputs(rng, B, T, Hk, Hv, dk, dv, G)
        beta = np.zeros_like(beta)
        R = Hv // Hk
        ch = (np.arange(dk) * G) // dk
        lam = np.cumsum(g[..., ch], axis=2)                      # [B,Hk,T,dk]
        lam_v = np.repeat(lam, R, axis=1)                        # value heads
        q_v = np.repeat(q, R, axis=1)
        o_ref = np.einsum("bhti,bhin->bhtn", q_v * np.exp(lam_v), S0)
        S_ref = np.exp(lam_v[:, :, -1, :])[..., None] * S0
        for _, o, Sf in _both_forms(q, k, v, g, beta, S0, chunks=(1, 4, 5)):
            worst = max(worst, _rel(o, o_ref), _rel(Sf, S_ref))
        # g = 0 as well: the state is left untouched.
        g0 = np.zeros_like(g)
        o_ref0 = np.einsum("bhti,bhin->bhtn", q_v, S0)
        for _, o, Sf in _both_forms(q, k, v, g0, beta, S0, chunks=(3,)):
            worst = max(worst, _rel(o, o_ref0), _rel(Sf, S0))
    return worst


# ---------------------------------------------------------------------------
# P4: keys that are distinct standard basis vectors never interfere, so the
# delta rule reduces to gated causal linear attention:
#   o_t = sum_{j<=t} beta_j q_t[p(j)] exp(Lam_t[p(j)] - Lam_j[p(j)]) v_j.
# With orthonormal keys and no decay: o = tril(Q K^T) diag(beta) V.
def pin_linear_attention(seed=2):
    rng = np.random.default_rng(seed)
    worst = 0.0
    B, Hk, Hv, dk, dv, T = 1, 1, 2, 16, 5, 12
    for G in (1, 4, 16):
        q, _, v, g, beta, _ = rand_inputs(rng, B, T, Hk, Hv, dk, dv, G)
        perm = rng.permutation(dk)[:T]
        k = np.zeros((B, Hk, T, dk))
        k[0, 0, np.arange(T), perm] = 1.0
        ch = (np.arange(dk) * G) // dk
        lam = np.cumsum(g[..., ch], axis=2)[0, 0]                # [T,dk]
        o_ref = np.zeros((B, Hv, T, dv))
        S_ref = np.zeros((B, Hv, dk, dv))
        for hv in range(Hv):
            for t in range(T):
                for j in range(t + 1):
                    p = perm[j]
                    w = beta[0, 0, j] * q[0, 0, t, p] * np.exp(lam[t, p] - lam[j, p])
                    o_ref[0, hv, t] += w * v[0, hv, j]
            for j in range(T):
                p = perm[j]
                S_ref[0, hv, p] += beta[0, 0, j] * np.exp(lam[-1, p] - lam[j, p]) * v[0, hv, j]
        for _, o, Sf in _both_forms(q, k, v, g, beta, None, chunks=(1, 4, 5, 12)):
            worst = max(worst, _rel(o, o_ref), _rel(Sf, S_ref))
    # orthonormal (rotated) keys, no decay: plain causal linear attention
    Qo, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
    k = Qo[:T][None, None]
    q, _, v, _, beta, _ = rand_inputs(rng, B, T, Hk, Hv, dk, dv, 1)
    g = np.zeros((B, Hk, T, 1))
    scores = np.tril(q[0, 0] @ k[0, 0].T) * beta[0, 0][None, :]
    o_ref = np.einsum("tj,hjn->htn", scores, v[0])[None]
    for _, o, Sf in _both_forms(q, k, v, g, beta, None, chunks=(3, 8)):
        worst = max(worst, _rel(o, o_ref))
    return worst


# ---------------------------------------------------------------------------
# P5: the token recurrence and the chunked dense-inverse form reach the same
# result (the WY equivalence of the SLA paper, §2.4.2), for every gate mode,
# chunk size, grouped-value ratio and a ragged last chunk.
def pin_chunked_equals_recurrent(seed=3):
    rng = np.random.default_rng(seed)
    worst = 0.0
    for (dk, G, Hk, Hv, T, C) in ((4, 1, 1, 1, 9, 2), (8, 2, 2, 4, 21, 4), (8, 8, 1, 2, 40, 16),
                                  (64, 1, 2, 2, 130, 64), (64, 64, 1, 4, 100, 16),
                                  (64, 4, 1, 1, 64, 64), (16, 4, 2, 8, 33, 8)):
        q, k, v, g, beta, S0 = rand_inputs(rng, 1, T, Hk, Hv, dk, 3, G)
        o1, S1 = oracle.recurrent(q, k, v, g, beta, S0)
        o2, S2 = oracle.chunked(q, k, v, g, beta, S0, chunk=C)
        worst = max(worst, _rel(o2, o1), _rel(S2, S1))
    return worst


# ---------------------------------------------------------------------------
# P6: (I + M) A = I for the exact inverse; Neumann is exact at order >= n-1.
def pin_inverse_identity(seed=4):
    rng = np.random.default_rng(seed)
    worst = 0.0
    for n in (1, 2, 5, 16, 64):
        N = np.tril(rng.standard_normal((n, n)) * 0.3, -1)
        X = oracle.tril_inverse(N)
        worst = max(worst, np.abs((np.eye(n) + N) @ X - np.eye(n)).max())
        worst = max(worst, np.abs(np.triu(X, 1)).max())
        Xn = oracle.neumann_inverse(N, order=max(n - 1, 0), resid=0)
        worst = max(worst, np.abs(Xn - X).max() / max(1.0, np.abs(X).max()))
        Xn = oracle.neumann_inverse(N, order=n, resid=0)
        worst = max(worst, np.abs(Xn - X).max() / max(1.0, np.abs(X).max()))
    return worst


# ---------------------------------------------------------------------------
# P7: band exactness (Lemma 3.1 of the Neumann-inversion paper: N^p vanishes on
# i - j < p).  X0 of order m is exact on i - j <= m and wrong at i - j = m + 1;
# one Newton/refine step makes it exact on i - j <= 2m + 1; a second Newton
# step doubles again (4m + 3), a second refine step adds m + 1 (3m + 2).
def pin_neumann_bands(seed=5):
    rng = np.random.default_rng(seed)
    n = 40
    N = np.tril(rng.uniform(0.2, 1.0, (n, n)), -1)  # positive: no accidental zeros
    X = oracle.tril_inverse(N)
    ij = np.subtract.outer(np.arange(n), np.arange(n))
    worst = 0.0
    for m in (1, 2, 3, 4):
        for resid, variant, band in ((0, oracle.NV_NEWTON, m), (1, oracle.NV_NEWTON, 2 * m + 1),
                                     (2, oracle.NV_NEWTON, 4 * m + 3),
                                     (2, oracle.NV_REFINE, 3 * m + 2)):
            Xa = oracle.neumann_inverse(N, order=m, resid=resid, variant=variant)
            inside = (ij >= 0) & (ij <= band)
            scale = np.abs(X[inside]).max()
            worst = max(worst, np.abs(Xa - X)[inside].max() / scale)
            if band + 1 < n:
                edge = ij == band + 1
                if np.abs(Xa - X)[edge].max() < 1e-6 * scale:
                    worst = max(worst, 1.0)   # should NOT be exact just past the band
    return worst


# P8: error bound of the truncated series for ||N||_2 < 1:
#   ||(I+N)^{-1} - X0||_2 <= ||N||_2^{m+1} / (1 - ||N||_2).
def pin_neumann_error_bound(seed=6):
    rng = np.random.default_rng(seed)
    viol = 0.0
    for n in (8, 32, 64):
        N = np.tril(rng.standard_normal((n, n)), -1)
        N *= 0.7 / np.linalg.norm(N, 2)
        X = oracle.tril_inverse(N)
        nrm = np.linalg.norm(N, 2)
        prev = None
        for m in range(0, 8):
            err = np.linalg.norm(X - oracle.neumann_inverse(N, order=m, resid=0), 2)
            bound = nrm ** (m + 1) / (1 - nrm)
            viol = max(viol, max(0.0, err - bound) / bound)
            if prev is not None and err > prev * (1 + 1e-12):
                viol = max(viol, 1.0)        # error must not grow with the order
            prev = err
    return viol


# ---------------------------------------------------------------------------
# P9: chunk matrices against the SLA Table 2 decay masks built from products of
# decays (Psi_g[t,j] = prod_{s=j+1..t} gamma_{s,g}; Gamma_g = beta_j Psi_g for
# t > j), i.e. M = sum_g Gamma_g * (K_g K_g^T), L = sum_g Psi_g * (Q_g K_g^T)
# (SLA §2.4.2) -- a product route, not the exp-of-difference route the oracle
# takes.
def pin_grouped_gram(seed=7):
    rng = np.random.default_rng(seed)
    worst = 0.0
    for dk, G in ((8, 1), (16, 4), (8, 8)):
        C = 12
        qc = rng.standard_normal((C, dk))
        kc = rng.standard_normal((C, dk))
        gc = -np.logaddexp(0, rng.standard_normal((C, G)))
        bc = rng.uniform(0.1, 1.0, C)
        Lam, M, L = oracle.chunk_matrices(qc, kc, gc, bc)
        gam = np.exp(gc)
        width = dk // G
        Mr = np.zeros((C, C))
        Lr = np.zeros((C, C))
        for gi in range(G):
            sl = slice(gi * width, (gi + 1) * width)
            Psi = np.zeros((C, C))
            for t in range(C):
                for j in range(t + 1):
                    Psi[t, j] = np.prod(gam[j + 1:t + 1, gi])
            Gam = np.tril(Psi, -1) * bc[None, :]
            Mr += Gam * (kc[:, sl] @ kc[:, sl].T)
            Lr += Psi * (qc[:, sl] @ kc[:, sl].T)
        lam_ref = np.cumsum(gc[:, (np.arange(dk) * G) // dk], axis=0)
        worst = max(worst, _rel(M, Mr), _rel(L, Lr), _rel(Lam, lam_ref))
    return worst


# ---------------------------------------------------------------------------
# P10: gate-mode consistency.  Per-channel decay with equal channels equals the
# scalar gate; a 64-channel-group gate expanded to channels equals itself.
def pin_gate_consistency(seed=8):
    rng = np.random.default_rng(seed)
    worst = 0.0
    dk, T = 128, 37
    q, k, v, g1, beta, S0 = rand_inputs(rng, 1, T, 1, 2, dk, 4, 1)
    gdk = np.repeat(g1, dk, axis=-1)
    for fn in (lambda *a: oracle.recurrent(*a), lambda *a: oracle.chunked(*a, chunk=16)):
        o1, S1 = fn(q, k, v, g1, beta, S0)
        o2, S2 = fn(q, k, v, gdk, beta, S0)
        worst = max(worst, _rel(o2, o1), _rel(S2, S1))
    _, _, _, g2, _, _ = rand_inputs(rng, 1, T, 1, 2, dk, 4, 2)
    g2x = np.repeat(g2, dk // 2, axis=-1)
    o1, S1 = oracle.recurrent(q, k, v, g2, beta, S0)
    o2, S2 = oracle.chunked(q, k, v, g2x, beta, S0, chunk=8)
    worst = max(worst, _rel(o2, o1), _rel(S2, S1))
    return worst


# P11: grouped value heads: R value heads packed on one key head equal R
# independent single-head runs that share q, k, g, beta (SLA §2.4.1).
def pin_gva(seed=9):
    rng = np.random.default_rng(seed)
    B, T, Hk, R, dk, dv = 2, 19, 2, 4, 8, 3
    q, k, v, g, beta, S0 = rand_inputs(rng, B, T, Hk, Hk * R, dk, dv, 2)
    worst = 0.0
    for fn in (lambda *a: oracle.recurrent(*a), lambda *a: oracle.chunked(*a, chunk=4)):
        o, Sf = fn(q, k, v, g, beta, S0)
        for b in range(B):
            for hv in range(Hk * R):
                hk = hv // R
                sl = lambda a: a[b:b + 1, hk:hk + 1]
                o1, S1 = fn(sl(q), sl(k), v[b:b + 1, hv:hv + 1], sl(g), sl(beta),
                            S0[b:b + 1, hv:hv + 1])
                worst = max(worst, _rel(o[b, hv], o1[0, 0]), _rel(Sf[b, hv], S1[0, 0]))
    return worst


# P12: resume: one run over T equals a run over T1 followed by a run over the
# rest started from the first run's final state.
def pin_resume(seed=10):
    rng = np.random.default_rng(seed)
    T, T1 = 50, 23
    q, k, v, g, beta, S0 = rand_inputs(rng, 1, T, 2, 2, 8, 3, 8)
    worst = 0.0
    for fn in (lambda *a: oracle.recurrent(*a), lambda *a: oracle.chunked(*a, chunk=8)):
        o, Sf = fn(q, k, v, g, beta, S0)
        oa, Sa = fn(q[:, :, :T1], k[:, :, :T1], v[:, :, :T1], g[:, :, :T1], beta[:, :, :T1], S0)
        ob, Sb = fn(q[:, :, T1:], k[:, :, T1:], v[:, :, T1:], g[:, :, T1:], beta[:, :, T1:], Sa)
        worst = max(worst, _rel(np.concatenate([oa, ob], axis=2), o), _rel(Sb, Sf))
    return worst


# P12b: the state after a stretch of tokens is affine in the state before it,
# S_end = A S_start + B, with A the end state from the identity when no value is
# written (v = 0, state dk x dk) and B the end state from zero; composing two
# stretches' maps gives the state of one pass over both (the segment-parallel
# state pass composes such maps).
def pin_affine_segments(seed=12):
    rng = np.random.default_rng(seed)
    T, T1, dk, dv = 40, 17, 8, 5
    q, k, v, g, beta, S0 = rand_inputs(rng, 1, T, 1, 1, dk, dv, dk)
    _, Sf = oracle.recurrent(q, k, v, g, beta, S0)

    def maps(sl):
        qs, ks, vs, gs, bs = q[:, :, sl], k[:, :, sl], v[:, :, sl], g[:, :, sl], beta[:, :, sl]
        zero_v = np.zeros(vs.shape[:3] + (dk,))
        _, A = oracle.recurrent(qs, ks, zero_v, gs, bs, np.eye(dk)[None, None])
        _, Bm = oracle.recurrent(qs, ks, vs, gs, bs, None)
        return A[0, 0], Bm[0, 0]

    A1, B1 = maps(slice(0, T1))
    A2, B2 = maps(slice(T1, T))
    S_seg = A2 @ (A1 @ S0[0, 0] + B1) + B2
    return _rel(S_seg, Sf[0, 0])


# P13: the chunked Neumann mode at order >= C-1 is the exact chunked form; at
# low order on a contractive chunk it stays close (reported, loosely bounded).
def pin_chunked_neumann(seed=11):
    rng = np.random.default_rng(seed)
    q, k, v, g, beta, S0 = rand_inputs(rng, 1, 48, 1, 2, 16, 4, 4)
    o1, S1 = oracle.chunked(q, k, v, g, beta, S0, chunk=16)
    o2, S2 = oracle.chunked(q, k, v, g, beta, S0, chunk=16, inverse="neumann", order=15, resid=0)
    return max(_rel(o2, o1), _rel(S2, S1))


# P13 ("Systolic Linear Attention ...", §2.4.3, block-doubling and block-Neumann
# factorization): with 8 blocks of 16 at C = 128, Nb = D^{-1} N_off (D the
# block-diagonal part of I + N) is nilpotent, so sum_{s<=7} (-Nb)^s equals
# (I + Nb^4)(I + Nb^2)(I - Nb) and sum_s (-Nb)^s D^{-1} is the exact inverse.  The
# oracle's 1-Step Neumann must be the exact inverse minus the pages' truncation
# sum_{s=2}^{7} (-Nb)^s D^{-1}; it is exact on the diagonal blocks and the first
# block sub-diagonal.  D^{-1}, the exact inverse and the powers come from LAPACK
# and numpy, not from the oracle.
def pin_block_neumann(seed=13):
    rng = np.random.default_rng(seed)
    n, blk = 128, 16
    N = np.tril(rng.standard_normal((n, n)) * 0.15, -1)
    bl = np.arange(n) // blk
    I = np.eye(n)
    Dinv = np.linalg.inv(I + np.where(bl[:, None] == bl[None, :], N, 0.0))
    Nb = Dinv @ np.where(bl[:, None] > bl[None, :], N, 0.0)
    powers = [np.linalg.matrix_power(-Nb, s) for s in range(8)]
    exact = np.linalg.inv(I + N)
    X1 = oracle.block_neumann1_inverse(N, blk)
    lag = bl[:, None] - bl[None, :]
    return max(_rel(sum(powers), (I + powers[4]) @ (I + Nb @ Nb) @ (I - Nb)),
               _rel(sum(powers) @ Dinv, exact),
               _rel(X1, exact - sum(powers[2:]) @ Dinv),
               np.abs((X1 - exact)[lag <= 1]).max() / np.abs(exact).max())


# The 1-Step Neumann chunk form is exact while a chunk holds at most two blocks
# of 16 (no block lag above 1): at C = 32 it is the token recurrence.
def pin_neumann1_short_chunks(seed=14):
    rng = np.random.default_rng(seed)
    q, k, v, g, beta, S0 = rand_inputs(rng, 1, 70, 2, 2, 8, 4, 8)
    o, Sf = oracle.recurrent(q, k, v, g, beta, S0)
    worst = 0.0
    for C in (16, 32):
        o1, S1 = oracle.chunked(q, k, v, g, beta, S0, chunk=C, inverse="neumann1")
        worst = max(worst, _rel(o1, o), _rel(S1, Sf))
    return worst


# Readout epilogue ("Systolic Linear Attention ...", §2.3 Eq. (5): output gate
# times per-value-head RMSNorm): a hand-worked row, unit mean square with the
# gate open (z large), eps = 0 and unit weight, invariance to a positive scale of
# o, and the weight applied channel by channel.
def pin_output_epilogue(seed=15):
    # o = (3, 4): mean square 12.5; z = 0 gates by 1/2
    out = oracle.output_gate_rmsnorm(np.array([[3.0, 4.0]]), np.zeros((1, 2)), eps=0.0)
    worst = _rel(out, np.array([[1.5, 2.0]]) / np.sqrt(12.5))
    # per-channel gates sigmoid(0) = 1/2, sigmoid(ln 3) = 3/4, and eps = 7.5 inside the
    # root: 1 / sqrt(12.5 + 7.5) = 1 / sqrt(20)
    out = oracle.output_gate_rmsnorm(np.array([[3.0, 4.0]]), np.array([[0.0, np.log(3.0)]]), eps=7.5)
    worst = max(worst, _rel(out, np.array([[1.5, 3.0]]) / np.sqrt(20.0)))
    rng = np.random.default_rng(seed)
    o, z = rng.standard_normal((5, 7, 16)), rng.standard_normal((5, 7, 16))
    w = rng.standard_normal(16)
    opened = oracle.output_gate_rmsnorm(o, np.full_like(o, 60.0), eps=0.0)
    worst = max(worst, np.abs(np.mean(opened ** 2, axis=-1) - 1.0).max())
    a = oracle.output_gate_rmsnorm(o, z, w, eps=0.0)
    worst = max(worst, _rel(a, oracle.output_gate_rmsnorm(3.7 * o, z, w, eps=0.0)))
    worst = max(worst, _rel(a, oracle.output_gate_rmsnorm(o, z, None, eps=0.0) * w))
    return worst


# Chunk-boundary momentum ("Systolic Linear Attention ...", §2.3): with mu = 0,
# or with every reset indicator kappa_c = 0, the momentum form is the plain
# chunked form.
def pin_momentum_reduces(seed=16):
    rng = np.random.default_rng(seed)
    q, k, v, g, beta, S0 = rand_inputs(rng, 2, 50, 2, 4, 8, 3, 8)
    o, Sf = oracle.chunked(q, k, v, g, beta, S0, chunk=8)
    worst = 0.0
    for kw in (dict(mu=0.0), dict(mu=0.25, kappa=np.zeros((2, 7), np.int32))):
        om, Sm = oracle.chunked(q, k, v, g, beta, S0, chunk=8, **kw)
        worst = max(worst, _rel(om, o), _rel(Sm, Sf))
    return worst


# The same momentum written as the pages' joint affine step of (S, Z) (§3.3,
# context parallelism): [S_c; Z_c] = [[J_c, mu kappa_c I], [J_c - F_c, mu kappa_c I]]
# [S_{c-1}; Z_{c-1}] + [B_c; B_c], with J_c the chunk's state map from the
# identity with no values, B_c its map from zero (both from plain chunked runs of
# that chunk alone) and F_c = diag(exp(sum of its log-decays)).
def pin_momentum_block_form(seed=17):
    rng = np.random.default_rng(seed)
    T, C, dk, dv, mu = 40, 8, 6, 3, 0.25
    q, k, v, g, beta, S0 = rand_inputs(rng, 1, T, 1, 1, dk, dv, dk)
    kappa = np.array([[1, 1, 0, 1, 1]], np.int32)
    _, Sm = oracle.chunked(q, k, v, g, beta, S0, chunk=C, mu=mu, kappa=kappa)
    S, Z = S0[0, 0].copy(), np.zeros((dk, dv))
    for c in range(T // C):
        sl = slice(c * C, (c + 1) * C)
        qs, ks, vs, gs, bs = q[:, :, sl], k[:, :, sl], v[:, :, sl], g[:, :, sl], beta[:, :, sl]
        _, J = oracle.chunked(qs, ks, np.zeros((1, 1, C, dk)), gs, bs, np.eye(dk)[None, None], chunk=C)
        _, Bc = oracle.chunked(qs, ks, vs, gs, bs, None, chunk=C)
        J, Bc = J[0, 0], Bc[0, 0]
        F = np.diag(np.exp(gs[0, 0].sum(axis=0)))
        m = mu * kappa[0, c]
        S, Z = J @ S + m * Z + Bc, (J - F) @ S + m * Z + Bc
    return _rel(S, Sm[0, 0])


# Gradients of the recurrence (the backward of NEXT #2 starts from this): the
# oracle's reverse sweep against central finite differences of its forward, for
# every input element of a tiny problem with two value heads per key head (the
# key-head gradients sum over them), per-channel and scalar gates, and S0.
def pin_grad_finite_differences(seed=18):
    rng = np.random.default_rng(seed)
    worst = 0.0
    for G in (3, 1):
        q, k, v, g, beta, S0 = rand_inputs(rng, 1, 5, 1, 2, 3, 2, G)
        Wo = rng.standard_normal((1, 2, 5, 2))
        Ws = rng.standard_normal((1, 2, 3, 2))
        x = {"q": q, "k": k, "v": v, "g": g, "beta": beta, "S0": S0}

        def loss(x):
            o, Sf = oracle.recurrent(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"])
            return float(np.sum(o * Wo) + np.sum(Sf * Ws))

        grads = oracle.recurrent_grad(q, k, v, g, beta, S0, Wo, Ws)
        h = 1e-6
        for name, arr in x.items():
            fd = np.zeros_like(arr)
            for idx in np.ndindex(arr.shape):
                old = arr[idx]
                arr[idx] = old + h
                lp = loss(x)
                arr[idx] = old - h
                lm = loss(x)
                arr[idx] = old
                fd[idx] = (lp - lm) / (2 * h)
            worst = max(worst, np.abs(grads[name] - fd).max() / max(np.abs(fd).max(), 1e-30))
    return worst


ALL_PINS = {
    "golden_examples": (pin_golden_examples, 1e-12),
    "golden_inverse": (pin_golden_inverse, 1e-12),
    "pure_decay": (pin_pure_decay, 1e-12),
    "linear_attention": (pin_linear_attention, 1e-12),
    "chunked_equals_recurrent": (pin_chunked_equals_recurrent, 1e-11),
    "inverse_identity": (pin_inverse_identity, 1e-11),
    "neumann_bands": (pin_neumann_bands, 1e-10),
    "neumann_error_bound": (pin_neumann_error_bound, 1e-9),
    "grouped_gram": (pin_grouped_gram, 1e-12),
    "gate_consistency": (pin_gate_consistency, 1e-12),
    "gva": (pin_gva, 1e-13),
    "resume": (pin_resume, 1e-12),
    "affine_segments": (pin_affine_segments, 1e-12),
    "block_neumann": (pin_block_neumann, 1e-10),
    "neumann1_short_chunks": (pin_neumann1_short_chunks, 1e-12),
    "output_epilogue": (pin_output_epilogue, 1e-13),
    "momentum_reduces": (pin_momentum_reduces, 1e-13),
    "momentum_block_form": (pin_momentum_block_form, 1e-12),
    "grad_finite_differences": (pin_grad_finite_differences, 1e-6),
    "chunked_neumann": (pin_chunked_neumann, 1e-11),
}


def failing_pins():
    """Names of pins that fail (or raise) under the currently loaded oracle."""
    bad = []
    for name, (fn, tol) in ALL_PINS.items():
        try:
            err = fn()
        except Exception:  # a broken build may also reject its inputs
            bad.append(name)
            continue
        if not (err <= tol):
            bad.append(name)
    return bad
