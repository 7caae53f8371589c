"""fp64 CPU oracle for the gated delta-rule forward (numpy front end).

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline / reference legs of ``bench.py``.  The CUDA product path
never imports, links or calls anything here, and this package imports nothing
from the product package.

The arithmetic lives in ``gdr_oracle.c`` (plain C99 + OpenMP, fp64); this file
only marshals numpy arrays.  Citations for each routine are in the C source:
the token recurrence follows "Systolic Linear Attention: Co-Designing
Tile-Grouped Gated Delta Attention for TPUs" §2.1 Eq. (2); the chunkwise WY
form follows its §2.3 Table 2 and §2.4.2, its 1-Step Neumann block inverse
§2.4.3, chunk-boundary momentum and the readout epilogue §2.3, and the gradient
(``recurrent_grad``) is the exact derivative of the token recurrence that the
backward of its §2.5 must reproduce; the truncated Neumann inverse follows "When
Good Enough Is Optimal: Multiplication-Only Matrix Inversion Approximation for
Quantized Gated DeltaNet" (Lemma 3.1, §4.1).

Pins: every function here is checked in ``tests/test_oracle_pins.py`` against
closed forms, invariants and hand-worked examples in ``tests/golden/``.
"""
from __future__ import annotations

import contextlib
import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdr_oracle.c")
_LIB_PATH = os.path.join(_HERE, "_gdr_oracle.so")
_lib = None

INV_EXACT = 0
INV_NEUMANN = 1
INV_NEUMANN1 = 2   # 1-Step Neumann, blocks of 16 rows
NV_NEWTON = 0      # residual step X <- X + X (I - (I+N) X)
NV_REFINE = 1      # residual step X <- X + X0 (I - (I+N) X)
NV_BANDCUT = 2     # zero X0 outside the band i - j <= order


def build(force: bool = False, src: str = _SRC, out: str = _LIB_PATH) -> str:
    """Compile the oracle C source into a shared library with gcc + OpenMP."""
    if (not force and os.path.exists(out)
            and os.path.getmtime(out) >= os.path.getmtime(src)):
        return out
    tmp = out + ".tmp%d" % os.getpid()
    cmd = ["gcc", "-O2", "-std=c99", "-fopenmp", "-fPIC", "-shared",
           "-Wall", "-o", tmp, src, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


def load_library(path: str):
    """Load an oracle build (the default one, or a test's mutated copy)."""
    lib = ctypes.CDLL(path)
    dp = ctypes.POINTER(ctypes.c_double)
    i = ctypes.c_int
    lib.gdro_recurrent.argtypes = [i] * 7 + [dp] * 8 + [i]
    lib.gdro_chunked.argtypes = [i] * 12 + [dp] * 8 + [i]
    lib.gdro_chunked_momentum.argtypes = ([i] * 12 + [ctypes.c_double, ctypes.POINTER(i)]
                                          + [dp] * 8 + [i])
    lib.gdro_tril_inverse.argtypes = [i, dp, dp]
    lib.gdro_neumann_inverse.argtypes = [i, dp, i, i, i, dp]
    lib.gdro_block_neumann1_inverse.argtypes = [i, dp, i, dp]
    lib.gdro_output_gate_rmsnorm.argtypes = [i, i, dp, dp, dp, ctypes.c_double, dp]
    lib.gdro_recurrent_grad.argtypes = [i] * 7 + [dp] * 14 + [i]
    lib.gdro_chunk_matrices.argtypes = [i, i, i] + [dp] * 7
    lib.gdro_max_threads.argtypes = []
    for f in (lib.gdro_recurrent, lib.gdro_chunked, lib.gdro_chunked_momentum, lib.gdro_tril_inverse,
              lib.gdro_neumann_inverse, lib.gdro_block_neumann1_inverse,
              lib.gdro_output_gate_rmsnorm, lib.gdro_recurrent_grad,
              lib.gdro_chunk_matrices, lib.gdro_max_threads):
        f.restype = ctypes.c_int
    return lib


@contextlib.contextmanager
def using_library(path: str):
    """Temporarily route every oracle call through another build (tests only)."""
    global _lib
    saved = _load()
    _lib = load_library(path)
    try:
        yield
    finally:
        _lib = saved


def _load():
    global _lib
    if _lib is None:
        _lib = load_library(build())
    return _lib


def max_threads() -> int:
    return int(_load().gdro_max_threads())


def _f64(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _dims(q, v, g):
    B, Hk, T, dk = q.shape
    Bv, Hv, Tv, dv = v.shape
    G = g.shape[-1]
    if Bv != B or Tv != T:
        raise ValueError("q and v disagree on B or T")
    return B, T, Hk, Hv, dk, dv, G


def _check(code, what):
    if code != 0:
        raise ValueError("%s failed with code %d" % (what, code))


def recurrent(q, k, v, g, beta, S0=None, nthreads=0):
    """Token-by-token fp64 recurrence.  Returns (o [B,Hv,T,dv], S_final [B,Hv,dk,dv])."""
    q, k, v, g, beta = map(_f64, (q, k, v, g, beta))
    S0 = None if S0 is None else _f64(S0)
    B, T, Hk, Hv, dk, dv, G = _dims(q, v, g)
    o = np.zeros((B, Hv, T, dv), np.float64)
    Sf = np.zeros((B, Hv, dk, dv), np.float64)
    _check(_load().gdro_recurrent(B, T, Hk, Hv, dk, dv, G, _ptr(q), _ptr(k), _ptr(v),
                                  _ptr(g), _ptr(beta), _ptr(S0), _ptr(o), _ptr(Sf),
                                  int(nthreads)), "gdro_recurrent")
    return o, Sf


def recurrent_grad(q, k, v, g, beta, S0, dO, dSf=None, nthreads=0):
    """Gradients of sum(dO * o) + sum(dSf * S_final) of the token recurrence with
    respect to (q, k, v, g, beta, S0), by a reverse sweep over the tokens.
    Returns a dict with those keys (dS0 is the gradient at the initial state,
    zero or S0)."""
    q, k, v, g, beta, dO = map(_f64, (q, k, v, g, beta, dO))
    S0 = None if S0 is None else _f64(S0)
    dSf = None if dSf is None else _f64(dSf)
    B, T, Hk, Hv, dk, dv, G = _dims(q, v, g)
    out = {"q": np.zeros_like(q), "k": np.zeros_like(k), "v": np.zeros_like(v),
           "g": np.zeros_like(g), "beta": np.zeros_like(beta),
           "S0": np.zeros((B, Hv, dk, dv), np.float64)}
    _check(_load().gdro_recurrent_grad(B, T, Hk, Hv, dk, dv, G, _ptr(q), _ptr(k), _ptr(v),
                                       _ptr(g), _ptr(beta), _ptr(S0), _ptr(dO), _ptr(dSf),
                                       _ptr(out["q"]), _ptr(out["k"]), _ptr(out["v"]),
                                       _ptr(out["g"]), _ptr(out["beta"]), _ptr(out["S0"]),
                                       int(nthreads)), "gdro_recurrent_grad")
    return out


def chunked(q, k, v, g, beta, S0=None, chunk=64, inverse="exact", order=4, resid=1,
            variant=NV_NEWTON, nthreads=0, mu=None, kappa=None):
    """Chunkwise WY form in fp64 with an exact (forward substitution), truncated
    Neumann ("neumann") or 1-Step Neumann in blocks of 16 ("neumann1") chunk
    inverse.  With `mu` (and optionally `kappa`, [B, ceil(T/chunk)] reset
    indicators in {0, 1}) the state carries chunk-boundary momentum.  Returns
    (o, S_final)."""
    q, k, v, g, beta = map(_f64, (q, k, v, g, beta))
    S0 = None if S0 is None else _f64(S0)
    B, T, Hk, Hv, dk, dv, G = _dims(q, v, g)
    mode = {"exact": INV_EXACT, "neumann": INV_NEUMANN, "neumann1": INV_NEUMANN1}[inverse]
    o = np.zeros((B, Hv, T, dv), np.float64)
    Sf = np.zeros((B, Hv, dk, dv), np.float64)
    if mu is None and kappa is None:
        _check(_load().gdro_chunked(B, T, Hk, Hv, dk, dv, G, int(chunk), mode, int(order),
                                    int(resid), int(variant), _ptr(q), _ptr(k), _ptr(v),
                                    _ptr(g), _ptr(beta), _ptr(S0), _ptr(o), _ptr(Sf),
                                    int(nthreads)), "gdro_chunked")
        return o, Sf
    kp = None
    if kappa is not None:
        kappa = np.ascontiguousarray(kappa, dtype=np.int32)
        if kappa.shape != (B, (T + int(chunk) - 1) // int(chunk)):
            raise ValueError("kappa must be [B, ceil(T / chunk)]")
        kp = kappa.ctypes.data_as(ctypes.POINTER(ctypes.c_int))
    _check(_load().gdro_chunked_momentum(B, T, Hk, Hv, dk, dv, G, int(chunk), mode, int(order),
                                         int(resid), int(variant), float(mu or 0.0), kp,
                                         _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                                         _ptr(S0), _ptr(o), _ptr(Sf), int(nthreads)),
           "gdro_chunked_momentum")
    return o, Sf


def tril_inverse(N):
    """(I + N)^{-1} for strictly lower-triangular N, by forward substitution."""
    N = _f64(N)
    n = N.shape[0]
    X = np.zeros((n, n), np.float64)
    _check(_load().gdro_tril_inverse(n, _ptr(N), _ptr(X)), "gdro_tril_inverse")
    return X


def neumann_inverse(N, order=4, resid=1, variant=NV_NEWTON):
    """Truncated Neumann approximation of (I + N)^{-1} with structural masking
    and `resid` residual-correction steps."""
    N = _f64(N)
    n = N.shape[0]
    X = np.zeros((n, n), np.float64)
    _check(_load().gdro_neumann_inverse(n, _ptr(N), int(order), int(resid), int(variant),
                                        _ptr(X)), "gdro_neumann_inverse")
    return X


def block_neumann1_inverse(N, blk=16):
    """1-Step Neumann approximation (I - Nb) D^{-1} of (I + N)^{-1}: D the
    block-diagonal part of I + N in blocks of `blk`, Nb = D^{-1} N_off."""
    N = _f64(N)
    n = N.shape[0]
    X = np.zeros((n, n), np.float64)
    _check(_load().gdro_block_neumann1_inverse(n, _ptr(N), int(blk), _ptr(X)),
           "gdro_block_neumann1_inverse")
    return X


def output_gate_rmsnorm(o, z, w=None, eps=1e-6):
    """sigmoid(z) * RMSNorm(o) over the last axis (dv) of o and z, with weight w [dv]
    (ones when None): the readout epilogue of the SLA recurrence."""
    o, z = _f64(o), _f64(z)
    dv = o.shape[-1]
    rows = o.size // dv if dv else 0
    out = np.zeros(o.shape, np.float64)
    wv = None if w is None else _f64(w)
    _check(_load().gdro_output_gate_rmsnorm(int(rows), int(dv), _ptr(o), _ptr(z), _ptr(wv),
                                            float(eps), _ptr(out)), "gdro_output_gate_rmsnorm")
    return out


def chunk_matrices(qc, kc, gc, bc):
    """Cumulative log-decay Lam [C,dk], Gram M [C,C] and score L [C,C] of one
    chunk of one key head (qc, kc [C,dk]; gc [C,G]; bc [C])."""
    qc, kc, gc, bc = map(_f64, (qc, kc, gc, bc))
    C, dk = kc.shape
    G = gc.shape[-1]
    Lam = np.zeros((C, dk), np.float64)
    M = np.zeros((C, C), np.float64)
    L = np.zeros((C, C), np.float64)
    _check(_load().gdro_chunk_matrices(C, dk, G, _ptr(qc), _ptr(kc), _ptr(gc), _ptr(bc),
                                       _ptr(Lam), _ptr(M), _ptr(L)), "gdro_chunk_matrices")
    return Lam, M, L
