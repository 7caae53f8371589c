"""Seeded synthetic inputs for the gated delta-rule forward.

This module holds no arithmetic of the method itself: it only draws random
numbers (numpy PCG64) and shapes them into the input distributions that the
workloads specify (L2-normalised queries and keys, sigmoid write gates,
negative-softplus log forget gates).  Both the CUDA path's tests/bench and the
fp64 oracle consume the same arrays; q, k, v are rounded to the input dtype
here, on the host, so the oracle reads exactly the values the GPU reads.

Workloads (synthetic; the pages train on no public data for this kernel):
  0  tiny scalar-gate GDN, fp32:     B=1  H=2        T=256   dk=dv=64  C=64
  1  scalar-gate GDN, bf16:          B=4  H=16       T=4096  dk=dv=128 C=64
  2  per-channel (KDA-style), bf16:  B=2  H=32       T=8192  dk=dv=128 C=64
  3  SLA wide-key GVA, bf16:         B=2  Hk=8 Hv=32 T=8192  dk=256 dv=128 C=64|128
  4  long-context strong decay:      B=1  H=16       T=65536 dk=dv=128 C=128
Draw order per workload (seed 1000 + index): q, k, v, beta-logit, g-logit, S0.
A normal N(0, s) takes s as the standard deviation.
"""
from __future__ import annotations

import dataclasses

import numpy as np

GATE_SCALAR = 0    # G = 1
GATE_GROUP64 = 1   # G = dk / 64
GATE_CHANNEL = 2   # G = dk


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    T: int
    Hk: int
    Hv: int
    dk: int
    dv: int
    chunk: int
    gate_mode: int
    in_dtype: str            # "f32" or "bf16"
    qk_silu: bool            # q, k = L2norm(SiLU(N(0,1))) instead of L2norm(N(0,1))
    g_std: float             # g-logit ~ N(0, g_std)
    g_scale: float           # g = -softplus(logit) * g_scale
    s0_std: float            # 0 -> S0 is NULL
    inverse_modes: tuple = ("exact",)
    chunks: tuple = ()

    @property
    def G(self) -> int:
        return {GATE_SCALAR: 1, GATE_GROUP64: self.dk // 64, GATE_CHANNEL: self.dk}[self.gate_mode]

    @property
    def R(self) -> int:
        return self.Hv // self.Hk

    def scaled(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = [
    Workload("tiny_gdn_fp32", B=1, T=256, Hk=2, Hv=2, dk=64, dv=64, chunk=64,
             gate_mode=GATE_SCALAR, in_dtype="f32", qk_silu=False, g_std=1.0, g_scale=1.0,
             s0_std=0.0),
    Workload("gdn_scalar_bf16", B=4, T=4096, Hk=16, Hv=16, dk=128, dv=128, chunk=64,
             gate_mode=GATE_SCALAR, in_dtype="bf16", qk_silu=False, g_std=1.0, g_scale=1.0,
             s0_std=0.02),
    Workload("kda_channel_bf16", B=2, T=8192, Hk=32, Hv=32, dk=128, dv=128, chunk=64,
             gate_mode=GATE_CHANNEL, in_dtype="bf16", qk_silu=True, g_std=1.0, g_scale=0.1,
             s0_std=0.0),
    Workload("sla_gva_dk256_bf16", B=2, T=8192, Hk=8, Hv=32, dk=256, dv=128, chunk=64,
             gate_mode=GATE_GROUP64, in_dtype="bf16", qk_silu=False, g_std=1.0, g_scale=0.1,
             s0_std=0.0, inverse_modes=("exact", "neumann"), chunks=(64, 128)),
    Workload("long_strong_decay_bf16", B=1, T=65536, Hk=16, Hv=16, dk=128, dv=128, chunk=128,
             gate_mode=GATE_CHANNEL, in_dtype="bf16", qk_silu=False, g_std=2.0, g_scale=1.0,
             s0_std=0.02, inverse_modes=("exact", "neumann")),
]


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to the nearest bf16 (ties to even); returns fp32."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return (u.astype(np.uint32) << 16).view(np.float32)


def _l2norm(x: np.ndarray) -> np.ndarray:
    n = np.sqrt(np.sum(x.astype(np.float64) ** 2, axis=-1, keepdims=True))
    return (x / np.maximum(n, 1e-12)).astype(np.float32)


def _softplus(x: np.ndarray) -> np.ndarray:
    return np.logaddexp(0.0, x.astype(np.float64))


def _sigmoid(x: np.ndarray) -> np.ndarray:
    return 1.0 / (1.0 + np.exp(-x.astype(np.float64)))


def make_inputs(w: Workload, seed: int) -> dict:
    """Draw one workload's inputs.  Returns fp32 numpy arrays:
    q, k [B,Hk,T,dk]; v [B,Hv,T,dv]; g [B,Hk,T,G]; beta [B,Hk,T]; S0 [B,Hv,dk,dv] or None.
    q, k, v already hold values representable in ``w.in_dtype``."""
    rng = np.random.Generator(np.random.PCG64(seed))
    B, T, Hk, Hv, dk, dv, G = w.B, w.T, w.Hk, w.Hv, w.dk, w.dv, w.G
    q = rng.standard_normal((B, Hk, T, dk), dtype=np.float32)
    k = rng.standard_normal((B, Hk, T, dk), dtype=np.float32)
    v = rng.standard_normal((B, Hv, T, dv), dtype=np.float32)
    b_logit = rng.standard_normal((B, Hk, T), dtype=np.float32)
    g_logit = rng.standard_normal((B, Hk, T, G), dtype=np.float32) * np.float32(w.g_std)
    S0 = None
    if w.s0_std > 0:
        S0 = rng.standard_normal((B, Hv, dk, dv), dtype=np.float32) * np.float32(w.s0_std)
    if w.qk_silu:
        q = q / (1.0 + np.exp(-q))
        k = k / (1.0 + np.exp(-k))
    q = _l2norm(q)
    k = _l2norm(k)
    beta = _sigmoid(b_logit).astype(np.float32)
    g = (-_softplus(g_logit) * w.g_scale).astype(np.float32)
    if w.in_dtype == "bf16":
        q, k, v = round_to_bf16(q), round_to_bf16(k), round_to_bf16(v)
    return dict(q=q, k=k, v=v, g=g, beta=beta, S0=S0)


def workload_inputs(index: int, seed=None, **overrides) -> tuple:
    """(workload, inputs) for workload `index` with the standard seed 1000 + index
    (or `seed`); `overrides` shrink a workload (e.g. T=512) while keeping its
    distributions."""
    w = WORKLOADS[index]
    if overrides:
        w = w.scaled(**overrides)
    return w, make_inputs(w, 1000 + index if seed is None else seed)
