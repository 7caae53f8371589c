"""Helpers for the GPU parity tests: run the CUDA path through the C ABI and
compare it with the fp64 oracle on the same seeded inputs."""
from __future__ import annotations

import numpy as np

import oracle
from gated_delta_rule_141_b200 import workloads as W

# Tolerances fixed by the acceptance criterion: relative error
# max|x - x_ref| / max|x_ref| on o and on S_final.
TOL_F32 = 1e-4
TOL_BF16 = 2e-2


def tol_for(in_dtype: str) -> float:
    return TOL_F32 if in_dtype == "f32" else TOL_BF16


def rel_err(x, ref) -> float:
    x = np.asarray(x, np.float64)
    ref = np.asarray(ref, np.float64)
    if ref.size == 0:
        return 0.0
    den = np.abs(ref).max()
    if den == 0:
        return float(np.abs(x).max())
    return float(np.abs(x - ref).max() / den)


def to_device(inputs: dict, in_dtype: str):
    import torch
    dt = torch.bfloat16 if in_dtype == "bf16" else torch.float32
    dev = {}
    for n in ("q", "k", "v"):
        dev[n] = torch.from_numpy(inputs[n]).to("cuda").to(dt).contiguous()
    for n in ("g", "beta"):
        dev[n] = torch.from_numpy(np.ascontiguousarray(inputs[n], np.float32)).to("cuda")
    dev["S0"] = None if inputs["S0"] is None else torch.from_numpy(inputs["S0"]).to("cuda")
    return dev


def run_gpu(inputs: dict, in_dtype: str, chunk: int, inverse: str = "exact", order: int = 4,
            resid: int = 1, kernel: str = "auto", out_dtype=None, want_state=True):
    import torch
    from gated_delta_rule_141_b200 import gdr
    dev = to_device(inputs, in_dtype)
    o, Sf = gdr.chunk_fwd(dev["q"], dev["k"], dev["v"], dev["g"], dev["beta"], dev["S0"],
                          chunk=chunk, inverse=inverse, neumann_order=order,
                          neumann_residual_steps=resid, out_dtype=out_dtype,
                          want_state=want_state, kernel=kernel)
    torch.cuda.synchronize()
    assert gdr.device_status() == gdr.OK
    o = o.float().cpu().numpy().astype(np.float64)
    Sf = None if Sf is None else Sf.cpu().numpy().astype(np.float64)
    return o, Sf


def slice_sequences(inputs: dict, R: int, seqs):
    """Inputs restricted to value heads `seqs` = [(b, hv), ...], each as its own
    batch entry with one key head and one value head."""
    out = {}
    for n in ("q", "k", "g", "beta"):
        out[n] = np.stack([inputs[n][b, hv // R] for b, hv in seqs])[:, None]
    out["v"] = np.stack([inputs["v"][b, hv] for b, hv in seqs])[:, None]
    out["S0"] = (None if inputs["S0"] is None
                 else np.stack([inputs["S0"][b, hv] for b, hv in seqs])[:, None])
    return out


def oracle_reference(inputs: dict, chunk: int, inverse: str, order: int = 4, resid: int = 1):
    """The oracle's answer: the token recurrence for the exact mode (the
    definition), the chunked form with the same approximate inverse otherwise
    ("neumann": truncated Neumann; "neumann1": 1-Step Neumann in blocks of 16)."""
    args = (inputs["q"], inputs["k"], inputs["v"], inputs["g"], inputs["beta"], inputs["S0"])
    if inverse == "exact":
        return oracle.recurrent(*args)
    return oracle.chunked(*args, chunk=chunk, inverse=inverse, order=order, resid=resid)


def sample_sequences(w: W.Workload, count: int = 8):
    """Deterministic sample of at least `count` (b, hv) pairs (all of them when
    there are fewer): the first and the last sequence, every value head of the
    middle key head of a middle batch entry (all R heads that share one key
    head's factors), then sequences spread evenly over the grid."""
    total = w.B * w.Hv
    picks = {0, total - 1}
    bm, hk = w.B // 2, w.Hk // 2
    picks.update(bm * w.Hv + hk * w.R + r for r in range(w.R))
    j = 0
    while len(picks) < min(count, total):
        picks.add((j * total) // count + (j * 3) % max(1, total // count))
        j += 1
    return [(s // w.Hv, s % w.Hv) for s in sorted(picks)]
