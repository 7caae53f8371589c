"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the
same seeded inputs.  Bounds (relative error max|x - x_ref| / max|x_ref| on o and
S_final): 1e-4 for the fp32 path, 2e-2 for bf16 inputs with fp32 state and
accumulation.  Neumann mode is compared with the oracle's chunked Neumann form
(same order and residual steps); its distance from the exact inverse is
reported separately."""
import numpy as np
import pytest

import gpu_util as U
from gated_delta_rule_141_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    from gated_delta_rule_141_b200 import build as gdr_build
    gdr_build.build()


# (workload index, overrides, chunk, inverse, kernel)
SMALL = [
    # fp32 path, tiny GDN workload at its own size (the whole workload, every output)
    (0, {}, 64, "exact", "auto"),
    (0, {}, 64, "exact", "simt"),
    # ragged last chunk, odd sizes, S0 present, fp32
    (0, dict(T=203, Hk=1, Hv=3, dv=40, s0_std=0.5), 64, "exact", "simt"),
    (0, dict(T=77, dk=32, dv=16, s0_std=0.3), 16, "exact", "simt"),
    (0, dict(T=130, gate_mode=W.GATE_CHANNEL), 32, "neumann", "simt"),
    # bf16 inputs, each gate mode, both inverse modes, shrunk workloads
    (1, dict(B=1, Hk=2, Hv=2, T=320), 64, "exact", "auto"),
    (1, dict(B=1, Hk=2, Hv=2, T=320), 64, "exact", "simt"),
    (2, dict(B=1, Hk=2, Hv=2, T=448), 64, "exact", "auto"),
    (2, dict(B=1, Hk=2, Hv=2, T=448), 64, "neumann", "auto"),
    (3, dict(B=1, Hk=2, Hv=8, T=384), 64, "exact", "auto"),
    (3, dict(B=1, Hk=2, Hv=8, T=384), 64, "neumann", "auto"),
    (3, dict(B=1, Hk=1, Hv=4, T=384, chunk=128), 128, "exact", "auto"),
    (4, dict(Hk=2, Hv=2, T=640), 128, "exact", "auto"),
    (4, dict(Hk=2, Hv=2, T=704 - 37), 128, "exact", "auto"),
    # tensor-core kernel for grouped / per-channel decay, forced
    (2, dict(B=1, Hk=2, Hv=2, T=448 - 37), 64, "exact", "tc"),
    (2, dict(B=1, Hk=1, Hv=1, T=256, gate_mode=W.GATE_GROUP64), 64, "exact", "tc"),
    (3, dict(B=1, Hk=1, Hv=4, T=256, gate_mode=W.GATE_SCALAR), 64, "exact", "tc"),
    (3, dict(B=1, Hk=1, Hv=4, T=256 - 21), 64, "neumann", "tc"),
    (4, dict(Hk=1, Hv=1, T=384), 64, "exact", "tc"),      # strong decay: exact fp32 Gram
    (4, dict(Hk=1, Hv=1, T=384), 64, "neumann", "tc"),
    # exact mode at C = 128 on the tensor-core kernels (blocked by 64 there), oracle at C = 128
    (1, dict(B=1, Hk=2, Hv=2, T=320 - 13), 128, "exact", "tc"),
    (3, dict(B=1, Hk=1, Hv=4, T=384 - 37), 128, "exact", "tc"),
    (4, dict(Hk=2, Hv=2, T=640), 128, "exact", "tc"),
    # two-pass tensor-core path (chunk factors in a workspace, then the state pass)
    (1, dict(B=1, Hk=2, Hv=2, T=320 - 13), 64, "exact", "tc2"),
    (1, dict(B=2, Hk=1, Hv=3, T=256, dv=192), 64, "exact", "tc2"),      # grouped values, 3 tiles
    (1, dict(B=1, Hk=1, Hv=1, T=256), 64, "neumann", "tc2"),
    (2, dict(B=1, Hk=2, Hv=2, T=448 - 37), 64, "exact", "tc2"),
    (2, dict(B=1, Hk=1, Hv=2, T=256, gate_mode=W.GATE_GROUP64), 64, "exact", "tc2"),
    # odd T: the second head's gate rows start off a 16-byte boundary (plain loads)
    (2, dict(B=1, Hk=2, Hv=2, T=256 - 27, gate_mode=W.GATE_GROUP64), 64, "exact", "tc2"),
    (2, dict(B=1, Hk=2, Hv=2, T=256), 64, "neumann", "tc2"),
    (4, dict(Hk=2, Hv=2, T=640 - 5), 128, "exact", "tc2"),               # strong decay, S0
    (4, dict(Hk=1, Hv=1, T=64), 64, "exact", "tc2"),                     # a single chunk
    # 1-Step Neumann inverse (blocks of 16): two-pass path at chunk 64, CUDA-core
    # kernel at chunk 128 (eight blocks, as in the pages)
    (1, dict(B=1, Hk=2, Hv=2, T=320 - 13), 64, "neumann1", "tc2"),
    (2, dict(B=1, Hk=2, Hv=2, T=448 - 37), 64, "neumann1", "tc2"),
    (4, dict(Hk=1, Hv=1, T=384), 64, "neumann1", "tc2"),                # pivoted blocks
    (0, {}, 128, "neumann1", "auto"),                                   # fp32
    (4, dict(Hk=1, Hv=1, T=300), 128, "neumann1", "auto"),
    # truncated Neumann at chunk 128 on the two-pass path: pairs of 64-token halves
    # with the pair correction; an odd number of halves (no second half in the last
    # pair), a partial second half, weak and strong per-channel decay, grouped and
    # scalar gates, grouped value heads
    (4, dict(Hk=2, Hv=2, T=640), 128, "neumann", "tc2"),
    (4, dict(Hk=1, Hv=1, T=704 - 37), 128, "neumann", "tc2"),
    (4, dict(Hk=1, Hv=1, T=600), 128, "neumann", "tc2"),
    (2, dict(B=1, Hk=2, Hv=2, T=448 - 37), 128, "neumann", "tc2"),
    (2, dict(B=1, Hk=1, Hv=2, T=256, gate_mode=W.GATE_GROUP64), 128, "neumann", "tc2"),
    (1, dict(B=1, Hk=2, Hv=2, T=320 - 13), 128, "neumann", "tc2"),
    (1, dict(B=2, Hk=1, Hv=3, T=256, dv=192), 128, "neumann", "tc2"),
    # the 128-column state pass forced (sequential here: one segment), both decays,
    # grouped gates, two value tiles, the Neumann inverse at chunk 64
    (4, dict(Hk=2, Hv=2, T=640 - 5), 128, "exact", "tc2w"),
    (2, dict(B=1, Hk=2, Hv=2, T=448 - 37), 64, "exact", "tc2w"),
    (2, dict(B=1, Hk=1, Hv=2, T=256, gate_mode=W.GATE_GROUP64), 64, "exact", "tc2w"),
    (2, dict(B=1, Hk=1, Hv=2, T=300, dv=256), 64, "neumann", "tc2w"),
    # ... and its pairs of 64-token halves at chunk 128 (Y E1 added to a second half)
    (4, dict(Hk=2, Hv=2, T=640 - 5), 128, "neumann", "tc2w"),
    (4, dict(Hk=1, Hv=1, T=704 - 37), 128, "neumann", "tc2w"),
    (2, dict(B=1, Hk=1, Hv=2, T=448 - 37), 128, "neumann1", "tc2w"),
    # dk = 256 with grouped gates on the two-pass path (one [Q | W | K] buffer), grouped
    # value heads, S0, ragged tails, both chunk lengths and every inverse
    (3, dict(B=1, Hk=2, Hv=8, T=384), 64, "exact", "tc2"),
    (3, dict(B=1, Hk=1, Hv=4, T=384 - 37, s0_std=0.05), 64, "exact", "tc2"),
    (3, dict(B=2, Hk=1, Hv=2, T=256, dv=192), 128, "exact", "tc2"),
    (3, dict(B=1, Hk=2, Hv=8, T=256), 64, "neumann", "tc2"),
    (3, dict(B=1, Hk=1, Hv=4, T=384 - 37, s0_std=0.05), 128, "neumann", "tc2"),
    (3, dict(B=1, Hk=1, Hv=4, T=320), 128, "neumann1", "tc2"),
    (3, dict(B=1, Hk=1, Hv=2, T=200, gate_mode=W.GATE_SCALAR), 64, "exact", "auto"),
    # 1-Step Neumann at chunk 128 (eight blocks of 16, as in the pages) the same way
    (4, dict(Hk=2, Hv=2, T=640 - 27), 128, "neumann1", "tc2"),
    (2, dict(B=1, Hk=2, Hv=2, T=448 - 37), 128, "neumann1", "tc2"),
    (1, dict(B=1, Hk=2, Hv=2, T=320 - 13), 128, "neumann1", "tc2"),
]


@pytest.mark.parametrize("idx,over,chunk,inverse,kernel", SMALL,
                         ids=["w%d-%s-C%d-%s-%s" % (c[0], "-".join("%s%s" % kv for kv in c[1].items())
                                                     or "full", c[2], c[3], c[4]) for c in SMALL])
def test_small_parity(idx, over, chunk, inverse, kernel):
    w, x = W.workload_inputs(idx, **over)
    o, Sf = U.run_gpu(x, w.in_dtype, chunk, inverse, kernel=kernel)
    o_ref, S_ref = U.oracle_reference(x, chunk, inverse)
    tol = U.tol_for(w.in_dtype)
    eo, es = U.rel_err(o, o_ref), U.rel_err(Sf, S_ref)
    print("rel err o %.3e  S_final %.3e  (tol %.0e)" % (eo, es, tol))
    assert eo <= tol and es <= tol


@pytest.mark.parametrize("inverse", ["exact", "neumann"])
def test_decay_past_pivot_guard(inverse):
    # log-gates x8: 16-token half blocks span more than the pivot guard, so the first
    # pass recomputes those Gram rows element by element in fp32 (and rebuilds the
    # state pass's decayed operands afterwards)
    w, x = W.workload_inputs(4, Hk=1, Hv=1, T=192 - 11)
    x["g"] = (x["g"] * 8.0).astype(np.float32)
    o, Sf = U.run_gpu(x, w.in_dtype, 64, inverse, kernel="tc2")
    o_ref, S_ref = U.oracle_reference(x, 64, inverse)
    eo, es = U.rel_err(o, o_ref), U.rel_err(Sf, S_ref)
    print("rel err o %.3e  S_final %.3e" % (eo, es))
    assert eo <= U.TOL_BF16 and es <= U.TOL_BF16


def test_edge_cases():
    # T = 0: no tokens, S_final = S0
    w, x = W.workload_inputs(0, T=0, s0_std=0.4)
    o, Sf = U.run_gpu(x, "f32", 64)
    assert o.shape == (1, 2, 0, 64)
    assert np.array_equal(Sf, x["S0"].astype(np.float64))
    # T = 1 and T = C + 1 with and without S0, bf16 in / fp32 out
    for T in (1, 65):
        for s0 in (0.0, 0.3):
            w, x = W.workload_inputs(1, B=1, Hk=1, Hv=1, T=T, s0_std=s0)
            o, Sf = U.run_gpu(x, "bf16", 64, out_dtype=__import__("torch").float32)
            o_ref, S_ref = U.oracle_reference(x, 64, "exact")
            assert U.rel_err(o, o_ref) <= U.TOL_BF16
            assert U.rel_err(Sf, S_ref) <= U.TOL_BF16
    # no S_final requested
    w, x = W.workload_inputs(0, T=64)
    o, Sf = U.run_gpu(x, "f32", 64, want_state=False)
    assert Sf is None
    assert U.rel_err(o, U.oracle_reference(x, 64, "exact")[0]) <= U.TOL_F32


def test_host_entry_matches_device_entry():
    import torch
    from gated_delta_rule_141_b200 import gdr
    w, x = W.workload_inputs(1, B=1, Hk=2, Hv=2, T=256)
    dev_in = U.to_device(x, "bf16")
    o_dev, S_dev = gdr.chunk_fwd(dev_in["q"], dev_in["k"], dev_in["v"], dev_in["g"],
                                 dev_in["beta"], dev_in["S0"], chunk=64)
    host = {n: (None if t is None else t.cpu().pin_memory()) for n, t in dev_in.items()}
    host["o"] = torch.empty(o_dev.shape, dtype=o_dev.dtype).pin_memory()
    host["S_final"] = torch.empty(S_dev.shape, dtype=torch.float32).pin_memory()
    dev = {n: (None if t is None else torch.empty_like(t)) for n, t in dev_in.items()}
    dev["o"] = torch.empty_like(o_dev)
    dev["S_final"] = torch.empty_like(S_dev)
    shape = gdr.make_shape(w.B, w.T, w.Hk, w.Hv, w.dk, w.dv)
    ws = torch.empty(gdr.workspace_bytes(shape, 64, gdr.GATE_SCALAR), dtype=torch.uint8,
                     device="cuda")
    gdr.chunk_fwd_host(host, dev, shape, 64, gdr.GATE_SCALAR, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(host["o"], o_dev.cpu())
    assert torch.equal(host["S_final"], S_dev.cpu())


# Full-size workloads, in the launch configuration bench.py times, checked on a
# deterministic sample of sequences that the oracle computes one by one.
FULL = [
    (1, 64, "exact"),
    (2, 64, "exact"),
    (3, 64, "exact"),
    (3, 128, "exact"),
    (3, 64, "neumann"),
    (3, 128, "neumann"),
    (4, 128, "exact"),
    (4, 128, "neumann"),
]


@pytest.mark.parametrize("idx,chunk,inverse", FULL,
                         ids=["w%d-C%d-%s" % c for c in FULL])
def test_full_size_sampled(idx, chunk, inverse):
    w, x = W.workload_inputs(idx)
    o, Sf = U.run_gpu(x, w.in_dtype, chunk, inverse)
    assert np.isfinite(o).all() and np.isfinite(Sf).all()
    seqs = U.sample_sequences(w)
    xs = U.slice_sequences(x, w.R, seqs)
    o_ref, S_ref = U.oracle_reference(xs, chunk, inverse)
    idx_b = [b for b, _ in seqs]
    idx_h = [h for _, h in seqs]
    o_s = o[idx_b, idx_h][:, None]
    S_s = Sf[idx_b, idx_h][:, None]
    eo, es = U.rel_err(o_s, o_ref), U.rel_err(S_s, S_ref)
    msg = "rel err o %.3e  S_final %.3e" % (eo, es)
    if inverse == "neumann":
        o_ex, S_ex = U.oracle_reference(xs, chunk, "exact")
        msg += "  | Neumann vs exact: o %.3e  S_final %.3e" % (U.rel_err(o_s, o_ex),
                                                              U.rel_err(S_s, S_ex))
    print(msg)
    tol = U.tol_for(w.in_dtype)
    assert eo <= tol and es <= tol, msg


# Chunks shorter than the CUDA-core kernel's 32-column value tile in the Neumann
# modes (Q S then has its own buffer, not the C x C series buffer).
SHORT_CHUNK = [
    (0, dict(T=101, s0_std=0.3), 16, "neumann"),
    (0, dict(T=93, dv=40, gate_mode=W.GATE_CHANNEL), 24, "neumann1"),
]


@pytest.mark.parametrize("idx,over,chunk,inverse", SHORT_CHUNK,
                         ids=["C%d-%s" % (c[2], c[3]) for c in SHORT_CHUNK])
def test_short_chunk_neumann_parity(idx, over, chunk, inverse):
    w, x = W.workload_inputs(idx, **over)
    o, Sf = U.run_gpu(x, w.in_dtype, chunk, inverse, kernel="simt")
    o_ref, S_ref = U.oracle_reference(x, chunk, inverse)
    eo, es = U.rel_err(o, o_ref), U.rel_err(Sf, S_ref)
    print("rel err o %.3e  S_final %.3e" % (eo, es))
    assert eo <= U.TOL_F32 and es <= U.TOL_F32


# The pair correction at other Neumann orders and residual steps (order 0 with one
# Newton step; order 2 without; order 3 with two), and on a long single sequence
# whose state pass runs segment-parallel (segments start on pair boundaries).
PAIR_ORDERS = [(0, 1), (2, 0), (3, 2)]


@pytest.mark.parametrize("order,resid", PAIR_ORDERS, ids=["m%d-r%d" % c for c in PAIR_ORDERS])
def test_pair_neumann_orders(order, resid):
    w, x = W.workload_inputs(2, B=1, Hk=1, Hv=1, T=384 - 5)
    o, Sf = U.run_gpu(x, w.in_dtype, 128, "neumann", order=order, resid=resid, kernel="tc2")
    o_ref, S_ref = U.oracle_reference(x, 128, "neumann", order=order, resid=resid)
    eo, es = U.rel_err(o, o_ref), U.rel_err(Sf, S_ref)
    print("rel err o %.3e  S_final %.3e" % (eo, es))
    assert eo <= U.TOL_BF16 and es <= U.TOL_BF16


def test_pair_neumann_segmented():
    from gated_delta_rule_141_b200 import gdr
    w, x = W.workload_inputs(4, Hk=1, Hv=1, T=64 * 60 + 17)
    shape = gdr.make_shape(w.B, w.T, w.Hk, w.Hv, w.dk, w.dv)
    assert gdr.state_segments(shape, 128, gdr.GATE_CHANNEL, "neumann") > 1
    o, Sf = U.run_gpu(x, w.in_dtype, 128, "neumann", kernel="tc2")
    o_ref, S_ref = U.oracle_reference(x, 128, "neumann")
    eo, es = U.rel_err(o, o_ref), U.rel_err(Sf, S_ref)
    print("rel err o %.3e  S_final %.3e" % (eo, es))
    assert eo <= U.TOL_BF16 and es <= U.TOL_BF16
