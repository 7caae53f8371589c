"""Chunk-boundary momentum ("Systolic Linear Attention: Co-Designing Tile-Grouped
Gated Delta Attention for TPUs", §2.3): the CUDA-core kernel and the two-pass
tensor-core path through the C ABI (gdr_chunk_fwd_momentum) against the oracle's
chunked form with momentum, on the same seeded inputs; kappa is a seeded 0/1
array of per-chunk gates."""
import numpy as np
import pytest

import gpu_util as U
import oracle
from gated_delta_rule_141_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    import torch
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    from gated_delta_rule_141_b200 import build as gdr_build
    gdr_build.build()


# (workload index, overrides, chunk, inverse, mu, kappa drawn?)
CASES = [
    (0, dict(T=203, s0_std=0.5), 64, "exact", 0.9, True),              # fp32, ragged tail, S0
    (0, dict(T=130, dv=40, gate_mode=W.GATE_CHANNEL), 32, "neumann", 0.5, False),
    (0, dict(T=77, dk=32, dv=16), 16, "neumann1", -0.3, True),         # chunk below the value tile
    (1, dict(B=2, Hk=2, Hv=4, T=320 - 13), 64, "exact", 0.9, True),    # bf16, grouped value heads
    (2, dict(B=1, Hk=2, Hv=2, T=256), 64, "exact", 0.7, True),         # bf16, per-channel decay
]

# the same on the two-pass tensor-core path (the velocity in tensor memory): scalar,
# grouped and per-channel gates, ragged tails, S0, grouped value heads, the Neumann
# inverses, strong decay
TC2_CASES = [
    (1, dict(B=2, Hk=2, Hv=4, T=320 - 13), 64, "exact", 0.9, True),
    (1, dict(B=1, Hk=1, Hv=1, T=256), 64, "exact", 0.25, False),
    (2, dict(B=1, Hk=2, Hv=2, T=256 - 27), 64, "exact", 0.7, True),
    (2, dict(B=1, Hk=1, Hv=2, T=200, gate_mode=W.GATE_GROUP64), 64, "neumann", 0.5, True),
    (2, dict(B=1, Hk=1, Hv=1, T=192), 64, "neumann1", -0.3, True),
    (4, dict(Hk=1, Hv=1, T=640 - 5), 64, "exact", 0.25, True),
]


def _kappa(B, T, chunk, seed):
    rng = np.random.default_rng(seed)
    nch = (T + chunk - 1) // chunk
    return (rng.random((B, nch)) < 0.75).astype(np.int32)


@pytest.mark.parametrize("idx,over,chunk,inverse,mu,with_kappa", CASES,
                         ids=["w%d-C%d-%s-mu%g-%s" % (c[0], c[2], c[3], c[4], "kappa" if c[5] else "ones")
                              for c in CASES])
def test_momentum_parity(idx, over, chunk, inverse, mu, with_kappa):
    import torch
    from gated_delta_rule_141_b200 import gdr
    w, x = W.workload_inputs(idx, **over)
    B, T = x["q"].shape[0], x["q"].shape[2]
    kappa = _kappa(B, T, chunk, 9000 + idx) if with_kappa else None
    dev = U.to_device(x, w.in_dtype)
    kd = None if kappa is None else torch.from_numpy(kappa).to("cuda")
    o, Sf = gdr.chunk_fwd_momentum(dev["q"], dev["k"], dev["v"], dev["g"], dev["beta"], dev["S0"],
                                   mu=mu, kappa=kd, chunk=chunk, inverse=inverse, kernel="simt")
    torch.cuda.synchronize()
    o = o.float().cpu().numpy().astype(np.float64)
    Sf = Sf.cpu().numpy().astype(np.float64)
    o_ref, S_ref = oracle.chunked(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"], chunk=chunk,
                                  inverse=inverse, mu=mu, kappa=kappa)
    tol = U.tol_for(w.in_dtype)
    eo, es = U.rel_err(o, o_ref), U.rel_err(Sf, S_ref)
    print("rel err o %.3e  S_final %.3e  (tol %.0e)" % (eo, es, tol))
    assert eo <= tol and es <= tol


@pytest.mark.parametrize("idx,over,chunk,inverse,mu,with_kappa", TC2_CASES,
                         ids=["w%d-C%d-%s-mu%g-%s" % (c[0], c[2], c[3], c[4], "kappa" if c[5] else "ones")
                              for c in TC2_CASES])
def test_momentum_parity_tensor_cores(idx, over, chunk, inverse, mu, with_kappa):
    import torch
    from gated_delta_rule_141_b200 import gdr
    w, x = W.workload_inputs(idx, **over)
    B, T = x["q"].shape[0], x["q"].shape[2]
    kappa = _kappa(B, T, chunk, 9200 + idx) if with_kappa else None
    dev = U.to_device(x, w.in_dtype)
    kd = None if kappa is None else torch.from_numpy(kappa).to("cuda")
    o, Sf = gdr.chunk_fwd_momentum(dev["q"], dev["k"], dev["v"], dev["g"], dev["beta"], dev["S0"],
                                   mu=mu, kappa=kd, chunk=chunk, inverse=inverse, kernel="tc2")
    torch.cuda.synchronize()
    assert gdr.device_status() == gdr.OK
    o = o.float().cpu().numpy().astype(np.float64)
    Sf = Sf.cpu().numpy().astype(np.float64)
    o_ref, S_ref = oracle.chunked(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"], chunk=chunk,
                                  inverse=inverse, mu=mu, kappa=kappa)
    eo, es = U.rel_err(o, o_ref), U.rel_err(Sf, S_ref)
    print("rel err o %.3e  S_final %.3e" % (eo, es))
    assert eo <= U.TOL_BF16 and es <= U.TOL_BF16


def test_momentum_zero_is_plain_forward():
    # mu = 0 leaves only the chunk's own update: the plain forward's result
    import torch
    from gated_delta_rule_141_b200 import gdr
    w, x = W.workload_inputs(0, T=150, s0_std=0.3)
    dev = U.to_device(x, w.in_dtype)
    o1, S1 = gdr.chunk_fwd_momentum(dev["q"], dev["k"], dev["v"], dev["g"], dev["beta"], dev["S0"],
                                    mu=0.0, chunk=32)
    o2, S2 = gdr.chunk_fwd(dev["q"], dev["k"], dev["v"], dev["g"], dev["beta"], dev["S0"], chunk=32,
                           kernel="simt")
    torch.cuda.synchronize()
    assert U.rel_err(o1.cpu().numpy(), o2.cpu().numpy()) <= 1e-6
    assert U.rel_err(S1.cpu().numpy(), S2.cpu().numpy()) <= 1e-6


def test_momentum_full_size_sampled():
    # the gdn_scalar_bf16 workload at full size (B=4, H=16, T=4096, dk=dv=128) with the
    # pages' mu = 0.25 and a seeded kappa, in the launch bench.py --momentum times (the
    # two-pass tensor-core path);
    # checked on a sample of sequences against the oracle
    import torch
    from gated_delta_rule_141_b200 import gdr
    w, x = W.workload_inputs(1)
    chunk, mu = w.chunk, 0.25
    kappa = _kappa(w.B, w.T, chunk, 9100)
    dev = U.to_device(x, w.in_dtype)
    o, Sf = gdr.chunk_fwd_momentum(dev["q"], dev["k"], dev["v"], dev["g"], dev["beta"], dev["S0"],
                                   mu=mu, kappa=torch.from_numpy(kappa).to("cuda"), chunk=chunk)
    torch.cuda.synchronize()
    o = o.float().cpu().numpy().astype(np.float64)
    Sf = Sf.cpu().numpy().astype(np.float64)
    assert np.isfinite(o).all() and np.isfinite(Sf).all()
    seqs = U.sample_sequences(w)
    xs = U.slice_sequences(x, w.R, seqs)
    kap = np.stack([kappa[b] for b, _ in seqs])
    o_ref, S_ref = oracle.chunked(xs["q"], xs["k"], xs["v"], xs["g"], xs["beta"], xs["S0"],
                                  chunk=chunk, inverse="exact", mu=mu, kappa=kap)
    ib, ih = [b for b, _ in seqs], [h for _, h in seqs]
    eo = U.rel_err(o[ib, ih][:, None], o_ref)
    es = U.rel_err(Sf[ib, ih][:, None], S_ref)
    print("rel err o %.3e  S_final %.3e" % (eo, es))
    assert eo <= U.TOL_BF16 and es <= U.TOL_BF16
