"""The two-pass CUDA-core form (GDR_KERNEL_SIMT2: the chunk inverse and L of every
chunk in parallel, then the value tiles' pass reading them) through the C ABI
against the oracle on the same seeded inputs: every inverse mode, small cases
with ragged tails, and the chunk-128 Neumann configuration of the grouped-value
workload at full size on a sample of sequences."""
import numpy as np
import pytest

import gpu_util as U
from gated_delta_rule_141_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    import torch
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    from gated_delta_rule_141_b200 import build as gdr_build
    gdr_build.build()


# (workload index, overrides, chunk, inverse)
CASES = [
    (0, {}, 64, "exact"),                                               # fp32, the whole workload
    (0, dict(T=203, Hk=1, Hv=3, dv=40, s0_std=0.5), 32, "neumann"),     # ragged, grouped values
    (0, dict(T=93, dv=40, gate_mode=W.GATE_CHANNEL), 24, "neumann1"),
    (3, dict(B=1, Hk=1, Hv=4, T=300), 128, "neumann"),                  # bf16, dk = 256, G = 4
    (4, dict(Hk=1, Hv=1, T=300), 128, "neumann"),                       # strong per-channel decay
    (4, dict(Hk=1, Hv=1, T=300), 128, "neumann1"),
]


@pytest.mark.parametrize("idx,over,chunk,inverse", CASES,
                         ids=["w%d-C%d-%s-%s" % (c[0], c[2], c[3], "-".join("%s%s" % kv for kv in c[1].items())
                                                  or "full") for c in CASES])
def test_two_pass_simt_parity(idx, over, chunk, inverse):
    w, x = W.workload_inputs(idx, **over)
    o, Sf = U.run_gpu(x, w.in_dtype, chunk, inverse, kernel="simt2")
    o_ref, S_ref = U.oracle_reference(x, chunk, inverse)
    tol = U.tol_for(w.in_dtype)
    eo, es = U.rel_err(o, o_ref), U.rel_err(Sf, S_ref)
    print("rel err o %.3e  S_final %.3e  (tol %.0e)" % (eo, es, tol))
    assert eo <= tol and es <= tol


def test_two_pass_simt_full_size_sampled():
    # kda-style grouped workload (B=2, T=8192, Hk=8, dk=256, Hv=32, dv=128, G=4) with
    # the Neumann inverse at chunk 128, as bench.py --kernel simt2 runs it
    w, x = W.workload_inputs(3)
    o, Sf = U.run_gpu(x, w.in_dtype, 128, "neumann", kernel="simt2")
    assert np.isfinite(o).all() and np.isfinite(Sf).all()
    seqs = U.sample_sequences(w)
    xs = U.slice_sequences(x, w.R, seqs)
    o_ref, S_ref = U.oracle_reference(xs, 128, "neumann")
    ib, ih = [b for b, _ in seqs], [h for _, h in seqs]
    eo = U.rel_err(o[ib, ih][:, None], o_ref)
    es = U.rel_err(Sf[ib, ih][:, None], S_ref)
    print("rel err o %.3e  S_final %.3e" % (eo, es))
    assert eo <= U.TOL_BF16 and es <= U.TOL_BF16
