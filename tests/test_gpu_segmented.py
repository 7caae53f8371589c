"""Segment-parallel state pass of the two-pass tensor-core path.

For few, long sequences the state pass cuts each sequence into segments: every
segment's end state from zero (B~) and the product of its chunk transitions
A_c = F_c - Khat_c^T W_c (A~, from the identity with no values) are formed in
parallel, composed in order into each segment's start state, and the segments
then run again from those states ("In-GPU affine two-level scan", the state
recurrence S_c = A_c S_{c-1} + B_c of the chunkwise form).  The composition is
exact algebra, so the result must match the oracle's token recurrence within the
bf16 bound like the sequential pass does.

The shapes below are chosen so that the segmented form is selected (its buffers
show up in the workspace size) and that segments end inside the sequence and on
a ragged last chunk.
"""
import numpy as np
import pytest

import gpu_util as U
from gated_delta_rule_141_b200 import workloads as W

pytestmark = pytest.mark.gpu

CASES = [
    (1, dict(B=1, Hk=1, Hv=1, T=64 * 48 + 1)),    # scalar gate, S0, one-token last chunk
    (1, dict(B=1, Hk=1, Hv=2, T=64 * 48)),        # two value heads share one transition
    (2, dict(B=1, Hk=1, Hv=1, T=64 * 52 - 9)),    # per-channel decay
    (4, dict(Hk=1, Hv=1, T=64 * 49 - 7)),         # strong per-channel decay, S0
]


def _records_bytes(w):
    from gated_delta_rule_141_b200 import gdr
    rec = gdr.TC2_SCALAR_RECORD_BYTES if w.G == 1 else gdr.TC2_EXT_RECORD_BYTES
    return w.B * w.Hk * ((w.T + 63) // 64) * rec


@pytest.mark.parametrize("idx,over", CASES,
                         ids=["w%d-%s" % (c[0], "-".join("%s%s" % kv for kv in c[1].items())) for c in CASES])
def test_segmented_state_pass(idx, over):
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    from gated_delta_rule_141_b200 import gdr
    w, x = W.workload_inputs(idx, **over)
    shape = gdr.make_shape(w.B, w.T, w.Hk, w.Hv, w.dk, w.dv)
    need = gdr.workspace_bytes(shape, 64, gdr.gate_mode_for(w.G, w.dk))
    assert need > _records_bytes(w), "the segmented state pass was not selected"
    o, Sf = U.run_gpu(x, w.in_dtype, 64, "exact", kernel="tc2")
    o_ref, S_ref = U.oracle_reference(x, 64, "exact")
    eo, es = U.rel_err(o, o_ref), U.rel_err(Sf, S_ref)
    print("rel err o %.3e  S_final %.3e" % (eo, es))
    assert np.isfinite(o).all() and np.isfinite(Sf).all()
    assert eo <= U.TOL_BF16 and es <= U.TOL_BF16


# The 128-column state pass (forced): one CTA per head and 128 value columns per
# segment, the first value tile of each key head also carrying its transition;
# U / P / E / O sharing one tensor-memory buffer.
WIDE = [
    (4, dict(Hk=1, Hv=1, T=64 * 60 + 17)),        # strong per-channel decay, S0
    (4, dict(B=2, Hk=2, Hv=4, T=64 * 64 + 3)),    # two batch entries, two value heads per key head
    (2, dict(B=1, Hk=1, Hv=2, T=64 * 52 - 9)),    # two value heads, one transition
    (2, dict(B=1, Hk=1, Hv=1, T=64 * 48, dv=256, gate_mode=W.GATE_GROUP64)),   # two value tiles
]


@pytest.mark.parametrize("idx,over", WIDE,
                         ids=["w%d-%s" % (c[0], "-".join("%s%s" % kv for kv in c[1].items())) for c in WIDE])
def test_wide_segmented_state_pass(idx, over):
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    from gated_delta_rule_141_b200 import gdr
    w, x = W.workload_inputs(idx, **over)
    shape = gdr.make_shape(w.B, w.T, w.Hk, w.Hv, w.dk, w.dv, kernel="tc2w")
    assert gdr.state_segments(shape, 64, gdr.gate_mode_for(w.G, w.dk)) > 1
    o, Sf = U.run_gpu(x, w.in_dtype, 64, "exact", kernel="tc2w")
    o_ref, S_ref = U.oracle_reference(x, 64, "exact")
    eo, es = U.rel_err(o, o_ref), U.rel_err(Sf, S_ref)
    print("rel err o %.3e  S_final %.3e" % (eo, es))
    assert np.isfinite(o).all() and np.isfinite(Sf).all()
    assert eo <= U.TOL_BF16 and es <= U.TOL_BF16


# The chunk-128 Neumann inverses run as pairs of 64-token halves: segments start at
# even halves, a second half adds Y E1 in both launches (ends / transitions and
# outputs); odd half counts leave a last half unpaired.
WIDE_PAIRS = [
    (4, dict(Hk=1, Hv=1, T=64 * 60 + 17), "neumann"),
    (4, dict(B=2, Hk=2, Hv=4, T=64 * 66 + 3), "neumann"),
    (2, dict(B=1, Hk=1, Hv=1, T=64 * 48, dv=256, gate_mode=W.GATE_GROUP64), "neumann1"),
    (2, dict(B=1, Hk=1, Hv=2, T=64 * 52 - 9), "neumann1"),
    # weak decay: the halves' W (written by the pair kernel) weigh on every output
    (2, dict(B=1, Hk=1, Hv=2, T=64 * 52 - 9), "neumann"),
]


@pytest.mark.parametrize("idx,over,inverse", WIDE_PAIRS,
                         ids=["w%d-%s-%s" % (c[0], "-".join("%s%s" % kv for kv in c[1].items()), c[2])
                              for c in WIDE_PAIRS])
def test_wide_segmented_pairs(idx, over, inverse):
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    from gated_delta_rule_141_b200 import gdr
    w, x = W.workload_inputs(idx, **over)
    shape = gdr.make_shape(w.B, w.T, w.Hk, w.Hv, w.dk, w.dv, kernel="tc2w")
    assert gdr.state_segments(shape, 128, gdr.gate_mode_for(w.G, w.dk), inverse) > 1
    o, Sf = U.run_gpu(x, w.in_dtype, 128, inverse, kernel="tc2w")
    o_ref, S_ref = U.oracle_reference(x, 128, inverse)
    eo, es = U.rel_err(o, o_ref), U.rel_err(Sf, S_ref)
    print("rel err o %.3e  S_final %.3e" % (eo, es))
    assert np.isfinite(o).all() and np.isfinite(Sf).all()
    assert eo <= U.TOL_BF16 and es <= U.TOL_BF16
