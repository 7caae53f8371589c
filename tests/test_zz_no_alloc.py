"""gdr_chunk_fwd_static -- the entry point for callers that may not allocate
device memory on their call path (its workspace is a fixed array inside the
library).  Called through the C ABI twice in a row on different inputs, it must give
exactly what gdr_chunk_fwd gives with a caller-owned workspace, and match the
oracle within the bf16 bound of the parity tests; requests too large for the
array are refused before any launch.

The file is named so that pytest collects it after every other test file."""
import ctypes

import numpy as np
import pytest

import gpu_util as U
from gated_delta_rule_141_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    from gated_delta_rule_141_b200 import build as gdr_build
    from gated_delta_rule_141_b200 import gdr
    gdr_build.build()
    return gdr.load()


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _static_call(lib, dev, shape, chunk, gate, o, Sf):
    import torch
    from gated_delta_rule_141_b200 import gdr
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.gdr_chunk_fwd_static(ctypes.byref(shape), _ptr(dev["q"]), _ptr(dev["k"]),
                                    _ptr(dev["v"]), _ptr(dev["g"]), _ptr(dev["beta"]),
                                    _ptr(dev["S0"]), chunk, gate, gdr.INV_EXACT, _ptr(o), _ptr(Sf),
                                    stream)


# (workload, overrides): scalar gate with grouped values; per-channel decay with a
# ragged tail; one long sequence, whose state pass runs segment-parallel (its
# segment states live in the array too)
CASES = [(1, dict(B=2, Hk=2, Hv=4, T=320)), (2, dict(B=1, Hk=2, Hv=2, T=448 - 37)),
         (1, dict(B=1, Hk=1, Hv=1, T=64 * 48 + 1))]


@pytest.mark.parametrize("idx,over", CASES, ids=["w%d-T%d" % (c[0], c[1]["T"]) for c in CASES])
def test_static_entry_matches_workspace_entry(lib, idx, over):
    """Two calls in a row on different seeded inputs: each must equal, bit for bit,
    gdr_chunk_fwd with a caller-owned workspace on the same inputs (the same kernels
    with no atomics, so the same bits), and match the oracle within the bf16
    bound.  Different inputs make stale contents of the shared array visible."""
    import torch
    from gated_delta_rule_141_b200 import gdr
    w, _ = W.workload_inputs(idx, **over)
    gate = gdr.gate_mode_for(w.G, w.dk)
    shape = gdr.make_shape(w.B, w.T, w.Hk, w.Hv, w.dk, w.dv)
    if over["T"] > 64 * 32:
        assert gdr.state_segments(shape, 64, gate) > 1
    for call in range(2):
        _, x = W.workload_inputs(idx, seed=5000 + 17 * call + idx, **over)
        dev = U.to_device(x, "bf16")
        o_ref, S_ref = gdr.chunk_fwd(dev["q"], dev["k"], dev["v"], dev["g"], dev["beta"],
                                     dev["S0"], chunk=64, gate_mode=gate, kernel="tc2")
        o = torch.full((w.B, w.Hv, w.T, w.dv), float("nan"), dtype=torch.bfloat16, device="cuda")
        Sf = torch.full((w.B, w.Hv, w.dk, w.dv), float("nan"), dtype=torch.float32, device="cuda")
        assert _static_call(lib, dev, shape, 64, gate, o, Sf) == gdr.OK
        torch.cuda.synchronize()
        assert gdr.device_status() == gdr.OK
        assert torch.equal(o, o_ref) and torch.equal(Sf, S_ref), "call %d differs" % call
        oo, So = U.oracle_reference(x, 64, "exact")
        eo = U.rel_err(o.float().cpu().numpy(), oo)
        es = U.rel_err(Sf.cpu().numpy(), So)
        print("call %d: rel err vs oracle o %.3e  S_final %.3e" % (call, eo, es))
        assert eo <= U.TOL_BF16 and es <= U.TOL_BF16


def test_static_entry_refuses_oversize_requests(lib):
    from gated_delta_rule_141_b200 import gdr
    # 64 key heads x 4096 chunks of per-channel records is far beyond the array
    big = gdr.make_shape(1, 4096 * 64, 64, 64, 128, 128)
    assert gdr.workspace_bytes(big, 64, gdr.GATE_CHANNEL) > gdr.STATIC_SCRATCH_BYTES
    fake = [ctypes.c_void_p(0x10000 * (i + 1)) for i in range(8)]
    st = lib.gdr_chunk_fwd_static(ctypes.byref(big), *fake[:6], 64, gdr.GATE_CHANNEL,
                                  gdr.INV_EXACT, fake[6], fake[7], None)
    assert st == gdr.ERR_SCRATCH_LIMIT
    # only the two-pass kernel runs here
    forced = gdr.make_shape(1, 64, 1, 1, 128, 128, kernel="tc")
    st = lib.gdr_chunk_fwd_static(ctypes.byref(forced), *fake[:6], 64, gdr.GATE_SCALAR,
                                  gdr.INV_EXACT, fake[6], fake[7], None)
    assert st == gdr.ERR_UNSUPPORTED
