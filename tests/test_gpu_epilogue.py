"""Readout epilogue of the SLA recurrence ("Systolic Linear Attention ...", §2.3
Eq. (5)): o <- sigmoid(z) * RMSNorm(o) per (token, value head) row, on the GPU
(gdr_output_gate_rmsnorm) against the oracle's fp64 definition.

The kernel alone is compared on identical inputs (what the GPU holds, rounded
to bf16 for the bf16 case): fp32 within 1e-5, bf16 within the output's bf16
rounding (1e-2 of the largest output).  The whole readout (chunk forward, then
the epilogue) is compared with the oracle's token recurrence plus epilogue
within the bf16 bound of the parity tests."""
import numpy as np
import pytest

import gpu_util as U
import oracle
from gated_delta_rule_141_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _torch():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    return torch


@pytest.mark.parametrize("dtype,dv,weighted", [("f32", 128, True), ("bf16", 128, True),
                                               ("bf16", 40, False), ("bf16", 256, True)])
def test_epilogue_kernel(dtype, dv, weighted):
    torch = _torch()
    from gated_delta_rule_141_b200 import gdr
    rng = np.random.default_rng(21 + dv)
    o = rng.standard_normal((2, 3, 37, dv)).astype(np.float32) * 0.3
    z = rng.standard_normal((2, 3, 37, dv)).astype(np.float32) * 2.0
    w = (rng.standard_normal(dv) * 0.5 + 1.0).astype(np.float32) if weighted else None
    if dtype == "bf16":
        o, z = W.round_to_bf16(o), W.round_to_bf16(z)
    dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    od = torch.from_numpy(o).cuda().to(dt)
    zd = torch.from_numpy(z).cuda().to(dt)
    wd = None if w is None else torch.from_numpy(w).cuda()
    gdr.output_gate_rmsnorm(od, zd, wd, eps=1e-6)
    torch.cuda.synchronize()
    got = od.float().cpu().numpy()
    ref = oracle.output_gate_rmsnorm(o, z, w, eps=1e-6)
    err = U.rel_err(got, ref)
    print("rel err %.3e" % err)
    assert err <= (1e-5 if dtype == "f32" else 1e-2)


def test_readout_with_epilogue():
    torch = _torch()
    from gated_delta_rule_141_b200 import gdr
    w_, x = W.workload_inputs(1, B=1, Hk=2, Hv=2, T=320 - 13)
    rng = np.random.default_rng(5)
    z = W.round_to_bf16(rng.standard_normal((w_.B, w_.Hv, w_.T, w_.dv)).astype(np.float32))
    wt = (rng.standard_normal(w_.dv) * 0.5 + 1.0).astype(np.float32)
    dev = U.to_device(x, "bf16")
    o, _ = gdr.chunk_fwd(dev["q"], dev["k"], dev["v"], dev["g"], dev["beta"], dev["S0"], chunk=64)
    gdr.output_gate_rmsnorm(o, torch.from_numpy(z).cuda().to(torch.bfloat16),
                            torch.from_numpy(wt).cuda(), eps=1e-6)
    torch.cuda.synchronize()
    o_ref, _ = oracle.recurrent(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"])
    ref = oracle.output_gate_rmsnorm(o_ref, z, wt, eps=1e-6)
    err = U.rel_err(o.float().cpu().numpy(), ref)
    print("rel err %.3e" % err)
    assert err <= U.TOL_BF16
