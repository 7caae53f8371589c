"""The failure path of the kernels' bounded waits, exercised without a fault:
the library's self-test launch waits on an mbarrier that nothing arrives on,
gives up after a few microseconds, sets the status word and releases its
tensor memory.  The host must read GDR_ERR_TIMEOUT once (reading clears it),
and the context must stay usable: the next forward on the same stream matches
the oracle and reports no timeout."""
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


def test_bounded_wait_gives_up_and_context_survives():
    import torch
    from gated_delta_rule_141_b200 import gdr
    assert gdr.device_status() == gdr.OK
    assert gdr.selftest_bounded_wait(5000) == gdr.OK          # 5 us limit
    torch.cuda.synchronize()
    assert gdr.device_status() == gdr.ERR_TIMEOUT
    assert gdr.device_status() == gdr.OK                        # reading cleared it
    # out-of-range limits are refused before any launch
    assert gdr.selftest_bounded_wait(10) == gdr.ERR_ARG
    assert gdr.selftest_bounded_wait(5 * 10 ** 9) == gdr.ERR_ARG
    # the same stream still runs the forward correctly
    w, x = W.workload_inputs(2, B=1, Hk=1, Hv=1, T=200)
    o, Sf = U.run_gpu(x, "bf16", 64)        # asserts device_status() == OK itself
    o_ref, S_ref = U.oracle_reference(x, 64, "exact")
    assert U.rel_err(o, o_ref) <= U.TOL_BF16 and U.rel_err(Sf, S_ref) <= U.TOL_BF16
