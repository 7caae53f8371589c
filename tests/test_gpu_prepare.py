"""GPU parity of the chunk-parallel first pass (gdr_chunk_prepare) on its own:
the per-chunk factors T = diag(beta) (I + M)^{-1} and L, decoded from the tile
images the kernel writes, against the oracle's chunk matrices and inverse
(fp64) on the same seeded inputs.  Bound: 2e-2 of max|ref| per chunk (bf16
inputs and bf16 output tiles, fp32 accumulation)."""
import numpy as np
import pytest

import gpu_util as U
import oracle
from gated_delta_rule_141_b200 import workloads as W

pytestmark = pytest.mark.gpu

TOL = 2e-2


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    from gated_delta_rule_141_b200 import build as gdr_build
    gdr_build.build()


def decode(record: np.ndarray):
    """One 16384-byte chunk record -> (T, L) as float64 64 x 64 matrices.  The
    16-byte piece with columns 8c..8c+7 of row r sits at (c XOR r % 8)."""
    u16 = record.view(np.uint16).reshape(2, 64, 8, 8)         # [T|L][row][piece][elem]
    out = []
    for m in range(2):
        rows = np.empty((64, 8, 8), np.uint16)
        for r in range(64):
            rows[r] = u16[m, r][np.arange(8) ^ (r % 8)]
        out.append((rows.reshape(64, 64).astype(np.uint32) << 16).view(np.float32)
                   .astype(np.float64))
    return out


def reference(x, b, hk, n, inverse, order=4, resid=1):
    T = x["q"].shape[2]
    lo, hi = 64 * n, min(64 * n + 64, T)
    Cl = hi - lo
    _, M, L = oracle.chunk_matrices(x["q"][b, hk, lo:hi], x["k"][b, hk, lo:hi],
                                    x["g"][b, hk, lo:hi], x["beta"][b, hk, lo:hi])
    A = oracle.tril_inverse(M) if inverse == "exact" else oracle.neumann_inverse(M, order, resid)
    Tm = np.zeros((64, 64))
    Lm = np.zeros((64, 64))
    Tm[:Cl, :Cl] = x["beta"][b, hk, lo:hi, None] * A
    Lm[:Cl, :Cl] = L
    return Tm, Lm


# (workload, overrides, inverse, extra gate scaling)
CASES = [
    (1, dict(B=1, Hk=2, T=256), "exact", None),                        # scalar gate
    (1, dict(B=1, Hk=1, T=200), "neumann", None),                      # ragged, Neumann
    (2, dict(B=1, Hk=2, T=192), "exact", None),                        # per channel, weak decay
    (2, dict(B=1, Hk=1, T=130, gate_mode=W.GATE_GROUP64), "exact", None),
    (2, dict(B=1, Hk=1, T=128), "neumann", None),
    (4, dict(Hk=2, T=256), "exact", None),                             # strong decay
    (4, dict(Hk=1, T=192), "exact", 8.0),                              # decay past the pivot guard
    (3, dict(B=1, Hk=2, T=160), "exact", None),                        # dk = 256, four groups
]


@pytest.mark.parametrize("idx,over,inverse,gscale", CASES,
                         ids=["w%d-%s-%s%s" % (c[0], "-".join("%s%s" % kv for kv in c[1].items()),
                                               c[2], "" if c[3] is None else "-g%g" % c[3])
                              for c in CASES])
def test_prepare_matches_oracle(idx, over, inverse, gscale):
    import torch
    from gated_delta_rule_141_b200 import gdr
    w, x = W.workload_inputs(idx, **over)
    if gscale is not None:
        x["g"] = (x["g"] * gscale).astype(np.float32)
    dev = U.to_device(x, "bf16")
    fac = gdr.chunk_prepare(dev["q"], dev["k"], dev["g"], dev["beta"], chunk=64,
                            inverse=inverse)
    torch.cuda.synchronize()
    assert gdr.device_status() == gdr.OK
    fac = fac.cpu().numpy()
    B, Hk, nch = fac.shape[:3]
    worst = 0.0
    for b in range(B):
        for hk in range(Hk):
            for n in range(nch):
                Tg, Lg = decode(fac[b, hk, n])
                Tr, Lr = reference(x, b, hk, n, inverse)
                et, el = U.rel_err(Tg, Tr), U.rel_err(Lg, Lr)
                worst = max(worst, et, el)
                assert et <= TOL and el <= TOL, (b, hk, n, et, el)
    print("worst chunk rel err %.3e" % worst)
