"""The backward (gdr_chunk_bwd: "Systolic Linear Attention: Co-Designing
Tile-Grouped Gated Delta Attention for TPUs", §2.5, custom VJP) through the C ABI
against the oracle's exact gradient of the token recurrence, on the same seeded
inputs and seeded upstream gradients dO, dS_final.  Every gradient (q, k, v, g,
beta, S0) is compared element by element with the relative-error bound of the
fp32 path."""
import numpy as np
import pytest

import gpu_util as U
import oracle
from gated_delta_rule_141_b200 import workloads as W

pytestmark = pytest.mark.gpu

TOL = 1e-4   # fp32 arithmetic throughout (bf16 q, k, v are exact fp32 values)


@pytest.fixture(scope="module", autouse=True)
def _built():
    import torch
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    from gated_delta_rule_141_b200 import build as gdr_build
    gdr_build.build()


# (workload index, overrides, chunk, upstream dS_final?, keep S0?)
CASES = [
    (0, dict(T=130, s0_std=0.5), 64, True, True),                       # fp32, ragged tail
    (0, dict(T=77, dk=32, dv=40), 16, False, False),                    # two value tiles, no S0
    (1, dict(B=1, Hk=2, Hv=4, T=200), 64, True, True),                  # bf16 q k v, grouped values
    (2, dict(B=1, Hk=1, Hv=2, T=150), 32, True, True),                  # per-channel decay
    (3, dict(B=1, Hk=1, Hv=2, T=100), 64, True, True),                  # dk = 256, 64-channel groups
]


def upstream(x, seed, with_dsf):
    rng = np.random.default_rng(seed)
    B, Hv, T, dv = x["v"].shape
    dk = x["q"].shape[3]
    dO = rng.standard_normal((B, Hv, T, dv))
    dSf = rng.standard_normal((B, Hv, dk, dv)) if with_dsf else None
    return dO, dSf


@pytest.mark.parametrize("idx,over,chunk,with_dsf,with_s0", CASES,
                         ids=["w%d-C%d-%s" % (c[0], c[2], "-".join("%s%s" % kv for kv in c[1].items()))
                              for c in CASES])
def test_backward_matches_exact_gradient(idx, over, chunk, with_dsf, with_s0):
    import torch
    from gated_delta_rule_141_b200 import gdr
    w, x = W.workload_inputs(idx, **over)
    if not with_s0:
        x["S0"] = None
    dO, dSf = upstream(x, 7100 + idx, with_dsf)
    dev = U.to_device(x, w.in_dtype)
    dO_d = torch.from_numpy(dO.astype(np.float32)).to("cuda")
    dSf_d = None if dSf is None else torch.from_numpy(dSf.astype(np.float32)).to("cuda")
    got = gdr.chunk_bwd(dev["q"], dev["k"], dev["v"], dev["g"], dev["beta"], dev["S0"], dO_d, dSf_d,
                        chunk=chunk)
    torch.cuda.synchronize()
    assert gdr.device_status() == gdr.OK
    ref = oracle.recurrent_grad(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"], dO, dSf)
    errs = {n: U.rel_err(got[n].cpu().numpy(), ref[n]) for n in ref}
    print(" ".join("d%s %.2e" % kv for kv in errs.items()))
    assert max(errs.values()) <= TOL, errs


def test_backward_full_size_sampled():
    # the gdn_scalar_bf16 workload at full size (B=4, H=16, T=4096, dk=dv=128), the
    # launch bench.py --pass backward times; the oracle's gradient for a sample of
    # key heads (with all their value heads) against the GPU's
    import torch
    from gated_delta_rule_141_b200 import gdr
    w, x = W.workload_inputs(1)
    dO, dSf = upstream(x, 7190, True)
    dev = U.to_device(x, w.in_dtype)
    got = gdr.chunk_bwd(dev["q"], dev["k"], dev["v"], dev["g"], dev["beta"], dev["S0"],
                        torch.from_numpy(dO.astype(np.float32)).to("cuda"),
                        torch.from_numpy(dSf.astype(np.float32)).to("cuda"), chunk=w.chunk)
    torch.cuda.synchronize()
    got = {n: t.cpu().numpy().astype(np.float64) for n, t in got.items()}
    for n, t in got.items():
        assert np.isfinite(t).all(), n
    heads = [(0, 0), (w.B - 1, w.Hk - 1)]              # (batch, key head)
    for b, hk in heads:
        hv = list(range(hk * w.R, (hk + 1) * w.R))
        key = lambda a: a[b:b + 1, hk:hk + 1]
        val = lambda a: a[b:b + 1, hv]
        ref = oracle.recurrent_grad(key(x["q"]), key(x["k"]), val(x["v"]), key(x["g"]),
                                    key(x["beta"]), None if x["S0"] is None else val(x["S0"]),
                                    val(dO), val(dSf))
        errs = {"q": U.rel_err(key(got["q"]), ref["q"]), "k": U.rel_err(key(got["k"]), ref["k"]),
                "g": U.rel_err(key(got["g"]), ref["g"]), "beta": U.rel_err(key(got["beta"]), ref["beta"]),
                "v": U.rel_err(val(got["v"]), ref["v"]), "S0": U.rel_err(val(got["S0"]), ref["S0"])}
        print((b, hk), " ".join("d%s %.2e" % kv for kv in errs.items()))
        assert max(errs.values()) <= TOL, errs
