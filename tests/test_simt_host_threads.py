"""Race check of the CUDA-core kernels on the host, without a GPU.

Their source (gdr_simt.cu: one-pass forward, momentum, the two-pass form;
gdr_bwd.cu: the backward) is built with g++ -fsanitize=thread against the
stand-in headers in tests/host_emu/threads/: each CUDA thread of a CTA is a host
thread and __syncthreads() a std::barrier, so ThreadSanitizer reports any two
threads touching the same shared or global word within one barrier phase with
at least one write (the atomics are std::atomic_ref).  A copy with one barrier
removed must be reported, which shows the check can fail."""
import os
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(ROOT, "gated_delta_rule_141_b200", "csrc")
EMU = os.path.join(HERE, "host_emu")


def _source(drop_barrier=False):
    def part(name, marker, ns):
        src = open(os.path.join(CSRC, name)).read()
        body = src[:src.index(marker)]
        assert body.count("namespace {") == 1
        body = body.replace("namespace {", "namespace %s {" % ns)
        return body.replace("extern __shared__ float sm[];", "float *const sm = host_smem_ptr();")

    fwd = part("gdr_simt.cu", "template <bool I, bool O, int NV, bool MOM, bool PRE>\nint launch_variant",
               "emu_f")
    bwd = part("gdr_bwd.cu", "template <bool I, int NV>\nint launch_bwd_variant", "emu_b")
    if drop_barrier:   # the barrier between R = V - Kbar S and its use in Y = A R
        old = "            dR[idx] = vv - acc;\n        }\n        __syncthreads();"
        assert bwd.count(old) == 1
        bwd = bwd.replace(old, "            dR[idx] = vv - acc;\n        }")
    main = open(os.path.join(EMU, "threads", "race_main.cpp")).read()
    return ("float *host_smem_ptr();\n" + fwd + "}  // namespace emu_f\n}  // namespace gdr\n" + bwd +
            "}  // namespace emu_b\n}  // namespace gdr\n" + main)


def _build(tmp_path, name, drop_barrier=False):
    cpp = tmp_path / (name + ".cpp")
    cpp.write_text(_source(drop_barrier))
    exe = tmp_path / name
    r = subprocess.run(["g++", "-std=c++20", "-w", "-fsanitize=thread", "-O1", "-g",
                        "-I" + os.path.join(EMU, "threads"), "-I" + EMU, "-I" + CSRC,
                        "-I" + os.path.join(ROOT, "include"), str(cpp), "-o", str(exe), "-lpthread"],
                       capture_output=True, text=True)
    if r.returncode != 0 and "sanitize" in r.stderr:
        pytest.skip("ThreadSanitizer is not available here: " + r.stderr.strip().splitlines()[-1])
    assert r.returncode == 0, r.stderr
    return str(exe)


def _run(exe, *args):
    r = subprocess.run([exe, *map(str, args)], capture_output=True, text=True, timeout=600)
    if "FATAL: ThreadSanitizer" in r.stderr:
        pytest.skip("ThreadSanitizer cannot run here: " + r.stderr.strip().splitlines()[0])
    return r


@pytest.fixture(scope="module")
def race_exe(tmp_path_factory):
    return _build(tmp_path_factory.mktemp("race"), "race")


@pytest.mark.parametrize("G,inverse", [(16, 0), (1, 0), (4, 1), (16, 2)],
                         ids=["per-channel-exact", "scalar-exact", "groups-neumann", "per-channel-neumann1"])
def test_no_data_race(race_exe, G, inverse):
    r = _run(race_exe, G, inverse)
    assert "ThreadSanitizer" not in r.stderr, r.stderr[:4000]
    assert r.returncode == 0, r.stderr[:4000]
    assert "two-pass vs one-pass: max|do| / max|o| = 0.00e+00" in r.stdout, r.stdout


def test_planted_race_is_reported(tmp_path):
    exe = _build(tmp_path, "planted", drop_barrier=True)
    r = _run(exe, 16, 0)
    assert "WARNING: ThreadSanitizer: data race" in r.stderr
