"""B200-native chunkwise gated delta-rule forward.

The computation runs in ``libgdr.so`` (hand-written sm_100a CUDA behind a
C ABI declared in ``include/gdr.h``).  ``gated_delta_rule_141_b200.gdr`` is the
thin ctypes binding with the same names; submodules are imported on demand so
that the seeded input generators in ``workloads`` load on machines without a
GPU.
"""
import importlib

__all__ = ["gdr", "workloads"]


def __getattr__(name):
    if name in __all__:
        return importlib.import_module(__name__ + "." + name)
    raise AttributeError(name)
