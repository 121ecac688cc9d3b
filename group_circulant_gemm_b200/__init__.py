"""B200-native (sm_100a) Flash EQ-Linear: group-circulant GEMM via the group DFT.

The compute lives in ``libeqlinear.so`` (C ABI declared in include/eqlinear.h);
:mod:`.native` binds it name for name and :class:`EqLinearPlan` wraps it for
torch tensors.  Importing the package does not load the library; the first use
of ``native`` or ``EqLinearPlan`` does, and raises if it is missing.
"""
import importlib

__all__ = ["EqLinearPlan", "forward_chain", "native", "synth"]


def __getattr__(name):
    if name in ("EqLinearPlan", "forward_chain"):
        return getattr(importlib.import_module(".layer", __name__), name)
    if name in ("native", "synth", "layer", "build"):
        return importlib.import_module("." + name, __name__)
    raise AttributeError(name)
