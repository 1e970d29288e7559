"""B200-native decode megakernel: one decode step of a decoder-only transformer as one persistent kernel.

The compute runs in ``libmk.so`` (CUDA, sm_100a); the ``mk`` submodule only
marshals arguments to its C ABI (``include/mk.h``).  There is no CPU path:
importing ``auto_regressive_decode_b200.mk`` raises if the library is missing.
"""
import importlib


def __getattr__(name):
    if name.startswith("__"):
        raise AttributeError(name)
    return getattr(importlib.import_module(__name__ + ".mk"), name)
