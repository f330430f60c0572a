"""B200 (sm_100a) library for the routed-expert matrix multiply of a trellis-coded
(T16 bitshift-trellis) quantised MoE layer.

The compute path is the C-ABI shared library ``libtrellis_moe.so`` built from
``csrc/``; ``api`` is a thin ctypes binding with the same entry-point names.  The
library is loaded on first use and an import or call fails loudly when it is missing:
there is no CPU fallback.
"""
import importlib

__all__ = ["api", "inputs"]


def __getattr__(name):
    if name in __all__:
        return importlib.import_module("." + name, __name__)
    raise AttributeError(name)
