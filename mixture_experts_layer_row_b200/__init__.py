"""B200-native (sm_100a) Mixture-of-Experts expert layer: C-ABI library + thin ctypes binding.

The compute path lives in libmoe_b200.so (built by `python mixture_experts_layer_row_b200/build.py`);
importing this package without the built library raises ImportError.
"""
from . import _lib
from ._lib import MoEError, version
from .layer import MoELayer

__all__ = ["_lib", "MoEError", "MoELayer", "version"]
