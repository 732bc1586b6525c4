"""B200-native (sm_100a) DeepSeekMoE layer forward behind a C ABI (libmoe.so).

The kernels live in csrc/ and are built in-tree by `build.py`; `_lib` binds
the C entry points under their own names; `layer.MoELayer` sequences them.
"""
from . import synth  # noqa: F401

__all__ = ["synth", "layer", "_lib", "build"]
