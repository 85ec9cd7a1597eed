"""B200-native forward pass of a Qwen-family sparse MoE FFN block.

The compute path is the C-ABI library ``libmoe_b200.so`` (hand-written sm_100a CUDA); the
Python names below are a thin ctypes binding with the library's own names.  Importing the
package does not load the library; the first call does, and fails loudly when it is missing.
"""
from .inputs import CONFIGS, MoEConfig, make_layer  # noqa: F401


def __getattr__(name):
    from . import binding
    return getattr(binding, name)
