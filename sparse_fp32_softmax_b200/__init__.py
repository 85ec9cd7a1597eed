"""B200-native forward pass of a Qwen-family sparse MoE FFN block.

The compute path is the C-ABI library ``libmoe_b200.so`` (hand-written sm_100a CUDA);
``sparse_fp32_softmax_b200.binding`` is a thin ctypes binding with the library's own names
(moe_route, moe_permute, moe_forward, moe_forward_ex, ...).  Importing the package does not
load the library; the binding's first call does, and fails loudly when it is missing.
"""
from .inputs import CONFIGS, MoEConfig, make_layer  # noqa: F401
