"""B200-native Qwen-family sparse MoE FFN block: the forward pass, its backward pass for a
given routing, and the router's Switch balance loss.

The compute path is the C-ABI library ``libmoe_b200.so`` (hand-written sm_100a CUDA);
``sparse_fp32_softmax_b200.binding`` is a thin ctypes binding with the library's own names
(moe_route, moe_permute, moe_forward, moe_forward_ex, moe_backward, moe_aux_loss, ...).  Importing the package does not
load the library; the binding's first call does, and fails loudly when it is missing.
"""
from .inputs import CONFIGS, MoEConfig, make_layer  # noqa: F401
