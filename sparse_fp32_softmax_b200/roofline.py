"""Algorithmic byte and FLOP counts of one MoE block forward pass.

These are the counts a roofline is taken against: what the method must move and compute,
not what an implementation happens to move (permuted copies, the intermediate h, the slot
buffer and L2 re-reads are not credited).

Parameter split: "27. Mixture of experts" (inference.shantanugoel.com), the stored/active
parameter function after the 'Note' box: per layer, each routed expert holds 3*D*I weights
(gate, up, down), the router holds E*D, a shared expert 3*D*I_s; a token touches k routed
experts, the shared expert and the whole router.
"""
from __future__ import annotations

BF16 = 2


def moe_parameter_split(hidden, layers, experts, top_k, intermediate, shared_intermediate=0):
    """(stored, active-per-token) expert-side parameter counts over ``layers`` MoE blocks."""
    expert = 3 * hidden * intermediate
    router = experts * hidden
    shared = 3 * hidden * shared_intermediate
    stored = layers * (experts * expert + router + shared)
    active = layers * (top_k * expert + router + shared)
    return stored, active


def expected_touched(E, k, T):
    """Expected distinct experts hit by T tokens routing uniformly to k of E:
    E * (1 - (1 - k/E)^T) ("27. Mixture of experts", section 'The economics of MoE inference')."""
    return E * (1.0 - (1.0 - k / E) ** T)


def algorithmic_bytes(T, D, E, k, I, touched, I_s=0, shared_gated=False, residual=False,
                      fp8_experts=False):
    """HBM bytes the block cannot avoid: each touched expert's weights once, the router,
    the shared expert (+ its gate vector), x in and y out (+ the residual in).  FP8 experts:
    one byte per weight plus an FP32 scale per weight row (2I + D rows per expert)."""
    if fp8_experts:
        b = touched * (3 * D * I + 4 * (2 * I + D)) + E * D * BF16
    else:
        b = touched * 3 * D * I * BF16 + E * D * BF16
    if I_s:
        b += 3 * D * I_s * BF16 + (D * BF16 if shared_gated else 0)
    b += 2 * T * D * BF16
    if residual:
        b += T * D * BF16
    return b


def algorithmic_flops(T, D, E, k, I, I_s=0, shared_gated=False):
    """Active FLOPs: k SwiGLU experts per token (3 matrices of D x I), the router, and the
    shared expert (+ its gate dot product)."""
    f = 2 * T * k * 3 * D * I + 2 * T * D * E
    if I_s:
        f += 2 * T * 3 * D * I_s + (2 * T * D if shared_gated else 0)
    return f


def expert_weight_bytes(D, I, experts):
    """Bytes of the gate_up and down weights of ``experts`` experts (the decode stream)."""
    return experts * 3 * D * I * BF16


def roofline_time_s(bytes_, flops, hbm_gbs, tflops):
    return max(bytes_ / (hbm_gbs * 1e9), flops / (tflops * 1e12))
