"""CPU oracle of the DeepSeekMoE layer forward -- test infrastructure only.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
and reference arms may import this package.  It shares no code with the GPU
path (``fine_grained_shared_b200``) and neither imports the other; the seeded
input generators in ``workloads`` serve both.  ``oracle.fp8`` holds the
fine-grained FP8 quantization of the expert GEMMs, ``oracle.moe_backward``
the layer's backward pass.
"""
from .moe_oracle import (  # noqa: F401
    GATE_SIGMOID, GATE_SOFTMAX, FLAG_NO_RESIDUAL, FLAG_NO_ROUTED, FLAG_NO_SHARED,
    Permutation, Routing, affinity_logits, bias_update, expert_permutation, f64, gate_values,
    moe_forward, route, select_top_k, select_top_k_node_limited, sigmoid_affinity, silu, softmax_affinity,
    swiglu_ffn,
)
