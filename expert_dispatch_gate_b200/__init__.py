"""B200-native MoE layer forward path (router -> capacity-limited grouping -> grouped SwiGLU
experts -> weighted combine) behind the C ABI of libmoe.so.

``expert_dispatch_gate_b200._lib`` binds the C ABI (same names as include/moe.h);
``expert_dispatch_gate_b200.layer`` allocates outputs/workspace with PyTorch and calls it;
``expert_dispatch_gate_b200.workloads`` draws the seeded synthetic inputs.
"""
__all__ = ["_lib", "layer", "workloads", "build"]
