"""NF4 fused-expert MoE layer for B200 (sm_100a): C-ABI library + thin binding.

``quantized_moe_expert_nf4_b200.e4b`` binds the four calls of include/e4b.h
(quantise a fused stack, route/permute, grouped NF4 GEMM, the layer forward);
``workloads`` draws the seeded synthetic inputs; ``build`` compiles libe4b.so
in-tree.  Importing the package does not load the library.
"""
__all__ = ["e4b", "workloads", "build"]
