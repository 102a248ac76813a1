"""CPU oracle for the NF4 fused-expert MoE layer.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call or
execute anything in this package: only the test-suite, the smoke check of the
graft entry point and the CPU-baseline leg of the benchmark use it.  It shares
no code, tables or constants with the CUDA library; it holds its own copy of
the NF4 codebook and computes everything in float64 (float32 only where the
method fixes it: the scaled value ``w / absmax`` of the quantiser).

Modules
-------
nf4      the 16-entry codebook, the blockwise stack quantiser, dequantisation
fp4      the same blockwise storage with e2m1 codes scaled to [-1, 1] (the
         pages' other 4-bit storage mode)
routing  router top-k, the renormalised weights, the token/expert permutation
moe      the grouped NF4 GEMM, the SwiGLU expert MLP with its optional LoRA
         delta, the weighted combine; a brute-force per-token form and a
         permuted grouped form of the same layer
mxfp4    e2m1 codes with e8m0 block-32 scales (the OCP microscaling format of
         released checkpoints) and their grouped GEMM
backward the layer's gradients through the frozen NF4 experts (input,
         router logits, LoRA A and B) with the routing ids held fixed, per
         token and in the grouped form built on the grouped dgrad product

Parity status: every function here is pinned by a ``-m "not gpu"`` test
against closed forms, brute force, invariants or a textbook routine, except
the reading noted in ``nf4``: byte-compatibility with the bitsandbytes
library's own packed bytes is parity unpinned (no such bytes are printed on the
pages and the library is not available to produce them).
"""
