"""CPU oracle for the grouped MXFP8 MoE expert MLP.

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the
benchmark's CPU-baseline leg may import this package.  The CUDA product
path never calls it, and the two share no code: this package has its own
MXFP8 codec, its own permutation and its own per-expert loop, all in
float64 with numpy.

Sources (pages of "Efficient MoE Training for Biological Foundation Models"):
* Challenge 1 (the Hugging Face per-expert loop and GroupedLinear with
  split_sizes) -- routing, gather by expert, index_add combine.
* Challenge 2 -- MXFP8: 8-bit values, one scale per 32 consecutive values.
* Challenge 3 -- quantise before each low-precision GEMM, BF16 master
  weights, GroupedLinear(gate_up) -> ScaledSwiGLU -> GroupedLinear(down),
  with the routing probability applied inside ScaledSwiGLU.

* The router (router.py): the pages show only where the routing weights
  are consumed; softmax over the experts, the k largest kept (ties to the
  lower id) and renormalised is the reading taken.

Every reading the pages leave open (scale rounding, gate/up order, saved
activations, backward quantisation directions, padding of ragged blocks) is
stated at the function that takes it.

Pins (tests/test_oracle_*.py): the codec against brute force and library
casts over every bf16 pattern; the forward against an independent
restatement of the per-expert loop; an identity-weight expert against its
closed form; the backward against central finite differences and the
closed form of d(prob); invariants of the permutation and the codec; the
quantisation axis of every GEMM operand by inputs scaled along one axis
(with planted axis swaps that must fail); the router against brute force
over expert subsets, its closed form and torch.
Parity unpinned: bit-level agreement of the scale rule with NVIDIA
Transformer Engine (not available here).
"""
from . import mxfp8, moe, router  # noqa: F401
