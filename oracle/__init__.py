"""CPU oracle of the routed-MoE layer over an expert-slot cache.

TEST INFRASTRUCTURE ONLY. This package is a plain, slow, obviously correct
restatement of what the layer computes, used to check the CUDA path. Only
tests/, __graft_entry__.smoke() and bench.py's CPU-baseline / reference leg
may import it; the library under sparse_moe_expert_topk_b200/ never does and
shares no code with it (the only common input is the seeded generator ftgen).

Precision: fp64 throughout, except where floating point decides an integer:
the router logits are rounded once to fp32 before the top-k, because that is
the precision the CUDA path takes the decision in.

Modules
  formats  e2m1 / e4m3 decoding and slot-blob unpacking
  moe      router logits, top-k, softmax weights, permutation, SwiGLU expert,
           per-token layer forward
  cache    q* split and the shared LRU expert cache (hit / staged / streamed);
           the best static placement, for the miss-rate comparison
  cpp      the plain C++ oracle (moe_oracle.cpp, built with the host
           compiler): the layer per token, one std::thread per token, with
           the roundings of the layer's fp32 definition, and the shared LRU
           simulator; pinned against the numpy modules; the CPU baseline
           that bench.py times
  ep       the layer with its experts split among G devices: dispatch plan,
           the all-to-all exchange, owner caches, combine at the source
  ep_compare  expert parallelism against replicas on the same trace: miss
           rates and blobs over each device's host link (python -m oracle.ep_compare)
  policy_compare  the shared LRU against static placements on the 43-layer
           trace (an analysis run of the oracle: python -m oracle.policy_compare)

Parity pins (tests/test_oracle_*.py): every function above is pinned to
something other than itself; see each module's docstring. Expert-value parity
has no printed example on the pages, so the expert math is pinned by a dense
brute-force evaluation, closed-form special cases and library routines.
"""
from . import cache, ep, formats, moe  # noqa: F401
