"""Sparse MoE FFN forward pass on B200 (sm_100a).

The compute lives in ``libmoe_b200.so`` (hand-written CUDA behind a C ABI,
declared in ``include/moe.h``). ``binding`` marshals arguments to it;
``inputs`` draws the seeded synthetic workloads.
"""
