"""deterministic_invariant_routing_b200: a batch-invariant top-k MoE FFN forward pass
for B200 (sm_100a), as a C-ABI library of hand-written CUDA kernels (libmoe_b200.so,
include/moe.h) with a thin torch binding.

    from deterministic_invariant_routing_b200 import moe
    out = moe.forward(moe.Config(T, H, E, K, I), x, w_router, w13, w2)

Submodules: ``moe`` (the binding), ``build`` (nvcc build of the library), ``synthetic``
(seeded inputs for tests and benchmarks). Importing the package loads nothing; the first
binding call loads the library and raises if it is not built.
"""
__all__ = ["moe", "build", "synthetic"]
__version__ = "0.1.0"
