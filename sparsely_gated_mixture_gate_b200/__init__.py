"""B200-native forward pass of the Sparsely-Gated Mixture-of-Experts layer.

The compute path is the C-ABI library ``libmoe_b200.so`` (CUDA kernels for
sm_100a) declared in ``include/moe.h``; ``moe`` is its thin Python binding
(argument marshalling over torch device memory and streams).  ``synth`` draws
the seeded synthetic inputs.  Nothing is imported eagerly so that the input
generator works on machines without the built library.
"""
__all__ = ["moe", "synth"]
