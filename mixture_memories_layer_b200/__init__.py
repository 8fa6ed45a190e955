"""B200-native Mixture-of-Memories layer: a C-ABI library of sm_100a CUDA
kernels (router, reordering, grouped projections, chunked Gated DeltaNet,
combine, recurrent decode) and a thin Python binding over it.

Importing the package loads nothing; ``mixture_memories_layer_b200.binding``
loads the shared library and fails loudly if it is missing.
"""
__all__ = ["binding", "layer", "synth"]
