"""B200-native MXFP4 block-scaled Mixture-of-Experts expert layer.

The compute path is the C-ABI library ``libmxfp4moe.so`` (hand-written CUDA for
sm_100a) declared in ``include/mxfp4_moe.h``; ``binding`` marshals torch tensors into
it. Importing this package does not load the library; the first call into ``binding``
does, and raises if the library is missing or no GPU is present: there is no CPU path.
"""
__all__ = ["binding", "inputs"]
