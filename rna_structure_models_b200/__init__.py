"""B200-native fused Invariant Point Attention (FlashIPA core) and the
geometric direction/distance attention variant.

The compute path is a C-ABI CUDA library (`libflashipa_b200.so`, built for
sm_100a).  Importing this package does not load it; the first call into
`rna_structure_models_b200.api` does, and raises if it is missing.
"""
__all__ = ["api", "synth"]
