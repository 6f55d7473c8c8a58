"""B200-native chunk-wise Gated DeltaNet inversion + WY library.

The compute lives in ``libgdn.so`` (CUDA, sm_100a; C ABI in ``include/gdn.h``);
``gated_deltanet_chunk_02_b200.gdn`` is its thin Python binding and
``gated_deltanet_chunk_02_b200.inputs`` the seeded synthetic input generator.
"""
__all__ = ["gdn", "inputs"]
