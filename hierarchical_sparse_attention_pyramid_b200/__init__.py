"""B200-native Lighthouse attention layer (hierarchical sparse attention pyramid).

The compute path is the CUDA library ``liblh.so`` (C ABI, ``include/lh.h``);
this package only marshals torch tensors into its calls.
"""
