"""B200-native fused softmax-weighted average: causal attention (forward and
backward, D = 64) and the Nadaraya-Watson regrid, as hand-written sm_100a
CUDA kernels behind a C ABI (``include/swa.h``).

The binding in ``swa`` loads the in-tree ``libswa.so`` lazily; importing this
package alone does not touch the GPU.
"""
__all__ = ["swa", "inputs"]
