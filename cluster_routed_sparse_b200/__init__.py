"""Cluster-routed sparse attention (AdaCluster) for one video-DiT attention
layer on NVIDIA B200 (sm_100a).

The product is libac.so, a C-ABI CUDA library (include/ac.h).  `SparseLayer`
is its thin Python binding over torch tensors; `synth` generates the seeded
synthetic inputs.  Importing the package does not load the library; the first
`SparseLayer` does, and fails loudly if libac.so is missing.
"""

__all__ = ["SparseLayer", "synth"]


def __getattr__(name):
    if name == "SparseLayer":
        from .api import SparseLayer
        return SparseLayer
    raise AttributeError(name)
