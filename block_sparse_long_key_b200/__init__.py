"""B200-native MoBA (Mixture of Block Attention) hot path.

The compute lives in the C-ABI CUDA library ``libmoba.so`` built from
``csrc/``; ``moba`` is its thin Python binding.  Importing the package loads
nothing: the library is loaded on first use and a missing library is an
error, never a silent fallback.
"""
