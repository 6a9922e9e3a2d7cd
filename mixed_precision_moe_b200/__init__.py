"""B200-native mixed-precision Mixture-of-Experts layer.

The compute path is the C-ABI library ``libmoe.so`` (hand-written CUDA for
sm_100a); ``binding`` marshals torch tensors into its entry points.  Importing
this package does not load the library; the first call into ``binding`` does,
and fails loudly if the library has not been built.
"""
