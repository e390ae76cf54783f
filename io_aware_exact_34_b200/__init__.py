"""libfattn: exact, IO-aware tiled attention for B200 (sm_100a).

The compute path is the C-ABI library ``libfattn.so`` (CUDA kernels for
sm_100a); ``io_aware_exact_34_b200.fattn`` is its Python binding.  Import the
binding explicitly: it fails loudly when the library has not been built.
"""
