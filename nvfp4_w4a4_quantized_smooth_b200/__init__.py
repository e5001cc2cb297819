"""SVDQuant W4A4 NVFP4 linear layer for B200 (sm_100a).

The compute path lives in the C-ABI library ``libsvdq.so`` (hand-written
CUDA kernels, built in-tree by ``build.py``); ``svdq`` is its thin ctypes
binding and ``synth`` draws seeded synthetic operands.
"""
