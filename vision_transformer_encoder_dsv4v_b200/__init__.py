"""B200 (sm_100a) forward pass of the DeepSeek-V4-Flash vision tower and aligner.

The compute lives in ``libdsv4v.so`` (hand-written CUDA behind the C ABI of include/dsv4v.h);
``dsv4v`` is the ctypes binding, ``synth`` the seeded input generator, ``build`` the in-tree
nvcc build.
"""
