"""B200-native DDTree tree-verify step: tree build, MLA-absorb verify
attention, greedy accept + latent-KV compaction, behind a C-ABI library
(libddt.so). The Python layer only marshals arguments; every step of the path
runs in the library's CUDA kernels.

Submodules: ``lib`` (ctypes binding of libddt.so), ``synth`` (seeded synthetic
inputs), ``build`` (compiles libddt.so in-tree for sm_100a).
"""
