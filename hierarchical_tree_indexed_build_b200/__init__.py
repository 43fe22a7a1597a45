"""B200-native ZHA tree build and tree-routed sparse decode.

Submodules:
  zha        - ctypes binding of libzha.so (C ABI in include/zha.h) + Tree/Decoder wrappers
  inputs     - seeded synthetic workloads (no method arithmetic)
  build_ext  - nvcc build of libzha.so for sm_100a
Submodules are imported on demand so that importing the package never loads CUDA.
"""
