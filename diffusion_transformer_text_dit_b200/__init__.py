"""B200-native (sm_100a) W8A8 DiT step of Qwen-Image-2.1 behind the libqi C ABI.

Submodules:
  qi         ctypes binding of libqi.so (include/qi.h); loading it needs the built library
  build_lib  in-tree nvcc build of libqi.so for sm_100a
  synth      seeded synthetic workloads (shapes, seeds, distributions only)
Importing the package loads nothing; the CUDA library is loaded on first use.
"""
