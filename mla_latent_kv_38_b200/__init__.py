"""B200-native (sm_100a) MLA decode over a paged latent KV cache.

Submodules:
  binding  -- ctypes binding of libmla_b200.so (the C ABI of include/mla.h)
  build    -- nvcc build of the in-tree shared library
  synth    -- seeded synthetic inputs (SplitMix64 + Box-Muller, bf16)
"""
