"""B200-native (sm_100a) tree-verify step for DDTree speculative decoding with MLA.

Submodules:
  kd        -- ctypes binding of the C-ABI library libkdverify.so (the CUDA path)
  workload  -- seeded synthetic inputs (no method arithmetic)
  build     -- nvcc build of the library for sm_100a

Importing the package loads nothing; ``from tree_speculative_decoding_kd_b200 import kd``
loads the CUDA library and raises if it is missing.
"""
