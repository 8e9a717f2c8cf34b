"""B200-native block-parallel draft step of the H-Spec hybrid Mamba-attention drafter.

Sub-modules:
  hspec   -- ctypes binding of libhspec.so (the C-ABI); importing it fails loudly
             when the CUDA library has not been built.
  inputs  -- seeded synthetic workload generators (shapes and value distributions
             only; none of the method's arithmetic).
  build   -- compiles libhspec.so for sm_100a with nvcc.

Importing the package itself loads nothing native, so the input generators can be
used on machines without a GPU.
"""

__all__ = ["hspec", "inputs", "build"]
__version__ = "0.1.0"
