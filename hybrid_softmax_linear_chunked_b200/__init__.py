"""B200-native (sm_100a) ReHyAt chunk-wise recurrent hybrid attention forward.

The compute lives in the CUDA library `librehyat.so` (C ABI declared in include/rehyat.h); the
Python module `binding` only marshals arguments to it.
"""
from . import configs, inputs  # noqa: F401
