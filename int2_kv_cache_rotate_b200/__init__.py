"""B200-native INT2 KV cache with attention-aware rotations (OSCAR-style).

The compute path is the C-ABI library ``libokv.so`` built from ``csrc/``;
``okv`` is its thin ctypes binding.  Importing the package does not load the
library; the first call through ``okv`` does, and fails loudly if it is
missing.
"""
