"""kv_cache_bit_b200: B200-native low-bit KV-cache quantization (nsep+pchan,
randomized Hadamard, NSN) and fused decode attention over the packed cache.

The compute path is the C-ABI library ``libkvq.so`` (CUDA, sm_100a) built from
``csrc/``; ``kvq`` is its thin ctypes binding.  Importing the package does not
load the library; ``from kv_cache_bit_b200 import kvq`` does, and fails loudly
when it is missing.
"""
