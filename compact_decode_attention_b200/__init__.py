"""compact_decode_attention_b200: compact-KV decode for Dynamic Memory
Sparsification on NVIDIA B200 (sm_100a).

The work is done by the CUDA library ``libdms.so`` (C ABI in
``include/dms.h``); ``compact_decode_attention_b200.dms`` is its ctypes
binding.  Importing the package loads nothing; build the library with
``python -m compact_decode_attention_b200.build``.
"""
