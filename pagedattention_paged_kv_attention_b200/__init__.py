"""B200-native paged KV-cache decode attention.

The product is the C-ABI library ``libpagedattn.so`` (hand-written CUDA for sm_100a, declared in
``include/pagedattn.h``); ``pagedattn`` is its thin ctypes binding and ``build`` compiles it in-tree.
Import ``pagedattention_paged_kv_attention_b200.pagedattn`` to use it (the import fails if the
library has not been built; there is no CPU fallback).
"""
