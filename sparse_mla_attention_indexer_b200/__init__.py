"""B200-native sparse-MLA decode step: DSA indexer scores, exact top-k and
absorbed-query sparse MLA over paged FP8 caches.

The compute lives in ``libsml.so`` (hand-written sm_100a CUDA behind a C ABI
declared in ``include/sml.h``); ``sparse_mla_attention_indexer_b200.sml`` is a
thin ctypes binding with the same entry-point names.  ``synth`` builds seeded
synthetic workloads.
"""
