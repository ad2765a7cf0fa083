"""B200-native sparse-MLA decode step: DSA indexer scores, exact top-k and
absorbed-query sparse MLA over paged FP8 caches (fp8_ds_mla or plain
per-tensor E4M3 latents), plus the producers that quantise new tokens into
those caches and the indexer queries.

The compute lives in ``libsml.so`` (hand-written sm_100a CUDA behind a C ABI
declared in ``include/sml.h``); ``sparse_mla_attention_indexer_b200.sml`` is a
thin ctypes binding with the same entry-point names.  ``synth`` builds seeded
synthetic workloads; ``run_stages`` runs them (or the producers) for profilers.
"""
