"""Plain float64 CPU oracle for the sparse-MLA decode step (indexer -> top-k ->
sparse MLA -> LSE merge).

TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only ``tests/``,
``__graft_entry__.smoke()`` and the CPU-baseline / reference legs of
``bench.py`` may import this package.  It shares no code, header, table or
constant with the CUDA library and never calls it; both sides take their
inputs from the seeded generator in ``sparse_mla_attention_indexer_b200.synth``,
which holds no arithmetic of the method.

Modules:
  formats -- E4M3 / bf16 decoding and the paged cache byte layouts
  dsa     -- indexer scores, visible lengths, exact top-k
  mla     -- absorbed-query attention, sparse and dense MLA, LSE merge, one layer
  producers -- FP8 quantisation and the cache writes just before the step
  dcp     -- the step with the cache sharded by token over ranks (decode
             context parallelism): candidates, stable merge, LSE combine

Every function is pinned by tests under ``tests/`` (``-m "not gpu"``) to
values the pages print, closed forms, invariants, library routines and brute
force on tiny inputs; none is "parity unpinned".
"""
from . import dcp, dsa, formats, mla, producers  # noqa: F401
