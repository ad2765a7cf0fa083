"""Host-side sharding for decode context parallelism (DCP): which pages of a
request's block table a rank holds, and its local lengths.

Token s of a request lives on rank (s // I) % R at local position
(s // (I R)) I + s % I (the convention of ``sml_dcp_merge_candidates`` and
``sml_dcp_split_selection``).  With I a multiple of the 64-token page a rank's
shard is a list of whole pages of the same pool, so a rank's problem is the
batch with a local block table and local lengths; no cache data moves.  Plain
integer bookkeeping on host arrays: no step of the computation runs here.
"""
from __future__ import annotations

import numpy as np

PAGE = 64


def rank_pages(length: int, rank: int, R: int, interleave: int) -> np.ndarray:
    """Logical pages (in order) of a request of `length` tokens held by `rank`."""
    if interleave % PAGE:
        raise ValueError("interleave must be a multiple of the 64-token page")
    npages = (int(length) + PAGE - 1) // PAGE
    j = np.arange(npages)
    return j[((j * PAGE) // interleave) % R == rank]


def rank_length(length: int, rank: int, R: int, interleave: int) -> int:
    """Tokens of a request of `length` tokens held by `rank`."""
    full, rest = divmod(int(length), interleave * R)
    return full * interleave + min(max(rest - rank * interleave, 0), interleave)


def shard(block_table: np.ndarray, ctx_len: np.ndarray, rank: int, R: int, interleave: int):
    """One rank's (local block table [B, width], local lengths [B]) from the
    batch's block table [B, max_pages] and lengths [B].  Raises if the rank
    would hold no token of some request (its problem would have an empty
    request)."""
    tables = [np.asarray(block_table[b])[rank_pages(L, rank, R, interleave)] for b, L in enumerate(ctx_len)]
    lens = np.array([rank_length(L, rank, R, interleave) for L in ctx_len], dtype=np.int32)
    if np.any(lens < 1):
        raise ValueError("every rank must hold at least one token of every request "
                         "(length > (R - 1) * interleave)")
    width = max(1, max(len(x) for x in tables))
    bt = np.zeros((len(tables), width), dtype=np.int32)
    for b, x in enumerate(tables):
        bt[b, :len(x)] = x
    return bt, lens


def global_position(local: np.ndarray, rank: int, R: int, interleave: int) -> np.ndarray:
    """Global positions of a rank's local positions."""
    local = np.asarray(local, dtype=np.int64)
    return ((local // interleave) * R + rank) * interleave + local % interleave
