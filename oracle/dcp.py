"""Decode context parallelism (DCP): the step with the KV cache sharded by
token over R ranks, in float64.

TEST INFRASTRUCTURE ONLY.  This module belongs to the CPU oracle: it may be
imported by ``tests/``, by ``__graft_entry__.smoke()`` and by the CPU-baseline
leg of ``bench.py``, and by nothing else.  It shares no code with the CUDA
library.

Source: vLLM blog "vLLM 首日支持 Mistral Large 4：1T 参数 MoE 多模态模型",
section "长上下文：解码和预填充的上下文并行", paragraph "DCP" and the list after
it: DCP shards the latent cache by token instead of replicating it on every
rank; per decode step each rank's indexer produces top-k candidates, which the
ranks exchange as packed (score, id) pairs and merge with a stable top-k; the
sparse attention of each rank covers the selected tokens it holds (a rank that
holds none of a query's top-k slots has an empty row), and the partial outputs
are combined by their log-sum-exp (an all-to-all LSE combine).

Readings (the blog gives the steps, not their definitions):

* token s of a request lives on rank (s // I) % R for an interleave size I
  (the blog says "by token"; I = 1 is the plainest reading, and I = 64 keeps a
  64-token page on one rank); a rank holds its tokens in ascending order;
* a rank's candidates for query t are the top min(K, m) of its m visible
  tokens by (score descending, position ascending), carried as (score, global
  position);
* the merge takes the top K of all candidates by the same key (the "stable
  top-k merge": ties to the lower global position);
* rank r attends over the selected positions it holds, giving (out_r, lse_r)
  with out_r normalised by its own sum (lse_r = -inf for an empty set); the
  combine is ``mla.lse_merge`` over the ranks.

Every global top-K position is among its own rank's candidates (a key in the
global top K has fewer than K keys of its rank above it), so the merged
selection is exactly the unsharded top K, and the combined attention is the
unsharded sparse MLA over it.
"""
from __future__ import annotations

import numpy as np

from . import dsa, mla


def owner(positions: np.ndarray, R: int, interleave: int) -> np.ndarray:
    """Rank holding each global position."""
    return (np.asarray(positions, dtype=np.int64) // interleave) % R


def rank_candidates(scores: np.ndarray, rank: int, R: int, interleave: int, k: int):
    """One rank's candidates from a query's visible score row: (scores,
    global positions), best first by (score descending, position ascending)."""
    n = scores.shape[0]
    mine = np.nonzero(owner(np.arange(n), R, interleave) == rank)[0]
    local = dsa.topk_row(scores[mine], k)          # local positions, ascending
    pos = mine[local]
    # the order of the oracle's top-k: numpy sorts NaN after every number, so
    # a NaN score ranks below -inf, and -0.0 ties with +0.0
    order = np.lexsort((pos, -np.asarray(scores[pos], dtype=np.float64)))
    return scores[pos][order], pos[order]


def merge_candidates(cand_scores, cand_pos, k: int) -> np.ndarray:
    """Stable top-k merge of all ranks' candidates: the top k by (score
    descending, global position ascending), returned in ascending position."""
    s = np.concatenate(cand_scores).astype(np.float64)
    p = np.concatenate(cand_pos)
    order = np.lexsort((p, -s))
    return np.sort(p[order[:k]])


def select(scores_row: np.ndarray, R: int, interleave: int, k: int) -> np.ndarray:
    """The DCP selection for one query from its visible score row."""
    cs, cp = zip(*(rank_candidates(scores_row, r, R, interleave, k) for r in range(R)))
    return merge_candidates(cs, cp, k)


def attention(wl, latent, t: int, selected: np.ndarray, R: int, interleave: int):
    """Per-rank partial attention over the selected positions each rank holds,
    then the LSE combine.  Returns (out [H, 512], lse [H], per-rank lse [R, H])."""
    own = owner(selected, R, interleave)
    outs, lses = [], []
    for r in range(R):
        o, l = mla.token_attention(wl, latent, t, selected[own == r])
        outs.append(o)
        lses.append(l)
    out, lse = mla.lse_merge(np.stack(outs), np.stack(lses))
    return out, lse, np.stack(lses)
