"""DSA indexer scores and exact top-k selection, in float64.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

What the pages fix (vLLM blog "vLLM 首日支持 Mistral Large 4", highlights list
and section "实现细节 / 模型架构", paragraph "稀疏 MLA + DSA indexer"):

* a DSA sparse indexer picks the top 2048 keys for every query, from an FP8
  indexer cache; the indexer has its own SSMax; NoPE layers use a NoPE indexer;
* the selection is exact ("精确的 top-2048", ROCm section "专用解码");
* shared-indexer layers reuse the top-k of the nearest preceding indexer layer.

The pages print no formula for the score.  The reading taken here is the
DeepSeek-style indexer named by the task: per indexer head h an FP8 dot product
q_{t,h} . k_s, a ReLU, and a weighted sum over heads with per-token head weights:

    I[t, s] = c_t * sum_h w[t, h] * ReLU(q_{t,h} . k_s),   s < n_t

with q_{t,h} = sq_t * e4m3(q8[t, h, :]), k_s = sk_s * e4m3(k8[s, :]) and
c_t = s_index * ln(n_t) when SSMax is on, else 1.  n_t is the visible length of
query token t: query j (0-based) of request r, which has Q_r query tokens and
L_r cached tokens (its own query tokens included), sees positions
[0, L_r - Q_r + j], so n_t = L_r - Q_r + j + 1.

Top-k: the K largest scores of I[t, 0:n_t]; ties go to the lower token index;
-0.0 equals +0.0; a NaN ranks below every number.  The result is returned as the
set of selected positions in ascending order, min(K, n_t) of them.
"""
from __future__ import annotations

import math

import numpy as np

from . import formats as F


def request_of_tokens(cu_q: np.ndarray) -> np.ndarray:
    """Request index of every query token, from the query offsets cu_q [B+1]."""
    B = len(cu_q) - 1
    out = np.empty(int(cu_q[-1]), dtype=np.int64)
    for r in range(B):
        out[cu_q[r]:cu_q[r + 1]] = r
    return out


def visible_lengths(cu_q: np.ndarray, ctx_len: np.ndarray) -> np.ndarray:
    """n_t for every query token t (causal within the request)."""
    req = request_of_tokens(cu_q)
    t = np.arange(len(req))
    j = t - np.asarray(cu_q)[req]
    q_count = np.diff(cu_q)[req]
    return np.asarray(ctx_len, dtype=np.int64)[req] - q_count + j + 1


def ssmax_factor(enabled: bool, s: float, n: int) -> float:
    """SSMax multiplier s * ln(n) on the logits, or 1 when SSMax is off."""
    return s * math.log(n) if enabled else 1.0


def indexer_scores_row(q8_t, q_scale_t, w_t, index_cache, bt_row, n, c_t, positions=None,
                       with_magnitude=False):
    """Scores of one query token against positions (default: all of 0..n-1).

    q8_t: [64, 128] uint8 e4m3 codes; q_scale_t: scalar; w_t: [64] head weights.
    With ``with_magnitude`` also returns the size of the summed terms,
    c_t * sum_h |w_h| * ReLU(q_h . k_s), against which a rounding error in the
    weighted sum is measured.
    """
    if positions is None:
        positions = np.arange(n)
    positions = np.asarray(positions, dtype=np.int64)
    q = F.decode_e4m3(q8_t) * float(q_scale_t)                     # [64, 128]
    w = np.asarray(w_t, dtype=np.float64)                          # [64]
    out = np.empty(len(positions), dtype=np.float64)
    mag = np.empty(len(positions), dtype=np.float64)
    chunk = 1 << 15
    for a in range(0, len(positions), chunk):
        pos = positions[a:a + chunk]
        pages, rows = F.physical(bt_row, pos)
        k = F.indexer_keys(index_cache, pages, rows)                # [m, 128]
        relu = np.maximum(q @ k.T, 0.0)                             # [64, m]
        out[a:a + chunk] = c_t * (w[:, None] * relu).sum(axis=0)
        if with_magnitude:
            mag[a:a + chunk] = abs(c_t) * (np.abs(w)[:, None] * relu).sum(axis=0)
    return (out, mag) if with_magnitude else out


def indexer_scores(wl, q8, q_scale, w, index_cache, tokens=None):
    """Score rows for the query tokens in ``tokens`` (default: all).

    ``wl`` carries cu_q, ctx_len, block_table, ssmax, ssmax_s_index.
    Returns a list of float64 arrays, row t of length n_t.
    """
    req = request_of_tokens(wl.cu_q)
    n_all = visible_lengths(wl.cu_q, wl.ctx_len)
    if tokens is None:
        tokens = range(len(req))
    rows = []
    for t in tokens:
        n = int(n_all[t])
        c = ssmax_factor(wl.ssmax, wl.ssmax_s_index, n)
        rows.append(indexer_scores_row(q8[t], q_scale[t], w[t], index_cache,
                                       wl.block_table[req[t]], n, c))
    return rows


def topk_row(scores: np.ndarray, k: int) -> np.ndarray:
    """Exact top-k of one score row; ties to the lower index; ascending positions."""
    s = np.asarray(scores, dtype=np.float64)
    n = len(s)
    # numpy orders NaN after every number, so a NaN score (negated: still NaN)
    # ranks below -inf; -0.0 and +0.0 compare equal, so the index decides.
    order = np.lexsort((np.arange(n), -s))
    return np.sort(order[:min(k, n)]).astype(np.int64)
