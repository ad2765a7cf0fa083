"""Absorbed-query sparse MLA over a paged fp8_ds_mla latent cache, in float64.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

What the pages fix (vLLM blog "vLLM 首日支持 Mistral Large 4"):

* highlights list: MLA with KV LoRA rank 512 and RoPE dim 64; each query
  attends to the top 2048 keys picked by the DSA indexer;
* section "实现细节 / 模型架构": sparse MLA runs over the fp8_ds_mla latent
  cache; NoPE layers are MLA with RoPE dim 0 and use the same kernels and cache
  layout; SSMax scales the MLA query; shared-indexer layers reuse the top-k of
  the preceding indexer layer;
* section "长上下文" (DCP): partial attention results are combined through
  their log-sum-exp (LSE), which is the merge written out in ``lse_merge``.

Absorbed MLA: the query arrives already multiplied into the latent space, so a
key is the 576-d row [c_hat (512) | k_pe (64)] and the value is c_hat itself.
For query token t, head h and a selected set S of positions:

    z_i = sigma * c_t * (q_nope[t,h] . c_hat_i + q_pe[t,h] . k_pe_i),  i in S
    out[t,h] = sum_i softmax(z)_i * c_hat_i,   lse[t,h] = ln sum_i exp(z_i)

sigma is the softmax scale, c_t = s * ln(n_t) with SSMax on (n_t = visible
length of token t), else 1.  A NoPE layer drops the q_pe . k_pe term (RoPE dim
0) and its query is 512-d.  An empty set gives out = 0 and lse = -inf.
"""
from __future__ import annotations

import numpy as np

from . import formats as F
from .dsa import (indexer_scores_row, request_of_tokens, ssmax_factor, topk_row,
                  visible_lengths)


def attend(q: np.ndarray, c_hat: np.ndarray, k_pe: np.ndarray, rope_dim: int, scale: float):
    """Softmax attention of q [H, 512 + rope_dim] over the given latent rows.

    ``scale`` = sigma * c_t.  Returns (out [H, 512], lse [H]).
    """
    H = q.shape[0]
    if c_hat.shape[0] == 0:
        return np.zeros((H, F.LATENT_DIM)), np.full(H, -np.inf)
    z = q[:, :F.LATENT_DIM] @ c_hat.T
    if rope_dim:
        z = z + q[:, F.LATENT_DIM:F.LATENT_DIM + rope_dim] @ k_pe.T
    z = scale * z                                                   # [H, m]
    zmax = z.max(axis=1, keepdims=True)
    e = np.exp(z - zmax)
    den = e.sum(axis=1)
    out = (e @ c_hat) / den[:, None]
    lse = zmax[:, 0] + np.log(den)
    return out, lse


def token_attention(wl, latent, t, positions):
    """Attention of query token t over the given logical positions of its request.

    ``wl`` carries the batch (cu_q, ctx_len, block_table), the layer's query
    ``q`` (bf16 bits [T, H, 512 + rope_dim]), rope_dim, sm_scale and SSMax.
    """
    req = request_of_tokens(wl.cu_q)[t]
    n = int(visible_lengths(wl.cu_q, wl.ctx_len)[t])
    q = F.decode_bf16(wl.q[t])                                      # [H, 512+rope]
    pages, rows = F.physical(wl.block_table[req], positions)
    c_hat, k_pe = F.latent_rows(latent, pages, rows)
    scale = wl.sm_scale * ssmax_factor(wl.ssmax, wl.ssmax_s, n)
    return attend(q, c_hat, k_pe, wl.rope_dim, scale)


def sparse_mla(wl, latent, idx, idx_len, tokens=None):
    """Sparse MLA for each token over its selected positions idx[t, :idx_len[t]].

    Returns (out [len(tokens), H, 512], lse [len(tokens), H]).
    """
    T = int(wl.cu_q[-1])
    tokens = range(T) if tokens is None else list(tokens)
    outs, lses = [], []
    for t in tokens:
        pos = np.asarray(idx[t][:int(idx_len[t])], dtype=np.int64)
        o, l = token_attention(wl, latent, t, pos)
        outs.append(o)
        lses.append(l)
    return np.stack(outs), np.stack(lses)


def dense_mla(wl, latent, tokens=None):
    """Plain (dense) MLA of each token over every visible position 0..n_t-1."""
    T = int(wl.cu_q[-1])
    tokens = range(T) if tokens is None else list(tokens)
    n_all = visible_lengths(wl.cu_q, wl.ctx_len)
    outs, lses = [], []
    for t in tokens:
        o, l = token_attention(wl, latent, t, np.arange(int(n_all[t])))
        outs.append(o)
        lses.append(l)
    return np.stack(outs), np.stack(lses)


def lse_merge(partial_out: np.ndarray, partial_lse: np.ndarray):
    """Combine attention over disjoint key sets from each set's (out, lse).

    partial_out [S, ..., 512] is each set's own normalised output, partial_lse
    [S, ...] its log-sum-exp; an empty set has lse = -inf and drops out.
    """
    m = partial_lse.max(axis=0)
    safe_m = np.where(np.isfinite(m), m, 0.0)
    wts = np.exp(partial_lse - safe_m)                              # [S, ...]
    den = wts.sum(axis=0)
    with np.errstate(invalid="ignore", divide="ignore"):
        out = (wts[..., None] * partial_out).sum(axis=0) / den[..., None]
        lse = safe_m + np.log(den)
    out = np.where((den > 0)[..., None], out, 0.0)
    return out, np.where(den > 0, lse, -np.inf)


def run_layer(wl, latent, index_cache, reuse_idx=None, tokens=None):
    """One sparse-attention layer: indexer -> top-k -> sparse MLA.

    ``wl`` holds the batch and the layer: q (bf16 bits), and unless
    ``reuse_idx`` is given (a shared-indexer layer, which skips scoring), iq8,
    iq_scale and iw.  Returns
    (idx list of ascending position arrays, out, lse) for ``tokens``.
    """
    T = int(wl.cu_q[-1])
    tokens = range(T) if tokens is None else list(tokens)
    req = request_of_tokens(wl.cu_q)
    n_all = visible_lengths(wl.cu_q, wl.ctx_len)
    idx_list = []
    for t in tokens:
        if reuse_idx is not None:
            idx_list.append(np.asarray(reuse_idx[t], dtype=np.int64))
            continue
        n = int(n_all[t])
        c = ssmax_factor(wl.ssmax, wl.ssmax_s_index, n)
        row = indexer_scores_row(wl.iq8[t], wl.iq_scale[t], wl.iw[t],
                                 index_cache, wl.block_table[req[t]], n, c)
        idx_list.append(topk_row(row, wl.topk))
    outs, lses = [], []
    for t, pos in zip(tokens, idx_list):
        o, l = token_attention(wl, latent, t, pos)
        outs.append(o)
        lses.append(l)
    return idx_list, np.stack(outs), np.stack(lses)
