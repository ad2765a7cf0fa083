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


def visible_lengths(cu_q: np.ndarray, ctx_len: np.ndarray) -> np.ndarray:
    """n_t of every query token under the causal rule (query j of request r
    sees positions [0, L_r - Q_r + j])."""
    cu_q = np.asarray(cu_q, dtype=np.int64)
    out = np.empty(int(cu_q[-1]), dtype=np.int64)
    for r in range(len(cu_q) - 1):
        Q = int(cu_q[r + 1] - cu_q[r])
        out[cu_q[r]:cu_q[r + 1]] = int(ctx_len[r]) - Q + np.arange(Q) + 1
    return out


def rank_arrays(cu_q: np.ndarray, ctx_len: np.ndarray, rank: int, R: int, interleave: int):
    """A rank's per-request local lengths [B] and per-token (local visible
    count, global visible length) [T] (int32): the ctx_len, vis_len and
    ssmax_len of its problem.  Query t's local visible count is the number of
    the rank's tokens among the query's global positions [0, n_t)."""
    n = visible_lengths(cu_q, ctx_len)
    local_len = np.array([rank_length(L, rank, R, interleave) for L in ctx_len], dtype=np.int32)
    vis = np.array([rank_length(int(x), rank, R, interleave) for x in n], dtype=np.int32)
    return local_len, vis, n.astype(np.int32)


def shard_pages(block_table: np.ndarray, ctx_len: np.ndarray, rank: int, R: int, interleave: int) -> np.ndarray:
    """A rank's local block table [B, width]: the pages of each request it
    holds, in order (a request it holds no token of has an empty row)."""
    tables = [np.asarray(block_table[b])[rank_pages(L, rank, R, interleave)] for b, L in enumerate(ctx_len)]
    width = max(1, max(len(x) for x in tables))
    bt = np.zeros((len(tables), width), dtype=np.int32)
    for b, x in enumerate(tables):
        bt[b, :len(x)] = x
    return bt


def _all_gather(t, group=None):
    """Every rank's copy of t (same shape on every rank), in rank order.  NCCL
    moves device tensors directly; other backends (gloo) through host memory."""
    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group)
    if dist.get_backend(group) == "nccl":
        out = [torch.empty_like(t) for _ in range(world)]
        dist.all_gather(out, t.contiguous(), group=group)
        return out
    h = t.detach().cpu().contiguous()
    out = [torch.empty_like(h) for _ in range(world)]
    dist.all_gather(out, h, group=group)
    return [x.to(t.device) for x in out]


def dcp_layer(problem, q, iq8, iq_scale, iw, latent, index_cache, *, rank: int, world: int, interleave: int,
              group=None, stream=None):
    """One sparse-attention layer with the cache sharded by token over the
    ranks of `group`, each rank holding its shard (its `problem` from
    rank_arrays / shard_pages).  The steps of the blog's DCP decode: the
    rank's own indexer and top-k; its candidates packed as (score, position)
    and exchanged (all-gather); the stable merge and the global top-k, the
    same on every rank; the selection split back to the rank's own tokens;
    its sparse MLA over them; the partial (out, lse) exchanged and combined by
    their LSE.  Every step runs in libsml.so; this function only moves arrays.
    Returns (idx of this rank's selected local positions, their count,
    out [T, H, 512], lse [T, H]) -- out and lse the same on every rank."""
    import torch
    from . import sml
    dev = q.device
    T, H, K = problem.num_tokens, problem.num_heads, problem.topk
    ws = torch.empty(sml.sml_workspace_size(problem, sml.SML_STAGE_LAYER), dtype=torch.uint8, device=dev)
    sml.sml_workspace_init(ws, stream)
    scores = torch.empty(T, problem.max_ctx, dtype=torch.float32, device=dev)
    idx = torch.empty(T, K, dtype=torch.int32, device=dev)
    ln = torch.empty(T, dtype=torch.int32, device=dev)
    sml.sml_indexer_scores(problem, iq8, iq_scale, iw, index_cache, scores, ws, stream)
    sml.sml_topk(problem, scores, idx, ln, ws, stream)
    cand = torch.empty(T, K, dtype=torch.float32, device=dev)
    sml.sml_dcp_pack_candidates(scores, idx, ln, cand, ws, stream)
    cands, idxs, lens = _all_gather(cand, group), _all_gather(idx, group), _all_gather(ln, group)
    m_scores = torch.empty(T, world * K, dtype=torch.float32, device=dev)
    m_pos = torch.empty(T, world * K, dtype=torch.int32, device=dev)
    m_len = torch.empty(T, dtype=torch.int32, device=dev)
    sml.sml_dcp_merge_candidates(cands, idxs, lens, interleave, K, m_scores, m_pos, m_len, ws, stream, packed=True)
    # the global top-k over each query's merged row: T one-token requests
    cu = torch.arange(T + 1, dtype=torch.int32, device=dev)
    bt = torch.zeros(T, (world * K + 63) // 64, dtype=torch.int32, device=dev)
    pm = sml.make_problem(num_heads=H, topk=K, rope_dim=problem.rope_dim, cu_q=cu, ctx_len=m_len, block_table=bt,
                          max_ctx=world * K, sm_scale=problem.sm_scale, num_tokens=T)
    ws_m = torch.empty(sml.sml_workspace_size(pm, sml.SML_STAGE_TOPK), dtype=torch.uint8, device=dev)
    sml.sml_workspace_init(ws_m, stream)
    sel = torch.empty(T, K, dtype=torch.int32, device=dev)
    sel_len = torch.empty(T, dtype=torch.int32, device=dev)
    sml.sml_topk(pm, m_scores, sel, sel_len, ws_m, stream)
    local_idx = [torch.empty(T, K, dtype=torch.int32, device=dev) for _ in range(world)]
    local_len = [torch.empty(T, dtype=torch.int32, device=dev) for _ in range(world)]
    sml.sml_dcp_split_selection(interleave, K, sel, sel_len, m_pos, local_idx, local_len, ws, stream)
    out = torch.empty(T, H, 512, dtype=torch.float32, device=dev)
    lse = torch.empty(T, H, dtype=torch.float32, device=dev)
    sml.sml_sparse_mla_decode(problem, q, latent, local_idx[rank], local_len[rank], out, lse, ws, stream)
    outs, lses = _all_gather(out, group), _all_gather(lse, group)
    out_c = torch.empty_like(out)
    lse_c = torch.empty_like(lse)
    sml.sml_lse_combine(outs, lses, out_c, lse_c, stream)
    for w in (ws, ws_m):
        code, bits = sml.sml_read_device_status(w, stream=stream)
        if code != sml.SML_OK:
            raise sml.SmlError(code, f"device status bits {bits:#x}")
    return local_idx[rank], local_len[rank], out_c, lse_c
