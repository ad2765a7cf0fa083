"""Decode context parallelism on one GPU: R ranks as page-interleaved shards of
the same pools (a rank's shard is a local block table).  Each rank runs the
indexer and top-k over its own tokens; the merge, the selection over the merged
candidates, the split and the LSE combine follow.  The selection must equal the
unsharded top-k bit for bit (a key's score does not depend on the tile it lands
in), and the combined attention must match the oracle."""
import numpy as np
import pytest
import torch

from sparse_mla_attention_indexer_b200 import sml, synth
from sparse_mla_attention_indexer_b200.device import DeviceWorkload
from oracle import dcp as odcp
from tests import parity

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from sparse_mla_attention_indexer_b200 import build
    build.build()
    sml.lib()


def shard(wl, R, I):
    """Per rank: (local block table [B, pages], local lengths [B]) of the page-
    interleaved shard (I a multiple of 64: token s on rank (s // I) % R)."""
    out = []
    for r in range(R):
        tables, lens = [], []
        for b in range(wl.B):
            L = int(wl.ctx_len[b])
            npages = (L + 63) // 64
            mine = [j for j in range(npages) if (j * 64 // I) % R == r]
            tables.append([int(wl.block_table[b, j]) for j in mine])
            s = np.arange(L)
            lens.append(int(np.sum((s // I) % R == r)))
        width = max(1, max(len(x) for x in tables))
        bt = np.zeros((wl.B, width), dtype=np.int32)
        for b, x in enumerate(tables):
            bt[b, :len(x)] = x
        out.append((bt, np.array(lens, dtype=np.int32)))
    return out


def run_dcp(dw, wl, R, I):
    lay = dw.layers[0]
    T, K, H = wl.T, wl.topk, wl.num_heads
    ranks = []
    for bt, lens in shard(wl, R, I):
        d_bt, d_len = torch.from_numpy(bt).to(DEV), torch.from_numpy(lens).to(DEV)
        p = sml.make_problem(num_heads=H, topk=K, rope_dim=lay.rope_dim, cu_q=dw.cu_q, ctx_len=d_len,
                             block_table=d_bt, max_ctx=int(lens.max()), sm_scale=wl.sm_scale, num_tokens=T)
        ws = torch.empty(sml.sml_workspace_size(p, sml.SML_STAGE_LAYER), dtype=torch.uint8, device=DEV)
        sml.sml_workspace_init(ws)
        scores = torch.empty(T, int(lens.max()), dtype=torch.float32, device=DEV)
        idx = torch.empty(T, K, dtype=torch.int32, device=DEV)
        ln = torch.empty(T, dtype=torch.int32, device=DEV)
        sml.sml_indexer_scores(p, lay.iq8, lay.iq_scale, lay.iw, dw.index_cache, scores, ws)
        sml.sml_topk(p, scores, idx, ln, ws)
        ranks.append(dict(p=p, ws=ws, scores=scores, idx=idx, len=ln, keep=(d_bt, d_len)))
    ws = torch.empty(256, dtype=torch.uint8, device=DEV)
    sml.sml_workspace_init(ws)
    m_scores = torch.empty(T, R * K, dtype=torch.float32, device=DEV)
    m_pos = torch.empty(T, R * K, dtype=torch.int32, device=DEV)
    m_len = torch.empty(T, dtype=torch.int32, device=DEV)
    sml.sml_dcp_merge_candidates([x["scores"] for x in ranks], [x["idx"] for x in ranks],
                                 [x["len"] for x in ranks], I, K, m_scores, m_pos, m_len, ws)
    # the selection over the merged candidates: T requests of one token each
    cu = torch.arange(T + 1, dtype=torch.int32, device=DEV)
    dummy_bt = torch.zeros(T, (R * K + 63) // 64, dtype=torch.int32, device=DEV)
    pm = sml.make_problem(num_heads=H, topk=K, rope_dim=lay.rope_dim, cu_q=cu, ctx_len=m_len, block_table=dummy_bt,
                          max_ctx=R * K, sm_scale=wl.sm_scale, num_tokens=T)
    ws_m = torch.empty(sml.sml_workspace_size(pm, sml.SML_STAGE_TOPK), dtype=torch.uint8, device=DEV)
    sml.sml_workspace_init(ws_m)
    sel = torch.empty(T, K, dtype=torch.int32, device=DEV)
    sel_len = torch.empty(T, dtype=torch.int32, device=DEV)
    sml.sml_topk(pm, m_scores, sel, sel_len, ws_m)
    local_idx = [torch.empty(T, K, dtype=torch.int32, device=DEV) for _ in range(R)]
    local_len = [torch.empty(T, dtype=torch.int32, device=DEV) for _ in range(R)]
    sml.sml_dcp_split_selection(I, K, sel, sel_len, m_pos, local_idx, local_len, ws)
    outs, lses = [], []
    for r, x in enumerate(ranks):
        o = torch.empty(T, H, 512, dtype=torch.float32, device=DEV)
        l = torch.empty(T, H, dtype=torch.float32, device=DEV)
        sml.sml_sparse_mla_decode(x["p"], lay.q, dw.latent, local_idx[r], local_len[r], o, l, x["ws"])
        outs.append(o)
        lses.append(l)
    out = torch.empty(T, H, 512, dtype=torch.float32, device=DEV)
    lse = torch.empty(T, H, dtype=torch.float32, device=DEV)
    sml.sml_lse_combine(outs, lses, out, lse)
    for x in ranks + [dict(ws=ws), dict(ws=ws_m)]:
        code, bits = sml.sml_read_device_status(x["ws"])
        assert code == sml.SML_OK, f"device status {code} bits {bits:#x}"
    sel_h, sel_len_h, pos_h = sel.cpu().numpy(), sel_len.cpu().numpy(), m_pos.cpu().numpy()
    gsel = np.full((T, K), -1, dtype=np.int64)
    for t in range(T):
        gsel[t, :sel_len_h[t]] = pos_h[t, sel_h[t, :sel_len_h[t]]]
    return dict(sel=gsel, sel_len=sel_len_h, out=out.cpu().numpy(), lse=lse.cpu().numpy(),
                local_len=np.stack([x.cpu().numpy() for x in local_len]),
                rank_scores=[x["scores"].cpu().numpy() for x in ranks])


def global_rows(wl, rank_scores, R, I):
    """Each query's visible score row in global positions, assembled from the
    ranks' own score rows (token s of a request is local position
    (s // (I R)) I + s % I on rank (s // I) % R)."""
    n_all = parity.dsa.visible_lengths(wl.cu_q, wl.ctx_len)
    rows = []
    for t in range(wl.T):
        s = np.arange(int(n_all[t]))
        rank = (s // I) % R
        local = (s // (I * R)) * I + s % I
        row = np.empty(len(s), dtype=np.float32)
        for r in range(R):
            m = rank == r
            row[m] = rank_scores[r][t, local[m]]
        rows.append(row)
    return rows


@pytest.mark.parametrize("R,I,K", [(2, 64, 2048), (4, 64, 2048), (8, 128, 2048), (3, 64, 128)])
def test_dcp_equals_the_unsharded_step(R, I, K):
    wl = synth.make_workload(f"dcp{R}_{I}_{K}", [9000, 20000, 1100, 4097, 1537], [1] * 5, 16, topk=K)
    dw = DeviceWorkload(wl)
    # the unsharded step on the same GPU
    p = dw.problem(0)
    lay = dw.layers[0]
    ws = dw.workspace()
    idx, ln, out, lse = dw.outputs()
    scores = dw.scores()
    sml.sml_indexer_scores(p, lay.iq8, lay.iq_scale, lay.iw, dw.index_cache, scores, ws)
    sml.sml_topk(p, scores, idx, ln, ws)
    assert sml.sml_read_device_status(ws)[0] == sml.SML_OK
    ref_idx, ref_len = idx.cpu().numpy(), ln.cpu().numpy()
    parity.check_topk(wl, scores.cpu().numpy(), ref_idx, ref_len)
    got = run_dcp(dw, wl, R, I)
    # the oracle's DCP selection (per-rank candidates, stable merge) over the
    # ranks' own score rows
    for t, row in enumerate(global_rows(wl, got["rank_scores"], R, I)):
        want = odcp.select(row, R, I, K)
        assert got["sel_len"][t] == len(want), f"token {t}: len"
        assert np.array_equal(got["sel"][t, :len(want)], want), f"token {t}: selection differs from the oracle"
    # and the unsharded step's selection
    assert np.array_equal(got["sel_len"], ref_len)
    for t in range(wl.T):
        assert np.array_equal(got["sel"][t, :ref_len[t]], ref_idx[t, :ref_len[t]]), f"token {t}"
    assert np.array_equal(got["local_len"].sum(axis=0), ref_len)
    parity.check_attention(wl, 0, ref_idx, ref_len, got["out"], got["lse"])


def run_dcp_packed(dw, wl, R, I):
    """The DCP step as the cross-GPU path runs it, ranks simulated as shards
    on one GPU: per rank a problem with local lengths, local visible counts
    (vis_len) and the global SSMax length (ssmax_len); candidates packed as
    (score, position); the packed merge; the selection; the split; per-rank
    attention; the LSE combine."""
    from sparse_mla_attention_indexer_b200 import dcp
    lay = dw.layers[0]
    T, K, H = wl.T, wl.topk, wl.num_heads
    ranks = []
    for r in range(R):
        local_len, vis, glob = dcp.rank_arrays(wl.cu_q, wl.ctx_len, r, R, I)
        bt = dcp.shard_pages(wl.block_table, wl.ctx_len, r, R, I)
        keep = [torch.from_numpy(a).to(DEV) for a in (bt, local_len, vis, glob)]
        p = sml.make_problem(num_heads=H, topk=K, rope_dim=lay.rope_dim, cu_q=dw.cu_q, ctx_len=keep[1],
                             block_table=keep[0], max_ctx=max(1, int(local_len.max())), ssmax=wl.ssmax,
                             sm_scale=wl.sm_scale, ssmax_s=wl.ssmax_s, ssmax_s_index=wl.ssmax_s_index,
                             num_tokens=T, vis_len=keep[2], ssmax_len=keep[3])
        ws = torch.empty(sml.sml_workspace_size(p, sml.SML_STAGE_LAYER), dtype=torch.uint8, device=DEV)
        sml.sml_workspace_init(ws)
        scores = torch.empty(T, p.max_ctx, dtype=torch.float32, device=DEV)
        idx = torch.empty(T, K, dtype=torch.int32, device=DEV)
        ln = torch.empty(T, dtype=torch.int32, device=DEV)
        sml.sml_indexer_scores(p, lay.iq8, lay.iq_scale, lay.iw, dw.index_cache, scores, ws)
        sml.sml_topk(p, scores, idx, ln, ws)
        cand = torch.empty(T, K, dtype=torch.float32, device=DEV)
        sml.sml_dcp_pack_candidates(scores, idx, ln, cand, ws)
        ranks.append(dict(p=p, ws=ws, scores=scores, idx=idx, len=ln, cand=cand, vis=vis, keep=keep))
    ws = torch.empty(256, dtype=torch.uint8, device=DEV)
    sml.sml_workspace_init(ws)
    m_scores = torch.empty(T, R * K, dtype=torch.float32, device=DEV)
    m_pos = torch.empty(T, R * K, dtype=torch.int32, device=DEV)
    m_len = torch.empty(T, dtype=torch.int32, device=DEV)
    sml.sml_dcp_merge_candidates([x["cand"] for x in ranks], [x["idx"] for x in ranks], [x["len"] for x in ranks],
                                 I, K, m_scores, m_pos, m_len, ws, packed=True)
    cu = torch.arange(T + 1, dtype=torch.int32, device=DEV)
    dummy_bt = torch.zeros(T, (R * K + 63) // 64, dtype=torch.int32, device=DEV)
    pm = sml.make_problem(num_heads=H, topk=K, rope_dim=lay.rope_dim, cu_q=cu, ctx_len=m_len, block_table=dummy_bt,
                          max_ctx=R * K, sm_scale=wl.sm_scale, num_tokens=T)
    ws_m = torch.empty(sml.sml_workspace_size(pm, sml.SML_STAGE_TOPK), dtype=torch.uint8, device=DEV)
    sml.sml_workspace_init(ws_m)
    sel = torch.empty(T, K, dtype=torch.int32, device=DEV)
    sel_len = torch.empty(T, dtype=torch.int32, device=DEV)
    sml.sml_topk(pm, m_scores, sel, sel_len, ws_m)
    local_idx = [torch.empty(T, K, dtype=torch.int32, device=DEV) for _ in range(R)]
    local_len = [torch.empty(T, dtype=torch.int32, device=DEV) for _ in range(R)]
    sml.sml_dcp_split_selection(I, K, sel, sel_len, m_pos, local_idx, local_len, ws)
    outs, lses = [], []
    for r, x in enumerate(ranks):
        o = torch.empty(T, H, 512, dtype=torch.float32, device=DEV)
        l = torch.empty(T, H, dtype=torch.float32, device=DEV)
        sml.sml_sparse_mla_decode(x["p"], lay.q, dw.latent, local_idx[r], local_len[r], o, l, x["ws"])
        outs.append(o)
        lses.append(l)
    out = torch.empty(T, H, 512, dtype=torch.float32, device=DEV)
    lse = torch.empty(T, H, dtype=torch.float32, device=DEV)
    sml.sml_lse_combine(outs, lses, out, lse)
    for x in ranks + [dict(ws=ws), dict(ws=ws_m)]:
        code, bits = sml.sml_read_device_status(x["ws"])
        assert code == sml.SML_OK, f"device status {code} bits {bits:#x}"
    sel_h, sel_len_h, pos_h = sel.cpu().numpy(), sel_len.cpu().numpy(), m_pos.cpu().numpy()
    gsel = np.full((T, K), -1, dtype=np.int64)
    for t in range(T):
        gsel[t, :sel_len_h[t]] = pos_h[t, sel_h[t, :sel_len_h[t]]]
    return dict(sel=gsel, sel_len=sel_len_h, out=out.cpu().numpy(), lse=lse.cpu().numpy(),
                rank_scores=[x["scores"].cpu().numpy() for x in ranks])


@pytest.mark.parametrize("R,I,K,Q,ssmax", [(2, 64, 2048, 4, True), (4, 64, 256, 3, True), (3, 128, 2048, 1, False),
                                           (8, 64, 512, 2, True)])
def test_dcp_multi_query_ssmax_packed(R, I, K, Q, ssmax):
    """Several query tokens per request (causal), SSMax on: each rank scores its
    own tokens with the global SSMax factor; the merged selection equals the
    oracle's DCP selection over the ranks' score rows and the unsharded top-k,
    and the combined attention matches the oracle."""
    ctx = [9000, 20000, 1100, 4097, 1537, 700]
    wl = synth.make_workload(f"dcpq{R}_{I}_{K}_{Q}", ctx, [Q] * len(ctx), 16, topk=K, ssmax=ssmax)
    dw = DeviceWorkload(wl)
    p = dw.problem(0)
    lay = dw.layers[0]
    ws = dw.workspace()
    idx, ln, out, lse = dw.outputs()
    scores = dw.scores()
    sml.sml_indexer_scores(p, lay.iq8, lay.iq_scale, lay.iw, dw.index_cache, scores, ws)
    sml.sml_topk(p, scores, idx, ln, ws)
    assert sml.sml_read_device_status(ws)[0] == sml.SML_OK
    ref_idx, ref_len = idx.cpu().numpy(), ln.cpu().numpy()
    parity.check_topk(wl, scores.cpu().numpy(), ref_idx, ref_len)
    got = run_dcp_packed(dw, wl, R, I)
    # every rank's scores are the unsharded ones at its tokens (same SSMax factor)
    for t, row in enumerate(global_rows(wl, got["rank_scores"], R, I)):
        want = odcp.select(row, R, I, K)
        assert got["sel_len"][t] == len(want), f"token {t}: len"
        assert np.array_equal(got["sel"][t, :len(want)], want), f"token {t}: selection differs from the oracle"
    assert np.array_equal(got["sel_len"], ref_len)
    for t in range(wl.T):
        assert np.array_equal(got["sel"][t, :ref_len[t]], ref_idx[t, :ref_len[t]]), f"token {t}"
    parity.check_attention(wl, 0, ref_idx, ref_len, got["out"], got["lse"])
