"""Decode context parallelism across processes: two ranks, each its own
process on the one GPU, each holding half of the cache by token, exchange
their packed candidates and partial attentions through torch.distributed
(gloo, staged through host memory) in sml's dcp.dcp_layer.  The ranks'
kernels never wait on each other; only the host-side collectives do.  The
result must equal the unsharded step's selection bit for bit, and its
attention must match the float64 oracle."""
import datetime
import multiprocessing as mp
import socket

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

CTX, Q, H, K, R, I = [3000, 5000, 900], [2, 1, 3], 16, 512, 2, 64


def _workload():
    from sparse_mla_attention_indexer_b200 import synth
    return synth.make_workload("dcp_proc", CTX, Q, H, topk=K, ssmax=True)


def _rank_main(rank, port, out_q):
    import os
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import torch
    import torch.distributed as dist

    from sparse_mla_attention_indexer_b200 import dcp, sml
    from sparse_mla_attention_indexer_b200.device import DeviceWorkload
    try:
        dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=R,
                                timeout=datetime.timedelta(seconds=120))
        torch.cuda.set_device(0)
        wl = _workload()
        dw = DeviceWorkload(wl)
        lay = dw.layers[0]
        local_len, vis, glob = dcp.rank_arrays(wl.cu_q, wl.ctx_len, rank, R, I)
        bt = dcp.shard_pages(wl.block_table, wl.ctx_len, rank, R, I)
        keep = [torch.from_numpy(a).cuda() for a in (bt, local_len, vis, glob)]
        p = sml.make_problem(num_heads=H, topk=K, rope_dim=lay.rope_dim, cu_q=dw.cu_q, ctx_len=keep[1],
                             block_table=keep[0], max_ctx=int(local_len.max()), ssmax=wl.ssmax,
                             sm_scale=wl.sm_scale, ssmax_s=wl.ssmax_s, ssmax_s_index=wl.ssmax_s_index,
                             num_tokens=wl.T, vis_len=keep[2], ssmax_len=keep[3])
        sel, sel_len, out, lse = dcp.dcp_layer(p, lay.q, lay.iq8, lay.iq_scale, lay.iw, dw.latent, dw.index_cache,
                                               rank=rank, world=R, interleave=I)
        torch.cuda.synchronize()
        sel_h, len_h = sel.cpu().numpy(), sel_len.cpu().numpy()
        mine = [dcp.global_position(sel_h[t, :len_h[t]], rank, R, I) for t in range(wl.T)]
        res = dict(rank=rank, mine=mine, out=out.cpu().numpy(), lse=lse.cpu().numpy())
        if rank == 0:
            # the unsharded step on the same GPU, for the bit-exact comparison
            ws = dw.workspace()
            idx, ln, o, l = dw.outputs()
            scores = dw.scores()
            pf = dw.problem(0)
            sml.sml_indexer_scores(pf, lay.iq8, lay.iq_scale, lay.iw, dw.index_cache, scores, ws)
            sml.sml_topk(pf, scores, idx, ln, ws)
            assert sml.sml_read_device_status(ws)[0] == sml.SML_OK
            res.update(ref_idx=idx.cpu().numpy(), ref_len=ln.cpu().numpy(), ref_scores=scores.cpu().numpy())
        out_q.put(res)
        dist.destroy_process_group()
    except Exception as e:  # reported to the parent
        out_q.put(dict(rank=rank, error=repr(e)))
        raise


def test_two_processes_exchange_over_gloo():
    from tests import parity
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, port, q)) for r in range(R)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(R):
        x = q.get(timeout=300)
        assert "error" not in x, x
        res[x["rank"]] = x
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    wl = _workload()
    r0 = res[0]
    parity.check_topk(wl, r0["ref_scores"], r0["ref_idx"], r0["ref_len"])
    for t in range(wl.T):
        got = np.sort(np.concatenate([res[r]["mine"][t] for r in range(R)]))
        want = r0["ref_idx"][t, :r0["ref_len"][t]]
        assert np.array_equal(got, want), f"token {t}: the ranks' selections differ from the unsharded top-k"
    for r in range(1, R):   # the combined attention is the same on every rank
        assert np.array_equal(res[r]["out"], r0["out"]) and np.array_equal(res[r]["lse"], r0["lse"], equal_nan=True)
    parity.check_attention(wl, 0, r0["ref_idx"], r0["ref_len"], r0["out"], r0["lse"])
