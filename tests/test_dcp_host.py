"""Host-side DCP sharding (CPU): a rank's local block table and lengths, and
the local <-> global position maps, against the ownership rule of the oracle;
two gloo ranks that shard the same batch independently partition its tokens."""
import numpy as np
import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import dcp as odcp
from sparse_mla_attention_indexer_b200 import dcp


def _batch(seed=0):
    rng = np.random.default_rng(seed)
    ctx = np.array([1100, 9000, 4097, 20000, 1537], dtype=np.int32)
    pages = (ctx + 63) // 64
    bt = np.zeros((len(ctx), pages.max()), dtype=np.int32)
    perm = rng.permutation(int(pages.sum()))
    off = 0
    for b, n in enumerate(pages):
        bt[b, :n] = perm[off:off + n]
        off += n
    return bt, ctx


@pytest.mark.parametrize("R,I", [(1, 64), (2, 64), (3, 64), (8, 128), (5, 192)])
def test_shards_partition_every_request_by_the_oracle_rule(R, I):
    bt, ctx = _batch()
    seen = [np.zeros(int(L), dtype=np.int32) for L in ctx]
    for r in range(R):
        lbt, lens = dcp.shard(bt, ctx, r, R, I)
        for b, L in enumerate(ctx):
            local = np.arange(lens[b])
            g = dcp.global_position(local, r, R, I)
            assert np.all(g < L) and np.all(np.diff(g) > 0)          # in range, order kept
            assert np.all(odcp.owner(g, R, I) == r)                  # the oracle's rule
            # the local table maps local positions to the same physical rows
            assert np.array_equal(lbt[b, local // 64], bt[b, g // 64])
            assert np.array_equal(local % 64, g % 64)
            seen[b][g] += 1
    assert all(np.all(s == 1) for s in seen)                          # each token on exactly one rank


def test_shard_matches_the_gpu_tests_sharding():
    from tests.test_gpu_dcp import shard as test_shard
    from types import SimpleNamespace
    bt, ctx = _batch(1)
    wl = SimpleNamespace(B=len(ctx), ctx_len=ctx, block_table=bt)
    for R, I in ((2, 64), (4, 64), (8, 128), (3, 64)):
        for r, (tbt, tlen) in enumerate(test_shard(wl, R, I)):
            lbt, lens = dcp.shard(bt, ctx, r, R, I)
            assert np.array_equal(lens, tlen)
            for b in range(len(ctx)):
                n = (int(lens[b]) + 63) // 64
                assert np.array_equal(lbt[b, :n], tbt[b, :n])


def test_shard_refuses_an_empty_rank():
    bt, ctx = _batch()
    with pytest.raises(ValueError):
        dcp.shard(bt, np.array([100], dtype=np.int32), 3, 4, 64)
    with pytest.raises(ValueError):
        dcp.rank_pages(1000, 0, 2, 96)


def _rank_main(rank, world, port, out_q):
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    bt, ctx = _batch()
    lbt, lens = dcp.shard(bt, ctx, rank, world, 64)
    mine = [dcp.global_position(np.arange(n), rank, world, 64).tolist() for n in lens]
    allp = [None] * world
    dist.all_gather_object(allp, mine)
    if rank == 0:
        ok = all(sorted(sum((allp[r][b] for r in range(world)), [])) == list(range(int(L)))
                 for b, L in enumerate(ctx))
        out_q.put(ok)
    dist.destroy_process_group()


def test_two_gloo_ranks_partition_the_batch():
    import socket
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    assert q.get(timeout=10) is True


def test_rank_arrays_count_each_querys_visible_tokens_by_the_oracle_rule():
    rng = np.random.default_rng(5)
    ctx = np.array([1100, 9000, 4097, 700], dtype=np.int32)
    qc = np.array([1, 4, 2, 3])
    cu_q = np.concatenate([[0], np.cumsum(qc)]).astype(np.int32)
    n = dcp.visible_lengths(cu_q, ctx)
    for R, I in ((2, 64), (3, 64), (8, 128), (5, 192)):
        tot = np.zeros_like(n)
        for r in range(R):
            local_len, vis, glob = dcp.rank_arrays(cu_q, ctx, r, R, I)
            assert np.array_equal(glob, n)
            for t in range(len(n)):
                assert vis[t] == np.sum(odcp.owner(np.arange(n[t]), R, I) == r)   # brute force
            for b, L in enumerate(ctx):
                assert local_len[b] == np.sum(odcp.owner(np.arange(L), R, I) == r)
            tot += vis
        assert np.array_equal(tot, n)                                            # the ranks partition every query
    assert rng is not None


def _gather_main(rank, world, port, out_q):
    import torch
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    t = torch.full((3, 5), float(rank)) + torch.arange(5.0)
    got = dcp._all_gather(t)
    out_q.put((rank, [x.numpy() for x in got]))
    dist.destroy_process_group()


def test_exchange_gathers_every_ranks_array_in_rank_order():
    import socket
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_gather_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank in range(2):
        for src in range(2):
            assert np.array_equal(res[rank][src], np.full((3, 5), float(src)) + np.arange(5.0))
