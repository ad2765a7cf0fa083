"""The multi-rank bench logic on CPU: two gloo ranks, each with its own timing,
agree on the slowest rank's time, and the whole-job rate counts both ranks'
work against it (weak scaling, independent replicas)."""
import multiprocessing as mp
import os
import socket
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, ms, out):
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        import bench
        ms_max = bench.max_over_ranks(ms[rank], device="cpu")
        bench.barrier()
        out.put((rank, ms_max, bench.whole_job_rate(world, 32, ms_max)))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_report_the_slowest_rank():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    ms = [0.10, 0.25]   # rank 1 is the slow one
    procs = [ctx.Process(target=_rank, args=(r, 2, port, ms, out)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [0.25, 0.25]
    # 2 ranks x 32 queries in 0.25 ms
    assert all(abs(r[2] - 2 * 32 / 0.25e-3) < 1e-6 for r in res)


def test_single_process_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(0.5, device="cpu") == 0.5
    assert bench.whole_job_rate(1, 32, 0.5) == 32 / 0.5e-3
