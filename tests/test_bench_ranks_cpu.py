"""bench.py's multi-rank host logic over a real two-rank gloo group on the CPU: the
timing that is reported is the slowest rank's, and every rank draws its own inputs."""
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _worker(rank, world, port, out):
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        import bench
        bench.WORKLOAD = "mha2k"
        out[rank] = (bench.max_over_ranks(10.0 + 5.0 * rank, world, "cpu"),
                     [w.seed for w in bench.workload_variants(rank)])
    finally:
        dist.destroy_process_group()


def test_two_ranks_report_the_slowest_time_and_distinct_inputs():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    ctx = mp.get_context("spawn")
    with ctx.Manager() as man:
        out = man.dict()
        procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
        assert all(p.exitcode == 0 for p in procs)
        res = dict(out)
    assert res[0][0] == res[1][0] == 15.0
    assert res[0][1] != res[1][1]                 # weak scaling: each rank its own batch
    assert len(set(res[0][1])) == 1               # the causal variant reuses the rank's tensors
