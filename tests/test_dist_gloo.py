"""The multi-rank path on CPU: two gloo ranks exercise the benchmark's host
logic for N > 1 -- every rank draws its own batch (weak scaling: the units
are independent (batch, head) problems, no data-path collective) and the
step time is the maximum over ranks."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import bench
    from diffusion_transformer_joint_jattn_b200 import workloads as W
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = 10.0 + 5.0 * rank                       # rank 1 is the slow one
        m = bench.max_over_ranks(local_ms, world, torch.device("cpu"))
        w = W.custom(B=1, H=2, d=64, S_txt=8, grid=4, n_ref=0)
        inp = W.make_inputs(w, seed=bench.rank_seed(rank))
        digest = float(inp["qkv_img"].float().sum())
        digests = [None] * world
        dist.all_gather_object(digests, digest)
        q.put((rank, m, digests, bench.whole_job_tflops(world, w.flops, m)))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_rank_max_time_and_independent_batches():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=100) for _ in procs]
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    res.sort()
    for rank, m, digests, value in res:
        assert m == 15.0                                  # both ranks see the slowest rank's time
        assert digests[0] != digests[1]                   # each rank has its own synthetic batch
    from diffusion_transformer_joint_jattn_b200 import workloads as W
    w = W.custom(B=1, H=2, d=64, S_txt=8, grid=4, n_ref=0)
    assert res[0][3] == pytest.approx(2 * w.flops / 15.0 / 1e9)


def test_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, 1, torch.device("cpu")) == 3.5
    assert bench.whole_job_tflops(1, 10 ** 12, 1.0) == pytest.approx(1000.0)
