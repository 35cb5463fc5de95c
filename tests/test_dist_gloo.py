"""The multi-rank benchmark path on CPU process groups (gloo): the step time
is the maximum over ranks, and the page's cfg_size x ulysses_size
arrangement (batch entries over rank groups, each entry's sequence over its
group) reproduces the single-process result.  The FP64 oracle stands in for
the device attention, so only the host logic and the exchanges are under
test here."""
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


def _oracle_attention(t, i, r, pos, split, theta):
    import oracle
    O, _ = oracle.joint_attention(t, i, r, pos, split, theta)          # [B, H', S, d] float64
    return torch.from_numpy(O).permute(0, 2, 1, 3).to(torch.bfloat16).contiguous()


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import bench
    from diffusion_transformer_joint_jattn_b200 import ulysses, workloads as W
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = 10.0 + 5.0 * rank                       # the last rank is the slow one
        m = bench.max_over_ranks(local_ms, world, torch.device("cpu"))
        # the benchmark's partition of one batch: B = 2 (the two guidance
        # branches), H = 4, streams divisible by the Ulysses size
        w = W.custom(B=2, H=4, d=64, S_txt=8, grid=4, n_ref=1)
        lens = [w.S_txt, w.S_img, w.S_ref]
        cfg, uly = ulysses.cfg_ulysses_layout(world, w.B, w.H, lens)
        groups = [dist.new_group(g) for g in ulysses.cfg_ulysses_groups(world, cfg, uly)]
        bsl, g, r = ulysses.rank_work(rank, w.B, cfg, uly)
        inp = W.make_inputs(w, seed=0)
        streams = [t[bsl] for t in (inp["qkv_txt"], inp["qkv_img"], inp["qkv_ref"])]
        shards = ulysses.shard_streams(streams, uly, r)
        out = ulysses.ulysses_attention(shards, inp["pos"], w.split, w.theta, group=groups[g],
                                        attention=_oracle_attention)
        full = _oracle_attention(inp["qkv_txt"], inp["qkv_img"], inp["qkv_ref"], inp["pos"], w.split, w.theta)
        ok, start = True, 0
        for t, o in zip(streams, out):
            S_s = t.shape[1]
            n = S_s // uly
            want = full[bsl, start + r * n:start + (r + 1) * n]
            ok = ok and o.shape == want.shape and torch.equal(o, want)
            start += S_s
        q.put((rank, m, (cfg, uly), ok))
        for grp in groups:
            dist.destroy_process_group(grp)
    except Exception as e:                                 # report, do not hang the parent
        q.put((rank, None, None, repr(e)))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(180)
@pytest.mark.parametrize("world,layout", [(2, (2, 1)), (4, (2, 2))])
def test_partition_matches_single_process(world, layout):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=150) for _ in procs]
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    for rank, m, lay, ok in res:
        assert ok is True, ok
        assert m == 10.0 + 5.0 * (world - 1)              # every rank sees the slowest rank's time
        assert lay == layout


def test_layout_rules():
    sys.path.insert(0, ROOT)
    from diffusion_transformer_joint_jattn_b200 import ulysses
    # the page's 8-GPU Base arrangement: cfg 2 x ulysses 4
    assert ulysses.cfg_ulysses_layout(8, 2, 24, [512, 16384]) == (2, 4)
    assert ulysses.cfg_ulysses_layout(4, 2, 24, [512, 16384]) == (2, 2)
    # distilled (B = 1, no guidance branches): the whole group is Ulysses
    assert ulysses.cfg_ulysses_layout(8, 1, 24, [512, 16384]) == (1, 8)
    with pytest.raises(ValueError):
        ulysses.cfg_ulysses_layout(8, 2, 6, [512, 16384])        # 6 heads over 4 ranks
    assert ulysses.cfg_ulysses_groups(8, 2, 4) == [[0, 1, 2, 3], [4, 5, 6, 7]]
    assert ulysses.rank_work(5, 2, 2, 4) == (slice(1, 2), 1, 1)


def test_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, 1, torch.device("cpu")) == 3.5
    assert bench.whole_job_tflops(10 ** 12, 1.0) == pytest.approx(1000.0)
