"""Ulysses sequence parallelism on CPU process groups (gloo, 2 and 4 ranks).

The exchange logic (two all-to-alls around a head-local attention) is checked
with the FP64 oracle as the local attention: every rank's output shard must
equal, bit for bit after the same bf16 rounding, its slice of the oracle run
on the whole sequence in one process.  Heads are independent, so any mix-up
of token or head order in either exchange changes some element."""
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


def _worker(rank, world, port, case, q):
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    from diffusion_transformer_joint_jattn_b200 import ulysses, workloads as W
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = W.custom(**case)
        inp = W.make_inputs(w, seed=4)
        streams = [inp["qkv_txt"], inp["qkv_img"], inp["qkv_ref"]]
        shards = ulysses.shard_streams(streams, world, rank)
        out = ulysses.ulysses_attention(shards, inp["pos"], w.split, w.theta, attention=_oracle_attention)
        full = _oracle_attention(*streams, inp["pos"], w.split, w.theta)   # [B, S, H, d]
        ok, start = True, 0
        for t, o in zip(streams, out):
            if t is None:
                ok = ok and o is None
                continue
            S_s = t.shape[1]
            n = S_s // world
            want = full[:, start + rank * n:start + (rank + 1) * n]
            ok = ok and o.shape == want.shape and torch.equal(o, want)
            start += S_s
        q.put((rank, ok))
    except Exception as e:                                               # report, do not hang the parent
        q.put((rank, repr(e)))
    finally:
        dist.destroy_process_group()


CASES = [
    dict(B=1, H=4, d=64, S_txt=8, grid=4, n_ref=1),      # txt 8, img 16, ref 16
    dict(B=2, H=8, d=128, S_txt=12, grid=4, n_ref=0),    # no reference stream
]


@pytest.mark.timeout(180)
@pytest.mark.parametrize("world", [2, 4])
@pytest.mark.parametrize("case", CASES, ids=lambda c: f"B{c['B']}H{c['H']}d{c['d']}r{c['n_ref']}")
def test_ulysses_matches_single_process(world, case):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, case, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=150) for _ in procs)
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    assert all(ok is True for _, ok in res), res


def test_shape_checks():
    sys.path.insert(0, ROOT)
    from diffusion_transformer_joint_jattn_b200 import ulysses
    t = torch.zeros(1, 6, 3, 4, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        ulysses.shard_streams([t, None, None], 4, 0)                     # 6 tokens over 4 ranks
    with pytest.raises(ValueError):
        ulysses._check_shards([torch.zeros(1, 2, 3, 6, 64)], 4)          # 6 heads over 4 ranks
