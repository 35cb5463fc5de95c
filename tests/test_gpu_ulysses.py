"""The Ulysses path on the GPU with a one-rank NCCL group: the exchanges are
NCCL all-to-alls (copies with one rank) around the library's device
attention; the result must equal the device path on the whole sequence, and
with the high-precision path (what the multi-GPU bench runs) it must meet
the BF16 bars against the FP64 oracle.
(More ranks need more GPUs than a test box has; the exchange logic itself is
checked on 2 and 4 CPU ranks in test_ulysses_gloo.py.)"""
import os
import socket

import pytest
import torch
import torch.distributed as dist

import oracle
from diffusion_transformer_joint_jattn_b200 import jattn, ulysses
from diffusion_transformer_joint_jattn_b200 import workloads as W
from parity_util import BF16_MAX_ABS, BF16_REL_L2, gather_rows, max_abs, rel_l2, to_device

pytestmark = pytest.mark.gpu


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def test_ulysses_single_rank_nccl(cuda_device):
    w = W.custom(B=2, H=4, d=128, S_txt=40, grid=12, n_ref=1)
    d = to_device(W.make_inputs(w, 8), cuda_device)
    streams = [d["qkv_txt"], d["qkv_img"], d["qkv_ref"]]
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=cuda_device)
    try:
        shards = ulysses.shard_streams(streams, 1, 0)
        out = ulysses.ulysses_attention(shards, d["pos"], w.split, w.theta, precise=False)
        out_hp = ulysses.ulysses_attention(shards, d["pos"], w.split, w.theta, precise=True)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    inp = W.make_inputs(w, 8)
    O, _ = oracle.joint_attention(inp["qkv_txt"], inp["qkv_img"], inp["qkv_ref"], inp["pos"], w.split, w.theta)
    got = gather_rows(torch.cat(out_hp, dim=1), torch.arange(w.S).expand(w.B, w.H, w.S))
    assert rel_l2(got, O) <= BF16_REL_L2
    assert max_abs(got, O) <= BF16_MAX_ABS
    o = jattn.joint_attention(*streams, d["pos"], w.split, w.theta, precise=False)
    torch.cuda.synchronize()
    assert torch.equal(torch.cat(out, dim=1), o)
    assert jattn.device_status()[0] == jattn.OK
