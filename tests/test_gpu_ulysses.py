"""The Ulysses path on the GPU with a one-rank NCCL group: the exchanges are
NCCL all-to-alls (copies with one rank) around the library's device
attention, and the result must equal the device path on the whole sequence.
(More ranks need more GPUs than a test box has; the exchange logic itself is
checked on 2 and 4 CPU ranks in test_ulysses_gloo.py.)"""
import os
import socket

import pytest
import torch
import torch.distributed as dist

from diffusion_transformer_joint_jattn_b200 import jattn, ulysses
from diffusion_transformer_joint_jattn_b200 import workloads as W
from parity_util import to_device

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
        out = ulysses.ulysses_attention(ulysses.shard_streams(streams, 1, 0), d["pos"], w.split, w.theta)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    o = jattn.joint_attention(*streams, d["pos"], w.split, w.theta)
    torch.cuda.synchronize()
    assert torch.equal(torch.cat(out, dim=1), o)
    assert jattn.device_status()[0] == jattn.OK
