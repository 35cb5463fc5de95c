"""The Python binding checks every tensor it hands to the C ABI (device,
dtype, contiguity and exact shape) before the call: the ABI sees only
pointers, so a wrong size would otherwise become an out-of-bounds device
access.  Each bad argument below must raise ValueError without launching
anything."""
import pytest
import torch

from diffusion_transformer_joint_jattn_b200 import jattn
from diffusion_transformer_joint_jattn_b200 import workloads as W
from parity_util import to_device

pytestmark = pytest.mark.gpu


def _case(dev):
    w = W.custom(B=1, H=2, d=128, S_txt=16, grid=8, n_ref=0)        # S = 80
    return w, to_device(W.make_inputs(w, 1), dev)


def test_repair_outputs_are_checked(cuda_device):
    w, d = _case(cuda_device)
    args = (d["qkv_txt"], d["qkv_img"], d["qkv_ref"], d["pos"], w.split)
    n = jattn.repair_count(w.B, w.H, w.S_txt, w.S_img, w.S_ref, w.d, 0.05)
    good_o = torch.empty(w.B, w.S, w.H, w.d, dtype=torch.bfloat16, device=cuda_device)
    bad = [
        dict(o=torch.empty(w.B, w.S - 1, w.H, w.d, dtype=torch.bfloat16, device=cuda_device)),
        dict(o=good_o, lse=torch.empty(w.B, w.H, w.S, dtype=torch.bfloat16, device=cuda_device)),
        dict(o=good_o, lse=torch.empty(w.B, w.H, w.S - 1, dtype=torch.float32, device=cuda_device)),
        dict(o=good_o, repaired=torch.empty(w.B, w.H, n + 1, dtype=torch.int32, device=cuda_device)),
        dict(o=good_o, norm_w=torch.ones(3, 2, w.d, dtype=torch.bfloat16, device=cuda_device)),
        dict(o=good_o, norm_w=torch.ones(3, 2, w.d)),                               # host tensor
        dict(o=good_o, norm_w=torch.ones(2, 2, w.d, device=cuda_device)),
    ]
    for kw in bad:
        with pytest.raises(ValueError):
            jattn.fwd_fp8_repair_noalloc(*args, theta=w.theta, rho=0.05, **kw)
    with pytest.raises(ValueError):
        jattn.fwd_fp8_repair_noalloc(*args, None, theta=w.theta, rho=0.05)       # o is required
    with pytest.raises(ValueError):
        jattn.fwd_fp8_repair(*args, theta=w.theta, rho=0.05, o=bad[0]["o"])
    with pytest.raises(ValueError):
        jattn.fwd_fp8_repair(*args, theta=w.theta, rho=0.05,
                             workspace=torch.empty(16, dtype=torch.uint8, device=cuda_device))


def test_path_buffers_are_checked(cuda_device):
    w, d = _case(cuda_device)
    args = (d["qkv_txt"], d["qkv_img"], d["qkv_ref"], d["pos"], w.split, w.theta)
    q = torch.empty(w.B, w.H, w.S, w.d, dtype=torch.float16, device=cuda_device)
    short = torch.empty(w.B, w.H, w.S - 1, w.d, dtype=torch.float16, device=cuda_device)
    with pytest.raises(ValueError):
        jattn.rope_qkv(*args, "fp16", out=(q, short, q.clone(), None))
    with pytest.raises(ValueError):
        jattn.rope_qkv(d["qkv_txt"], d["qkv_img"], None, d["pos"][:-1], w.split, w.theta, "fp16")
    with pytest.raises(ValueError):
        jattn.fwd_bf16(q, q, short)
    with pytest.raises(ValueError):
        jattn.fwd_bf16(q, q, q, o=torch.empty(w.B, w.H, w.S, w.d, dtype=torch.bfloat16, device=cuda_device))
    q8, k8, v8, sc = jattn.rope_qkv(*args, "e4m3")
    with pytest.raises(ValueError):
        jattn.fwd_fp8(q8, k8, v8, sc[:2].contiguous())
    assert jattn.device_status()[0] == jattn.OK
