"""The allocation-free FP8-with-repair entry point (jattn_fwd_fp8_repair_noalloc).

Collected last on purpose: it must pass on its own and after every other
test.  It checks that the path gives exactly the result of the workspace
entry point (the same kernels on the same inputs), that a repeated call
leaves the device's free memory unchanged (nothing is allocated once the
library's scratch array is mapped), and that an input whose workspace would
not fit the array is refused before anything runs.
"""
import pytest
import torch

from diffusion_transformer_joint_jattn_b200 import jattn
from diffusion_transformer_joint_jattn_b200 import workloads as W
from parity_util import to_device

pytestmark = pytest.mark.gpu


def _inputs(dev, seed=12):
    w = W.custom(B=2, H=2, d=128, S_txt=77, grid=9, n_ref=1)     # S = 239
    return w, to_device(W.make_inputs(w, seed), dev)


def _outputs(w, dev, rho):
    n = jattn.repair_count(w.B, w.H, w.S_txt, w.S_img, w.S_ref, w.d, rho)
    return (torch.empty(w.B, w.S, w.H, w.d, dtype=torch.bfloat16, device=dev),
            torch.empty(w.B, w.H, w.S, dtype=torch.float32, device=dev),
            torch.empty(w.B, w.H, n, dtype=torch.int32, device=dev))


@pytest.mark.parametrize("rho", [0.05, 0.0])
def test_noalloc_equals_workspace_path(cuda_device, rho):
    w, d = _inputs(cuda_device)
    o, lse, rep = _outputs(w, cuda_device, rho)
    jattn.fwd_fp8_repair_noalloc(d["qkv_txt"], d["qkv_img"], d["qkv_ref"], d["pos"], w.split, o, w.theta, rho=rho,
                                 lse=lse, repaired=rep if rep.numel() else None)
    o2, lse2, rep2 = jattn.fwd_fp8_repair(d["qkv_txt"], d["qkv_img"], d["qkv_ref"], d["pos"], w.split, w.theta,
                                          rho=rho, want_lse=True, want_repaired=True)
    torch.cuda.synchronize()
    assert torch.equal(o, o2)
    assert torch.equal(lse, lse2)
    assert torch.equal(rep, rep2)
    assert jattn.device_status()[0] == jattn.OK


def test_noalloc_makes_no_allocation(cuda_device):
    w, d = _inputs(cuda_device, seed=13)
    o, lse, rep = _outputs(w, cuda_device, 0.05)
    nw = W.norm_weights(w.d, 13).to(cuda_device)

    def call():
        jattn.fwd_fp8_repair_noalloc(d["qkv_txt"], d["qkv_img"], d["qkv_ref"], d["pos"], w.split, o, w.theta,
                                     rho=0.05, norm_w=nw, lse=lse, repaired=rep)
        torch.cuda.synchronize()

    call()                                       # maps the scratch array and loads the kernels
    free0, _ = torch.cuda.mem_get_info()
    torch_alloc0 = torch.cuda.memory_allocated()
    for _ in range(3):
        call()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0
    assert torch.cuda.memory_allocated() == torch_alloc0
    assert jattn.device_status()[0] == jattn.OK


def test_noalloc_refuses_oversize_inputs(cuda_device):
    """i2i at 2048x2048 (S = 33280, B = 2, H = 24) needs ~1 GB of workspace,
    more than the array: refused on the host before anything is launched.
    Every tensor pointer is NULL, so even if the size check stopped coming
    first, the call would end in the argument checks (INVALID_ARG) and never
    reach a kernel."""
    w = W.BY_NAME["i2i_2048_base"]
    need = jattn.repair_workspace_bytes(w.B, w.H, w.S_txt, w.S_img, w.S_ref, w.d, 0.005)
    assert need > jattn.NOALLOC_SCRATCH_BYTES
    lib = jattn.load()
    shape = jattn.make_shape(w.B, w.H, w.S_txt, w.S_img, w.S_ref, w.d)
    sp = (jattn.ctypes.c_int32 * 3)(*w.split)
    code = lib.jattn_fwd_fp8_repair_noalloc(jattn.ctypes.byref(shape), None, None, None, None, w.theta, sp, None,
                                            1e-6, 0.005, None, None, None, 0.0, None)
    assert code == jattn.ERR_UNSUPPORTED
    assert jattn.device_status()[0] == jattn.OK
