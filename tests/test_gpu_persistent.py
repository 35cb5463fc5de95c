"""The forward kernel's persistent grid.  When every work item (batch * head,
pair of query tiles) walks at most four key tiles and there are more items
than SMs, one CTA per SM walks items in turn, with every barrier phase and
ring position carried on from one item to the next.  The case below has 160
items of four key tiles each, so on a 148-SM part some CTAs take two items;
every row is checked against the oracle for the 16-bit, high-precision and
e4m3 instances."""
import numpy as np
import pytest
import torch

import oracle
from diffusion_transformer_joint_jattn_b200 import jattn
from diffusion_transformer_joint_jattn_b200 import workloads as W
from parity_util import BF16_MAX_ABS, BF16_REL_L2, gather_lse, gather_rows, max_abs, rel_l2, to_device

pytestmark = pytest.mark.gpu

CASE = dict(B=2, H=40, d=128, S_txt=64, grid=20, n_ref=0)     # S = 464: 4 key tiles, 2 query-tile pairs


def _items(w):
    return ((w.S + 127) // 128 + 1) // 2 * w.B * w.H


@pytest.fixture(scope="module")
def case(cuda_device):
    w = W.custom(**CASE)
    if _items(w) <= torch.cuda.get_device_properties(cuda_device).multi_processor_count:
        pytest.skip("fewer work items than SMs: the grid would not be persistent")
    inp = W.make_inputs(w, seed=31)
    O, L = oracle.joint_attention(inp["qkv_txt"], inp["qkv_img"], inp["qkv_ref"], inp["pos"], w.split, w.theta)
    return w, inp, O, L


def test_persistent_fp16(cuda_device, case):
    w, inp, O, L = case
    d = to_device(inp, cuda_device)
    q, k, v, _ = jattn.rope_qkv(d["qkv_txt"], d["qkv_img"], d["qkv_ref"], d["pos"], w.split, w.theta, "fp16")
    o, lse = jattn.fwd_bf16(q, k, v, want_lse=True)
    torch.cuda.synchronize()
    rows = torch.arange(w.S).expand(w.B, w.H, w.S)
    got = gather_rows(o, rows)
    assert rel_l2(got, O) <= BF16_REL_L2
    assert max_abs(got, O) <= BF16_MAX_ABS
    np.testing.assert_allclose(gather_lse(lse, rows), L, rtol=0, atol=2e-3)
    assert jattn.device_status()[0] == jattn.OK


def test_persistent_high_precision(cuda_device, case):
    w, inp, O, L = case
    d = to_device(inp, cuda_device)
    ops = jattn.rope_qkv_hp(d["qkv_txt"], d["qkv_img"], d["qkv_ref"], d["pos"], w.split, w.theta)
    o, lse = jattn.fwd_bf16_hp(*ops, want_lse=True)
    torch.cuda.synchronize()
    rows = torch.arange(w.S).expand(w.B, w.H, w.S)
    got = gather_rows(o, rows)
    assert rel_l2(got, O) <= BF16_REL_L2
    assert max_abs(got, O) <= BF16_MAX_ABS
    np.testing.assert_allclose(gather_lse(lse, rows), L, rtol=0, atol=2e-3)
    assert jattn.device_status()[0] == jattn.OK


def test_persistent_fp8(cuda_device, case):
    w, inp, _, _ = case
    d = to_device(inp, cuda_device)
    q8, k8, v8, sc = jattn.rope_qkv(d["qkv_txt"], d["qkv_img"], d["qkv_ref"], d["pos"], w.split, w.theta, "e4m3")
    o, lse = jattn.fwd_fp8(q8, k8, v8, sc, want_lse=True)
    torch.cuda.synchronize()
    deq = [oracle.dequantize_blocks(t.cpu().view(torch.uint8).numpy(), sc[i].cpu().numpy())
           for i, t in enumerate((q8, k8, v8))]
    O2, L2 = oracle.attention_on(*deq)
    rows = torch.arange(w.S).expand(w.B, w.H, w.S)
    assert rel_l2(gather_rows(o, rows), O2) <= 3e-2
    np.testing.assert_allclose(gather_lse(lse, rows), L2, rtol=0, atol=1e-4)
    assert jattn.device_status()[0] == jattn.OK
