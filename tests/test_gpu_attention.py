"""GPU parity of the attention forward (jattn_fwd_bf16 / jattn_fwd_fp8) and
of the whole path (prologue + forward) against the FP64 oracle, through the
C ABI.

BF16 path (bf16 in, fp16 operands in the MMAs, bf16 out): rel-L2 <= 5e-3 and
max-abs <= 2e-2 over the sampled rows (all rows for the small cases, 4096
rows per (b, h) for the large workloads).  On the outlier workloads the
max-abs bar lies below what 16-bit tensor-core operands can reach at all:
the oracle itself, run on fp16-rounded rotated Q/K with a bf16 result,
already shows max-abs 2.7e-2 .. 5e-2 there.  Those tests therefore assert
max-abs within 1.25x of that measured floor (and 2e-2 where the floor is
below it), plus the kernel's own deviation from the floored oracle.  The
pure-bf16-operand variant is checked against its own format floor.  The
high-precision pair (jattn_rope_qkv_hp + jattn_fwd_bf16_hp), the BF16 path
that joint_attention() uses by default, meets both bars unrelaxed on every
workload (test_gpu_hp.py).
"""
import numpy as np
import pytest
import torch

import oracle
from diffusion_transformer_joint_jattn_b200 import jattn
from diffusion_transformer_joint_jattn_b200 import workloads as W
from parity_util import (BF16_MAX_ABS, BF16_REL_L2, fp16_operand_floor, gather_lse, gather_rows, max_abs,
                         rel_l2, round_bf16, to_device, workload_case)

pytestmark = pytest.mark.gpu


def _run_bf16(w, inp, dev, operand="fp16", want_lse=True):
    d = to_device(inp, dev)
    q, k, v, _ = jattn.rope_qkv(d["qkv_txt"], d["qkv_img"], d["qkv_ref"], d["pos"], w.split, w.theta, operand)
    o, lse = jattn.fwd_bf16(q, k, v, want_lse=want_lse)
    torch.cuda.synchronize()
    return o, lse


SMALL = [
    dict(B=1, H=2, d=64, S_txt=32, grid=16, n_ref=0),      # tiny workload, S = 288 (ragged tail)
    dict(B=1, H=1, d=128, S_txt=1, grid=0, n_ref=0),       # S = 1
    dict(B=1, H=1, d=128, S_txt=0, grid=16, n_ref=0),      # no text, S = 256 (exact tiles)
    dict(B=2, H=2, d=128, S_txt=77, grid=9, n_ref=1),      # S = 239, reference image
    dict(B=1, H=3, d=64, S_txt=3, grid=11, n_ref=0),       # S = 124 < one tile
    dict(B=1, H=1, d=128, S_txt=129, grid=0, n_ref=0),     # S = 129: one-row tail tile
]


@pytest.mark.parametrize("case", SMALL, ids=lambda c: f"B{c['B']}H{c['H']}d{c['d']}t{c['S_txt']}g{c['grid']}r{c['n_ref']}")
def test_joint_attention_small_full_rows(cuda_device, case):
    w = W.custom(**case)
    inp = W.make_inputs(w, seed=3)
    o, lse = _run_bf16(w, inp, cuda_device)
    O, L = oracle.joint_attention(inp["qkv_txt"], inp["qkv_img"], inp["qkv_ref"], inp["pos"], w.split, w.theta)
    rows = torch.arange(w.S).expand(w.B, w.H, w.S)
    got = gather_rows(o, rows)
    assert rel_l2(got, O) <= BF16_REL_L2, rel_l2(got, O)
    assert max_abs(got, O) <= BF16_MAX_ABS, max_abs(got, O)
    np.testing.assert_allclose(gather_lse(lse, rows), L, rtol=0, atol=2e-3)
    assert jattn.device_status()[0] == jattn.OK


def test_tiny_workload_bf16_operands(cuda_device):
    """Pure bf16 MMA operands (bf16 rounding of the rotated Q/K and of P):
    a looser floor set by bf16's 8-bit mantissa, 1e-2 rel-L2."""
    w = W.BY_NAME["tiny"]
    inp = W.make_inputs(w, 0)
    o, _ = _run_bf16(w, inp, cuda_device, operand="bf16")
    O, _ = oracle.joint_attention(inp["qkv_txt"], inp["qkv_img"], inp["qkv_ref"], inp["pos"], w.split, w.theta)
    got = gather_rows(o, torch.arange(w.S).expand(w.B, w.H, w.S))
    assert rel_l2(got, O) <= 1e-2


def test_constant_values_through_kernel(cuda_device):
    """V constant per head -> O equals that constant for every row (checks
    the P.V product and the normalisation independently of the logits)."""
    w = W.custom(B=1, H=2, d=128, S_txt=40, grid=15, n_ref=0)        # S = 265
    inp = W.make_inputs(w, 1)
    for key in ("qkv_txt", "qkv_img"):
        inp[key][:, :, 2] = torch.linspace(-2, 2, 128).to(torch.bfloat16)
    o, _ = _run_bf16(w, inp, cuda_device, want_lse=False)
    want = torch.linspace(-2, 2, 128).to(torch.bfloat16).to(torch.float32)
    np.testing.assert_allclose(o.float().cpu().numpy(), np.broadcast_to(want.numpy(), o.shape), atol=2e-2, rtol=0)


@pytest.mark.slow
@pytest.mark.parametrize("name", ["t2i_1024_base", "t2i_2048_base", "i2i_2048_base"])
def test_workload_bf16_sampled_rows(cuda_device, name):
    w, inp, rows, O, L = workload_case(name)
    o, lse = _run_bf16(w, inp, cuda_device)
    got = gather_rows(o, rows)
    floor = fp16_operand_floor(w, inp, rows)              # float64, fp16 Q/K operands
    r, m = rel_l2(got, O), max_abs(got, O)
    rf, mf = rel_l2(round_bf16(floor), O), max_abs(round_bf16(floor), O)
    r_kernel = rel_l2(got, floor)
    print(f"{name}: rel-L2 {r:.3e} max-abs {m:.3e} | fp16-operand floor (bf16 out) rel-L2 {rf:.3e} "
          f"max-abs {mf:.3e} | kernel vs fp16-operand oracle rel-L2 {r_kernel:.3e}")
    assert r <= BF16_REL_L2
    assert m <= max(BF16_MAX_ABS, 1.25 * mf)
    assert r_kernel <= 2.5e-3
    # LSE ~ the row's largest logit (up to ~40 here); fp16 rounding of the
    # rotated Q/K makes its error relative (~7e-4), hence rtol.
    np.testing.assert_allclose(gather_lse(lse, rows), L, rtol=2e-3, atol=5e-3)
    assert jattn.device_status()[0] == jattn.OK


@pytest.mark.parametrize("case", SMALL[:4], ids=lambda c: f"B{c['B']}H{c['H']}d{c['d']}t{c['S_txt']}g{c['grid']}r{c['n_ref']}")
def test_joint_attention_with_qk_norm(cuda_device, case):
    """The whole path with the query/key RMSNorm fused into the prologue,
    against the oracle's norm -> RoPE -> attention, every row."""
    w = W.custom(**case)
    inp = W.make_inputs(w, seed=21)
    nw = W.norm_weights(w.d, 21)
    d = to_device(inp, cuda_device)
    q, k, v, _ = jattn.rope_qkv(d["qkv_txt"], d["qkv_img"], d["qkv_ref"], d["pos"], w.split, w.theta, "fp16",
                                norm_w=nw.to(cuda_device))
    o, lse = jattn.fwd_bf16(q, k, v, want_lse=True)
    torch.cuda.synchronize()
    O, L = oracle.joint_attention(inp["qkv_txt"], inp["qkv_img"], inp["qkv_ref"], inp["pos"], w.split, w.theta,
                                  norm_w=nw, eps=1e-6)
    rows = torch.arange(w.S).expand(w.B, w.H, w.S)
    got = gather_rows(o, rows)
    assert rel_l2(got, O) <= BF16_REL_L2, rel_l2(got, O)
    assert max_abs(got, O) <= BF16_MAX_ABS, max_abs(got, O)
    np.testing.assert_allclose(gather_lse(lse, rows), L, rtol=0, atol=2e-3)
    assert jattn.device_status()[0] == jattn.OK


@pytest.mark.parametrize("pinned", [False, True])
def test_host_buffers_end_to_end(cuda_device, pinned):
    """The public one-call API with host tensors (jattn_joint_attention_host:
    copies in, the path pipelined over the batch, copy out): the same bytes
    as the device-tensor call -- the high-precision pair by default, the
    plain pair on bf16 operands with precise=False -- from pageable or pinned
    host memory."""
    w = W.BY_NAME["tiny"]
    inp = W.make_inputs(w, 0)
    if pinned:
        inp = {k: (None if v is None else v.pin_memory()) for k, v in inp.items()}
    o_host = jattn.joint_attention(inp["qkv_txt"], inp["qkv_img"], inp["qkv_ref"], inp["pos"], w.split, w.theta)
    assert o_host.device.type == "cpu"
    d = to_device(inp, cuda_device)
    o_dev = jattn.joint_attention(d["qkv_txt"], d["qkv_img"], d["qkv_ref"], d["pos"], w.split, w.theta)
    hp = jattn.rope_qkv_hp(d["qkv_txt"], d["qkv_img"], d["qkv_ref"], d["pos"], w.split, w.theta)
    o_hp, _ = jattn.fwd_bf16_hp(*hp)
    torch.cuda.synchronize()
    assert torch.equal(o_dev, o_hp)
    assert torch.equal(o_host, o_hp.cpu())
    o_plain = jattn.joint_attention(inp["qkv_txt"], inp["qkv_img"], inp["qkv_ref"], inp["pos"], w.split, w.theta,
                                    precise=False)
    o_dev, _ = _run_bf16(w, inp, cuda_device, operand="bf16", want_lse=False)
    assert torch.equal(o_plain, o_dev.cpu())
    with pytest.raises(ValueError):
        jattn.joint_attention(inp["qkv_txt"], inp["qkv_img"], inp["qkv_ref"], inp["pos"], w.split, w.theta,
                              precise=False, operand_dtype="fp16")


@pytest.mark.parametrize("path,B,H", [("bf16", 3, 2), ("fp8", 3, 2), ("bf16", 2, 12), ("fp8", 1, 9),
                                      ("bf16", 2, 5), ("plain", 2, 12), ("bf16", 1, 9)])
def test_host_entry_pipelined_batch(cuda_device, path, B, H):
    """Every (batch entry, head group) chunk runs as its own (2-D copy in,
    kernels, 2-D copy out) stage on the three streams -- H = 12 splits into
    6 groups of 2 heads, 9 into 3 groups of 3, 2 and 5 stay whole; the result
    equals the device entry points' on the whole batch (the high-precision
    pair, whose per-head channel-pair choice and block scales do not depend
    on the chunking; the plain bf16-operand pair; the e4m3 pair), also when
    the caller's stream already has work queued and the output buffer is
    reused."""
    w = W.custom(B=B, H=H, d=128, S_txt=77, grid=9, n_ref=1)
    inp = {k: (None if v is None else v.pin_memory()) for k, v in W.make_inputs(w, 5).items()}
    d = to_device(inp, cuda_device)
    kw = {}
    if path == "bf16":
        hp = jattn.rope_qkv_hp(d["qkv_txt"], d["qkv_img"], d["qkv_ref"], d["pos"], w.split, w.theta)
        o_dev, _ = jattn.fwd_bf16_hp(*hp)
    elif path == "plain":
        q, k, v, _ = jattn.rope_qkv(d["qkv_txt"], d["qkv_img"], d["qkv_ref"], d["pos"], w.split, w.theta, "bf16")
        o_dev, _ = jattn.fwd_bf16(q, k, v)
        path, kw = "bf16", dict(precise=False)
    else:
        q, k, v, sc = jattn.rope_qkv(d["qkv_txt"], d["qkv_img"], d["qkv_ref"], d["pos"], w.split, w.theta, "e4m3")
        o_dev, _ = jattn.fwd_fp8(q, k, v, sc)
    out = torch.empty(w.B, w.S, w.H, w.d, dtype=torch.bfloat16).pin_memory()
    for _ in range(2):
        torch.cuda._sleep(1000000)                 # work already queued on the caller's stream
        o_host = jattn.joint_attention(inp["qkv_txt"], inp["qkv_img"], inp["qkv_ref"], inp["pos"], w.split,
                                       w.theta, path=path, out=out, **kw)
        assert torch.equal(o_host, o_dev.cpu())
    assert jattn.device_status()[0] == jattn.OK


def test_cuda_graph_capture_and_replay(cuda_device):
    """The device entry points enqueue work only (no allocation, no host
    synchronisation), so the prologue + forward pair can be captured into a
    CUDA graph and replayed: the replay gives the eager result, also after
    the inputs change in place."""
    w = W.custom(B=1, H=2, d=128, S_txt=40, grid=12, n_ref=0)
    inp = W.make_inputs(w, 3)
    d = to_device(inp, cuda_device)
    q = torch.empty(w.B, w.H, w.S, w.d, dtype=torch.float16, device=cuda_device)
    bufs = (q, torch.empty_like(q), torch.empty_like(q), None)
    o = torch.empty(w.B, w.S, w.H, w.d, dtype=torch.bfloat16, device=cuda_device)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())

    def step():
        jattn.rope_qkv(d["qkv_txt"], d["qkv_img"], None, d["pos"], w.split, w.theta, "fp16", out=bufs, stream=s)
        jattn.fwd_bf16(bufs[0], bufs[1], bufs[2], o=o, stream=s)

    with torch.cuda.stream(s):
        step()                                            # warm-up: module loading, tensor maps
    torch.cuda.synchronize()
    eager = o.clone()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        step()
    o.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(o, eager)
    d["qkv_img"].mul_(0.5)                                # new inputs, same buffers
    g.replay()
    torch.cuda.synchronize()
    replayed = o.clone()
    with torch.cuda.stream(s):
        step()
    torch.cuda.synchronize()
    assert torch.equal(replayed, o)
    assert not torch.equal(replayed, eager)
    assert jattn.device_status()[0] == jattn.OK


@pytest.mark.slow
def test_long_sequence_and_wide_grid(cuda_device):
    """Sizes far from the workloads: S = 65613 (513 key tiles, ragged tail;
    256 sampled rows per head against the oracle) and B*H = 1600 small heads
    (grid.y = 1600, every row checked)."""
    w = W.custom(B=1, H=2, d=128, S_txt=77, grid=256, n_ref=0)            # S = 77 + 65536
    inp = W.make_inputs(w, 2)
    o, lse = _run_bf16(w, inp, cuda_device)
    rows = W.sample_rows(w, 256, 2)
    O, L = oracle.joint_attention(inp["qkv_txt"], inp["qkv_img"], None, inp["pos"], w.split, w.theta, rows=rows,
                                  workers=4)
    got = gather_rows(o, rows)
    assert rel_l2(got, O) <= BF16_REL_L2
    assert max_abs(got, O) <= BF16_MAX_ABS
    np.testing.assert_allclose(gather_lse(lse, rows), L, rtol=2e-3, atol=5e-3)
    w2 = W.custom(B=40, H=40, d=64, S_txt=5, grid=11, n_ref=0)           # S = 126 < one tile
    inp2 = W.make_inputs(w2, 3)
    o2, _ = _run_bf16(w2, inp2, cuda_device, want_lse=False)
    O2, _ = oracle.joint_attention(inp2["qkv_txt"], inp2["qkv_img"], None, inp2["pos"], w2.split, w2.theta,
                                   workers=4)
    got2 = gather_rows(o2, torch.arange(w2.S).expand(w2.B, w2.H, w2.S))
    assert rel_l2(got2, O2) <= BF16_REL_L2
    assert max_abs(got2, O2) <= BF16_MAX_ABS
    assert jattn.device_status()[0] == jattn.OK


def test_output_only_16_byte_aligned(cuda_device):
    """The epilogue writes 32-byte pieces of each output row when o is 32-byte
    aligned and 16-byte pieces otherwise (the C ABI asks only for 16): an o
    that starts 16 bytes into an allocation gets the same bits, for the plain
    forward and for the repair path, whose FP8 pass also reads the partial
    rows back from o."""
    w = W.custom(B=1, H=3, d=128, S_txt=40, grid=15, n_ref=0)        # S = 265
    inp = W.make_inputs(w, 5)
    d = to_device(inp, cuda_device)
    q, k, v, _ = jattn.rope_qkv(d["qkv_txt"], d["qkv_img"], d["qkv_ref"], d["pos"], w.split, w.theta, "fp16")
    n = w.B * w.S * w.H * w.d
    flat = torch.empty(n + 8, dtype=torch.bfloat16, device=cuda_device)
    o16 = flat[8:].view(w.B, w.S, w.H, w.d)                           # 16 bytes past a 256-byte boundary
    assert o16.data_ptr() % 32 == 16
    o_ref, _ = jattn.fwd_bf16(q, k, v)
    jattn.fwd_bf16(q, k, v, o=o16)
    torch.cuda.synchronize()
    assert torch.equal(o16, o_ref)
    args = (d["qkv_txt"], d["qkv_img"], d["qkv_ref"], d["pos"], w.split, w.theta)
    r_ref = jattn.fwd_fp8_repair(*args, rho=0.05)
    jattn.fwd_fp8_repair(*args, rho=0.05, o=o16)
    torch.cuda.synchronize()
    assert torch.equal(o16, r_ref)
    assert jattn.device_status()[0] == jattn.OK
