"""GPU parity of the FP8 path (jattn_rope_qkv e4m3 + jattn_fwd_fp8) and of
the FP8 path with token repair at full size.

What is checked, and against what:
  * The quantised operands are checked bit-for-bit in test_gpu_rope.py.
  * The forward kernel is checked against the FP64 oracle run on the SAME
    dequantised operands with an exact softmax ("dequantised-operand
    oracle").  What separates the two is only the kernel's rounding of the
    probabilities P to e4m3 (3 mantissa bits, relative step 2^-4) and fp32
    accumulation: measured 2.5e-2 .. 2.8e-2 on every case, bar 3e-2.  (An
    emulation of the P rounding alone, with exact logits, gives 2.1e-2 ..
    2.7e-2 whatever headroom P keeps below 448, so the bar cannot go lower
    for e4m3 P.)
  * Closed-form cases (Q = 0, chosen per-block V scales): the output is the
    scale-weighted mean of V, exact up to the bf16 output rounding.
  * Against the exact FP64 result on the original bf16 inputs the error is
    the e4m3 format floor of Q/K/V, far above the 3e-2 target for plain FP8;
    each workload is held to 1.1 x its measured floor.
  * The FP8 path with the pages' token repair meets the 3e-2 target where
    the repair budget rho reaches it (i2i_2048_base at rho = 0.005,
    t2i_2048_base at 0.01, t2i_2048_distilled at 0.05) and is held to 1.1 x
    its measured error where it does not (rho = 0.005 on the two t2i
    workloads).
"""
import math

import numpy as np
import pytest
import torch

import oracle
from diffusion_transformer_joint_jattn_b200 import jattn
from diffusion_transformer_joint_jattn_b200 import workloads as W
from parity_util import FP8_REL_L2, gather_lse, gather_rows, rel_l2, to_device, workload_case

pytestmark = pytest.mark.gpu

KERNEL_VS_DEQUANT = 3e-2
# Plain FP8 against the exact result: the e4m3 floor of Q/K/V.  No-outlier
# d = 64 / 128 cases measure 5.3e-2 .. 5.6e-2; the workloads' floors below.
SMALL_VS_EXACT = 6.2e-2
WORKLOAD_VS_EXACT = {"t2i_2048_base": 1.1 * 9.48e-2, "t2i_2048_distilled": 1.1 * 2.83e-1,
                     "i2i_2048_base": 1.1 * 8.78e-2}


def _run(w, inp, dev):
    d = to_device(inp, dev)
    q8, k8, v8, sc = jattn.rope_qkv(d["qkv_txt"], d["qkv_img"], d["qkv_ref"], d["pos"], w.split, w.theta, "e4m3")
    o, lse = jattn.fwd_fp8(q8, k8, v8, sc, want_lse=True)
    torch.cuda.synchronize()
    return (q8, k8, v8, sc), o, lse


def _dequant(t8, sc):
    return oracle.dequantize_blocks(t8.cpu().view(torch.uint8).numpy(), sc.cpu().numpy())


SMALL = [
    dict(B=1, H=2, d=128, S_txt=64, grid=16, n_ref=0),     # S = 320
    dict(B=2, H=2, d=128, S_txt=77, grid=9, n_ref=1),      # S = 239, reference image
    dict(B=1, H=1, d=128, S_txt=1, grid=0, n_ref=0),       # S = 1
    dict(B=1, H=3, d=64, S_txt=32, grid=16, n_ref=0),      # d = 64 (64-byte swizzle)
    dict(B=1, H=1, d=128, S_txt=0, grid=23, n_ref=0),      # S = 529, no text
]


@pytest.mark.parametrize("case", SMALL, ids=lambda c: f"B{c['B']}H{c['H']}d{c['d']}t{c['S_txt']}g{c['grid']}r{c['n_ref']}")
def test_fp8_kernel_against_dequantised_operands(cuda_device, case):
    w = W.custom(**case)
    inp = W.make_inputs(w, seed=7)
    (q8, k8, v8, sc), o, lse = _run(w, inp, cuda_device)
    dq, dk, dv = (_dequant(t, sc[i]) for i, t in enumerate((q8, k8, v8)))
    O2, L2 = oracle.attention_on(dq, dk, dv)
    rows = torch.arange(w.S).expand(w.B, w.H, w.S)
    got = gather_rows(o, rows)
    r2 = rel_l2(got, O2)
    assert r2 <= KERNEL_VS_DEQUANT, r2
    np.testing.assert_allclose(gather_lse(lse, rows), L2, rtol=0, atol=1e-4)
    O, _ = oracle.joint_attention(inp["qkv_txt"], inp["qkv_img"], inp["qkv_ref"], inp["pos"], w.split, w.theta)
    r = rel_l2(got, O)
    print(f"{case}: rel-L2 vs dequantised-operand oracle {r2:.3e}, vs exact {r:.3e}")
    assert r <= SMALL_VS_EXACT
    assert jattn.device_status()[0] == jattn.OK


def test_fp8_with_qk_norm(cuda_device):
    """FP8 path with the fused query/key RMSNorm: against the oracle on the
    dequantised (normalised, rotated) operands, and against the exact result."""
    w = W.custom(B=2, H=2, d=128, S_txt=77, grid=9, n_ref=1)
    inp = W.make_inputs(w, seed=23)
    nw = W.norm_weights(128, 23)
    d = to_device(inp, cuda_device)
    q8, k8, v8, sc = jattn.rope_qkv(d["qkv_txt"], d["qkv_img"], d["qkv_ref"], d["pos"], w.split, w.theta, "e4m3",
                                    norm_w=nw.to(cuda_device))
    o, _ = jattn.fwd_fp8(q8, k8, v8, sc)
    torch.cuda.synchronize()
    dq, dk, dv = (_dequant(t, sc[i]) for i, t in enumerate((q8, k8, v8)))
    O2, _ = oracle.attention_on(dq, dk, dv)
    got = gather_rows(o, torch.arange(w.S).expand(w.B, w.H, w.S))
    O, _ = oracle.joint_attention(inp["qkv_txt"], inp["qkv_img"], inp["qkv_ref"], inp["pos"], w.split, w.theta,
                                  norm_w=nw, eps=1e-6)
    print(f"fp8 with query/key norm: vs dequantised-operand oracle {rel_l2(got, O2):.3e}, vs exact {rel_l2(got, O):.3e}")
    assert rel_l2(got, O2) <= KERNEL_VS_DEQUANT
    assert rel_l2(got, O) <= SMALL_VS_EXACT


@pytest.mark.parametrize("sv", [(1.0, 1.0), (1.0, 0.5), (0.5, 1.0), (1.0, 0.25), (2.0 ** -6, 1.0), (1.0, 0.125),
                                (3.0, 0.75)])
def test_fp8_value_scales_closed_form(cuda_device, sv):
    """Q = 0: every logit is 0, so O = (sum over tiles of s_v,j * sum of the
    tile's decoded V rows) / S.  Catches errors in the per-block V scale
    folding and the final rescale.  The scale ratios s_v,j / max s_v used here
    are powers of two (or 1/4 of 3), for which the rounded probabilities stay
    exact in e4m3; smaller or other ratios lose P precision by design."""
    S, d = 256, 128
    rng = np.random.default_rng(1)
    v8 = oracle.e4m3_encode(rng.standard_normal((1, 1, S, d)) * 40)
    k8 = oracle.e4m3_encode(rng.standard_normal((1, 1, S, d)) * 40)
    q8 = np.zeros((1, 1, S, d), np.uint8)
    sc = np.ones((3, 1, 1, 2), np.float32)
    sc[2, 0, 0] = sv
    t = lambda a: torch.from_numpy(a).to(cuda_device).view(torch.float8_e4m3fn)
    o, lse = jattn.fwd_fp8(t(q8), t(k8), t(v8), torch.from_numpy(sc).to(cuda_device), want_lse=True)
    torch.cuda.synchronize()
    vd = oracle.e4m3_decode(v8)[0, 0]
    want = (vd[:128].sum(0) * sv[0] + vd[128:].sum(0) * sv[1]) / S
    got = o[0, 0, 0].float().cpu().numpy()
    bf16_step = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(want), 1e-30))) - 7)
    tol = bf16_step + 1e-5 * np.abs(want) + 1e-6
    assert np.all(np.abs(got - want) <= tol), np.max(np.abs(got - want) / tol)
    assert abs(lse[0, 0, 0].item() - math.log(S)) < 1e-5


@pytest.mark.slow
@pytest.mark.parametrize("name", ["t2i_2048_base", "t2i_2048_distilled", "i2i_2048_base"])
def test_workload_fp8_sampled_rows(cuda_device, name):
    w, inp, rows, O, L = workload_case(name)
    (q8, k8, v8, sc), o, lse = _run(w, inp, cuda_device)
    got = gather_rows(o, rows)
    # dequantised-operand oracle, one head at a time, on the sampled rows
    O2 = np.empty_like(O)
    for b in range(w.B):
        for h in range(w.H):
            qs = oracle.dequantize_blocks(q8[b:b + 1, h:h + 1].cpu().view(torch.uint8).numpy(), sc[0, b:b + 1, h:h + 1].cpu().numpy())[0, 0]
            ks = oracle.dequantize_blocks(k8[b:b + 1, h:h + 1].cpu().view(torch.uint8).numpy(), sc[1, b:b + 1, h:h + 1].cpu().numpy())[0, 0]
            vs = oracle.dequantize_blocks(v8[b:b + 1, h:h + 1].cpu().view(torch.uint8).numpy(), sc[2, b:b + 1, h:h + 1].cpu().numpy())[0, 0]
            O2[b, h], _ = oracle.attention_rows(qs[rows[b, h].numpy()], ks, vs, 1 / math.sqrt(w.d))
    r2, r = rel_l2(got, O2), rel_l2(got, O)
    print(f"{name}: rel-L2 vs dequantised-operand oracle {r2:.3e}, vs exact (format floor) {r:.3e}")
    assert r2 <= KERNEL_VS_DEQUANT
    assert r <= WORKLOAD_VS_EXACT[name]
    assert jattn.device_status()[0] == jattn.OK


# (workload, rho, bar against the exact result): FP8_REL_L2 where the repair
# budget reaches it, else 1.1 x the measured error at that budget.
REPAIR_CASES = [("t2i_2048_base", 0.005, 1.1 * 3.23e-2), ("t2i_2048_base", 0.01, FP8_REL_L2),
                ("t2i_2048_distilled", 0.005, 1.1 * 1.83e-1), ("t2i_2048_distilled", 0.05, FP8_REL_L2),
                ("i2i_2048_base", 0.005, FP8_REL_L2)]


@pytest.mark.slow
@pytest.mark.parametrize("name,rho,bar", REPAIR_CASES, ids=lambda x: str(x))
def test_workload_fp8_repair_against_exact(cuda_device, name, rho, bar):
    """The FP8 path with token repair at full size in the bench's launch
    configuration, against the exact FP64 attention on 8 heads x 512 sampled
    rows (the oracle rotates each checked head's keys in FP64)."""
    w = W.BY_NAME[name]
    inp = W.make_inputs(w, 0)
    d = to_device(inp, cuda_device)
    o = jattn.fwd_fp8_repair(d["qkv_txt"], d["qkv_img"], d["qkv_ref"], d["pos"], w.split, w.theta, rho=rho)
    torch.cuda.synchronize()
    assert jattn.device_status()[0] == jattn.OK
    o = o.cpu()
    qkv = torch.cat([t for t in (inp["qkv_txt"], inp["qkv_img"], inp["qkv_ref"]) if t is not None], dim=1)
    pos = inp["pos"].numpy()
    rows = W.sample_rows(w, 512, 3)
    num = den = 0.0
    for bh in range(0, w.B * w.H, max(1, w.B * w.H // 8)):
        b, h = divmod(bh, w.H)
        x = qkv[b, :, :, h].to(torch.float64).numpy()
        k = oracle.rope_rotate(x[:, 1], pos, w.split, w.theta)
        rr = rows[b, h].numpy()
        q = oracle.rope_rotate(x[rr, 0], pos[rr], w.split, w.theta)
        O, _ = oracle.attention_rows(q, k, x[:, 2], 1 / math.sqrt(w.d))
        num += np.sum((o[b, rr, h].double().numpy() - O) ** 2)
        den += np.sum(O ** 2)
    r = math.sqrt(num / den)
    print(f"{name} rho {rho}: FP8 with repair vs exact {r:.4e} (bar {bar:.3e})")
    assert r <= bar
