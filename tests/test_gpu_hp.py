"""GPU parity of the high-precision 16-bit path (jattn_rope_qkv_hp +
jattn_fwd_bf16_hp) against the FP64 oracle, through the C ABI.

The bars are the BF16 path's, unrelaxed: rel-L2 <= 5e-3 and max-abs <= 2e-2
over the sampled rows (every row for the small cases, 4096 rows per (b, h)
on the full-size workloads).  The plain fp16-operand path sits above the
max-abs bar on the outlier workloads (test_gpu_attention.py measures that
floor); this path restores the fp16 rounding residual of the 4 channel
pairs per head with the largest max|q_pair| * max|k_pair| and scales blocks
that would leave the fp16 range instead of saturating them.

Pieces checked on their own:
  * prologue: for ordinary inputs the same fp16 values as the plain
    prologue, bit for bit, with every range scale 1;
  * correction rows: the hi parts equal the stored q / k values of a valid
    top-4 channel-pair selection (checked against the oracle's statistic),
    hi + lo equals the exact rotated value to fp32 precision;
  * range: blocks past 65504 are scaled by powers of two, the device status
    stays clear, and the attention still meets the bars.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from diffusion_transformer_joint_jattn_b200 import jattn
from diffusion_transformer_joint_jattn_b200 import workloads as W
from parity_util import (BF16_MAX_ABS, BF16_REL_L2, gather_lse, gather_rows, max_abs, rel_l2, to_device,
                         workload_case)

pytestmark = pytest.mark.gpu


def _run_hp(w, inp, dev, norm_w=None, want_lse=True):
    d = to_device(inp, dev)
    nw = None if norm_w is None else norm_w.to(dev)
    ops = jattn.rope_qkv_hp(d["qkv_txt"], d["qkv_img"], d["qkv_ref"], d["pos"], w.split, w.theta, norm_w=nw)
    o, lse = jattn.fwd_bf16_hp(*ops, want_lse=want_lse)
    torch.cuda.synchronize()
    return ops, o, lse


CASES = [
    dict(B=1, H=2, d=64, S_txt=32, grid=16, n_ref=0),                                   # tiny, S = 288
    dict(B=1, H=1, d=128, S_txt=1, grid=0, n_ref=0),                                    # S = 1
    dict(B=2, H=2, d=128, S_txt=77, grid=9, n_ref=1),                                   # S = 239, reference
    dict(B=1, H=3, d=64, S_txt=3, grid=11, n_ref=0),                                    # S = 124 < a tile
    dict(B=1, H=2, d=128, S_txt=129, grid=16, n_ref=0, outlier_frac=0.01, outlier_mult=8.0),   # S = 385
    dict(B=1, H=2, d=128, S_txt=40, grid=20, n_ref=0, outlier_frac=0.02, outlier_mult=16.0),   # S = 440
]


def _id(c):
    return f"B{c['B']}H{c['H']}d{c['d']}t{c['S_txt']}g{c['grid']}r{c['n_ref']}o{c.get('outlier_frac', 0)}"


@pytest.mark.parametrize("case", CASES, ids=_id)
def test_hp_attention_every_row(cuda_device, case):
    w = W.custom(**case)
    inp = W.make_inputs(w, seed=5)
    _, o, lse = _run_hp(w, inp, cuda_device)
    O, L = oracle.joint_attention(inp["qkv_txt"], inp["qkv_img"], inp["qkv_ref"], inp["pos"], w.split, w.theta)
    rows = torch.arange(w.S).expand(w.B, w.H, w.S)
    got = gather_rows(o, rows)
    r, m = rel_l2(got, O), max_abs(got, O)
    print(f"{_id(case)}: rel-L2 {r:.3e} max-abs {m:.3e}")
    assert r <= BF16_REL_L2
    assert m <= BF16_MAX_ABS
    np.testing.assert_allclose(gather_lse(lse, rows), L, rtol=2e-4, atol=2e-3)
    assert jattn.device_status()[0] == jattn.OK


def test_hp_prologue_equals_plain_prologue(cuda_device):
    """Ordinary inputs: every range scale is 1 and q, k, v are the plain
    fp16 prologue's values bit for bit (the same rounding helpers)."""
    w = W.custom(B=2, H=3, d=128, S_txt=77, grid=9, n_ref=1, outlier_frac=0.01, outlier_mult=8.0)
    inp = W.make_inputs(w, seed=2)
    d = to_device(inp, cuda_device)
    q, k, v, sc, qc, kc = jattn.rope_qkv_hp(d["qkv_txt"], d["qkv_img"], d["qkv_ref"], d["pos"], w.split, w.theta)
    q0, k0, v0, _ = jattn.rope_qkv(d["qkv_txt"], d["qkv_img"], d["qkv_ref"], d["pos"], w.split, w.theta, "fp16")
    torch.cuda.synchronize()
    assert torch.all(sc == 1.0)
    assert torch.equal(q.view(torch.int16), q0.view(torch.int16))
    assert torch.equal(k.view(torch.int16), k0.view(torch.int16))
    assert torch.equal(v.view(torch.int16), v0.view(torch.int16))
    assert jattn.device_status()[0] == jattn.OK


def _columns_of(x16, hi):
    """Channel of x16 [S, d] equal to each column of hi [S, 8] on every token."""
    cols = []
    for c in range(hi.shape[1]):
        match = [ch for ch in range(x16.shape[1]) if torch.equal(x16[:, ch].view(torch.int16),
                                                                   hi[:, c].view(torch.int16))]
        assert len(match) >= 1, f"correction column {c} matches no stored channel"
        cols.append(match[0])
    return cols


@pytest.mark.parametrize("norm", [False, True])
def test_hp_correction_rows(cuda_device, norm):
    """qc = [hi | lo] and kc = [lo | hi] of 4 channel pairs per (b, h):
    hi equals the stored fp16 value, the pairs are a valid top-4 of the
    oracle's max|q_pair|^2 * max|k_pair|^2, and hi + lo is the exact rotated
    value to fp32 accuracy."""
    w = W.custom(B=1, H=3, d=128, S_txt=20, grid=15, n_ref=0, outlier_frac=0.02, outlier_mult=16.0)   # S = 245
    inp = W.make_inputs(w, seed=11)
    nw = W.norm_weights(w.d, 11) if norm else None
    d = to_device(inp, cuda_device)
    q, k, v, sc, qc, kc = jattn.rope_qkv_hp(d["qkv_txt"], d["qkv_img"], d["qkv_ref"], d["pos"], w.split, w.theta,
                                            norm_w=None if nw is None else nw.to(cuda_device))
    torch.cuda.synchronize()
    qe, ke, _ = oracle.rotated_qkv(inp["qkv_txt"], inp["qkv_img"], inp["qkv_ref"], inp["pos"], w.split, w.theta,
                                   norm_w=nw, eps=1e-6)
    q, k, qc, kc = q.cpu(), k.cpu(), qc.cpu(), kc.cpu()
    for h in range(w.H):
        chans = _columns_of(q[0, h], qc[0, h, :, :8])
        assert chans == _columns_of(k[0, h], kc[0, h, :, 8:])
        pairs = sorted(set(c // 2 for c in chans))
        assert len(pairs) == 4 and chans == [c for p in pairs for c in (2 * p, 2 * p + 1)]
        mq = (qe[0, h, :, 0::2] ** 2 + qe[0, h, :, 1::2] ** 2).max(0)
        mk = (ke[0, h, :, 0::2] ** 2 + ke[0, h, :, 1::2] ** 2).max(0)
        prod = mq * mk
        rest = np.delete(prod, pairs)
        assert prod[pairs].min() >= rest.max() * (1 - 1e-5)
        for x_exact, hi, lo in ((qe[0, h][:, chans], qc[0, h, :, :8], qc[0, h, :, 8:]),
                                (ke[0, h][:, chans], kc[0, h, :, 8:], kc[0, h, :, :8])):
            rec = hi.double().numpy() + lo.double().numpy()
            norm2 = np.repeat(np.sqrt(x_exact[:, 0::2] ** 2 + x_exact[:, 1::2] ** 2), 2, axis=1)
            # fp32 rotation: 2^-20 of the pair norm; with the RMSNorm the fp32
            # sum of squares behind the row factor adds up to 2^-18
            tol = (2.0 ** -18 if norm else 2.0 ** -20) * norm2 + 2.0 ** -22 * np.abs(x_exact) + 1e-30
            assert np.all(np.abs(rec - x_exact) <= tol)
    assert jattn.device_status()[0] == jattn.OK


def test_hp_range_scaling(cuda_device):
    """Q x 2^12 and K x 2^-12 (the logits are unchanged, the rotated Q
    outlier channel reaches ~1e5) and V x 2^15 (values past 65504): the
    blocks are stored scaled, nothing saturates, JATTN_DEV_RANGE stays
    clear, and the output matches the oracle at the BF16 bars relative to
    the V scale."""
    w = W.custom(B=1, H=2, d=128, S_txt=64, grid=16, n_ref=0, outlier_frac=0.01, outlier_mult=8.0)   # S = 320
    inp = W.make_inputs(w, seed=8)
    for key in ("qkv_txt", "qkv_img"):
        t = inp[key].float()
        t[:, :, 0] *= 2.0 ** 12
        t[:, :, 1] *= 2.0 ** -12
        t[:, :, 2] *= 2.0 ** 15
        inp[key] = t.to(torch.bfloat16)                 # powers of two: exact in bf16
    jattn.device_status(clear=True)
    (q, k, v, sc, qc, kc), o, lse = _run_hp(w, inp, cuda_device)
    assert sc[0].max().item() > 1.0 and sc[2].max().item() > 1.0
    assert torch.all(torch.isfinite(q.float())) and torch.all(torch.isfinite(v.float()))
    code, bits = jattn.device_status(clear=True)
    assert code == jattn.OK and bits == 0
    O, L = oracle.joint_attention(inp["qkv_txt"], inp["qkv_img"], None, inp["pos"], w.split, w.theta)
    rows = torch.arange(w.S).expand(w.B, w.H, w.S)
    got = gather_rows(o, rows) / 2.0 ** 15
    O = O / 2.0 ** 15
    assert rel_l2(got, O) <= BF16_REL_L2
    assert max_abs(got, O) <= BF16_MAX_ABS
    np.testing.assert_allclose(gather_lse(lse, rows), L, rtol=2e-4, atol=2e-3)


def test_hp_with_qk_norm(cuda_device):
    w = W.custom(B=2, H=2, d=128, S_txt=77, grid=9, n_ref=1, outlier_frac=0.01, outlier_mult=8.0)
    inp = W.make_inputs(w, seed=14)
    nw = W.norm_weights(w.d, 14)
    _, o, _ = _run_hp(w, inp, cuda_device, norm_w=nw, want_lse=False)
    O, _ = oracle.joint_attention(inp["qkv_txt"], inp["qkv_img"], inp["qkv_ref"], inp["pos"], w.split, w.theta,
                                  norm_w=nw, eps=1e-6)
    got = gather_rows(o, torch.arange(w.S).expand(w.B, w.H, w.S))
    assert rel_l2(got, O) <= BF16_REL_L2
    assert max_abs(got, O) <= BF16_MAX_ABS


def test_hp_graph_capture(cuda_device):
    """The four launches of the path enqueue work only: captured into a CUDA
    graph and replayed they give the eager result."""
    w = W.custom(B=1, H=2, d=128, S_txt=40, grid=12, n_ref=0, outlier_frac=0.01, outlier_mult=8.0)
    d = to_device(W.make_inputs(w, 3), cuda_device)
    B, H, S, dd = w.B, w.H, w.S, w.d
    q = torch.empty(B, H, S, dd, dtype=torch.float16, device=cuda_device)
    ops = (q, torch.empty_like(q), torch.empty_like(q),
           torch.empty(3, B, H, jattn.n_blocks(S), dtype=torch.float32, device=cuda_device),
           torch.empty(B, H, S, jattn.CORR_COLS, dtype=torch.float16, device=cuda_device),
           torch.empty(B, H, S, jattn.CORR_COLS, dtype=torch.float16, device=cuda_device))
    ws = torch.empty(jattn.rope_qkv_hp_workspace_bytes(B, H, w.S_txt, w.S_img, w.S_ref, dd), dtype=torch.uint8,
                     device=cuda_device)
    o = torch.empty(B, S, H, dd, dtype=torch.bfloat16, device=cuda_device)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())

    def step():
        jattn.rope_qkv_hp(d["qkv_txt"], d["qkv_img"], None, d["pos"], w.split, w.theta, out=ops, workspace=ws,
                          stream=s)
        jattn.fwd_bf16_hp(*ops, o=o, stream=s)

    with torch.cuda.stream(s):
        step()
    torch.cuda.synchronize()
    eager = o.clone()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        step()
    o.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(o, eager)
    assert jattn.device_status()[0] == jattn.OK


@pytest.mark.slow
@pytest.mark.parametrize("name", ["t2i_1024_base", "t2i_2048_base", "i2i_2048_base"])
def test_workload_bf16_hp_sampled_rows(cuda_device, name):
    """The BF16 workloads at full size in the bench's launch configuration,
    4096 sampled rows per (b, h): the stated bars, unrelaxed."""
    w, inp, rows, O, L = workload_case(name)
    _, o, lse = _run_hp(w, inp, cuda_device)
    got = gather_rows(o, rows)
    r, m = rel_l2(got, O), max_abs(got, O)
    print(f"{name} (high-precision path): rel-L2 {r:.3e} max-abs {m:.3e}")
    assert r <= BF16_REL_L2
    assert m <= BF16_MAX_ABS
    np.testing.assert_allclose(gather_lse(lse, rows), L, rtol=2e-4, atol=2e-3)
    assert jattn.device_status()[0] == jattn.OK
