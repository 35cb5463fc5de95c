"""GPU parity of the block-sparse forward (jattn_fwd_block_sparse) against
oracle/block_sparse.py, through the C ABI.

* Selection: the kernel's kept key blocks (kv_list / kv_count) are sorted,
  distinct, always hold the largest share, and are a valid selection under
  the oracle's FP64 shares of the same operands: every block whose share
  clears tau / n_kb by a relative 1e-4 is kept, every block below it by
  1e-4 is dropped (in between, fp32 against fp64 may decide either way, so
  only validity is checked there).
* Output: against the oracle's block-sparse attention on the kernel's own
  selection, with the exact rotated operands: the BF16 path's bars.
* tau = 0 keeps every block and reproduces the dense forward bit for bit.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import block_sparse as bs
from diffusion_transformer_joint_jattn_b200 import jattn
from diffusion_transformer_joint_jattn_b200 import workloads as W
from parity_util import BF16_MAX_ABS, BF16_REL_L2, gather_lse, gather_rows, max_abs, rel_l2, to_device

pytestmark = pytest.mark.gpu


def _keep_mask(kv_list, kv_count, n_kb):
    B, H, n_qb, _ = kv_list.shape
    keep = np.zeros((B, H, n_qb, n_kb), dtype=bool)
    for b in range(B):
        for h in range(H):
            for I in range(n_qb):
                c = int(kv_count[b, h, I])
                lst = kv_list[b, h, I, :c]
                assert 1 <= c <= n_kb and np.all(np.diff(lst) > 0) and lst.min() >= 0 and lst.max() < n_kb
                keep[b, h, I, lst] = True
    return keep


def _run(w, inp, dev, tau):
    d = to_device(inp, dev)
    q, k, v, _ = jattn.rope_qkv(d["qkv_txt"], d["qkv_img"], d["qkv_ref"], d["pos"], w.split, w.theta, "fp16")
    o, lse, kl, kc = jattn.fwd_block_sparse(q, k, v, tau, want_lse=True, want_blocks=True)
    torch.cuda.synchronize()
    return (q, k, v), o, lse, kl.cpu().numpy(), kc.cpu().numpy()


def _check_selection(keep, q16, k16, tau):
    """keep [B, H, n_qb, n_kb] from the kernel; q16 / k16 the kernel's fp16
    operands as float64 [B, H, S, d]."""
    B, H, n_qb, n_kb = keep.shape
    for b in range(B):
        for h in range(H):
            sh = bs.block_shares(q16[b, h], k16[b, h])
            cut = tau / n_kb
            top = np.argmax(sh, axis=1)
            assert keep[b, h, np.arange(n_qb), top].all()
            must = sh >= cut * (1 + 1e-4)
            never = sh < cut * (1 - 1e-4)
            never[np.arange(n_qb), top] = False
            assert np.all(keep[b, h][must]), (b, h)
            assert not np.any(keep[b, h][never]), (b, h)


CASES = [
    dict(B=1, H=2, d=128, S_txt=44, grid=16, n_ref=0),      # S = 300: 2 query blocks, 3 key blocks (ragged)
    dict(B=2, H=2, d=128, S_txt=77, grid=9, n_ref=1),       # S = 239: one query block
    dict(B=1, H=3, d=64, S_txt=40, grid=24, n_ref=0),       # S = 616, d = 64
    dict(B=1, H=2, d=128, S_txt=128, grid=31, n_ref=1),     # S = 2050: 9 query blocks, 17 key blocks
]


@pytest.mark.parametrize("tau", [0.5, 1.0, 2.0])
@pytest.mark.parametrize("case", CASES, ids=lambda c: f"B{c['B']}H{c['H']}d{c['d']}t{c['S_txt']}g{c['grid']}r{c['n_ref']}")
def test_block_sparse_selection_and_parity(cuda_device, case, tau):
    w = W.custom(**case)
    inp = W.make_inputs(w, seed=17)
    (q, k, v), o, lse, kl, kc = _run(w, inp, cuda_device, tau)
    n_kb = jattn.n_blocks(w.S)
    keep = _keep_mask(kl, kc, n_kb)
    _check_selection(keep, q.double().cpu().numpy(), k.double().cpu().numpy(), tau)
    qe, ke, ve = oracle.rotated_qkv(inp["qkv_txt"], inp["qkv_img"], inp["qkv_ref"], inp["pos"], w.split, w.theta)
    O, L, _ = bs.block_sparse_attention(qe, ke, ve, tau, keep=keep)
    rows = torch.arange(w.S).expand(w.B, w.H, w.S)
    got = gather_rows(o, rows)
    r, m = rel_l2(got, O), max_abs(got, O)
    print(f"tau {tau} S {w.S}: kept {keep.mean():.2f} of the blocks, rel-L2 {r:.3e} max-abs {m:.3e}")
    assert r <= BF16_REL_L2
    assert m <= BF16_MAX_ABS
    np.testing.assert_allclose(gather_lse(lse, rows), L, rtol=0, atol=2e-3)
    assert jattn.device_status()[0] == jattn.OK


def test_tau_zero_is_the_dense_forward(cuda_device):
    w = W.custom(B=2, H=2, d=128, S_txt=64, grid=20, n_ref=0)      # S = 464
    inp = W.make_inputs(w, seed=3)
    (q, k, v), o, lse, kl, kc = _run(w, inp, cuda_device, 0.0)
    assert np.all(kc == jattn.n_blocks(w.S))
    o_dense, lse_dense = jattn.fwd_bf16(q, k, v, want_lse=True)
    torch.cuda.synchronize()
    assert torch.equal(o, o_dense)
    assert torch.equal(lse, lse_dense)


def test_large_tau_keeps_one_block(cuda_device):
    w = W.custom(B=1, H=2, d=128, S_txt=0, grid=24, n_ref=0)       # S = 576
    inp = W.make_inputs(w, seed=4)
    (q, k, v), o, _, kl, kc = _run(w, inp, cuda_device, 1e6)
    assert np.all(kc == 1)
    keep = _keep_mask(kl, kc, jattn.n_blocks(w.S))
    qe, ke, ve = oracle.rotated_qkv(None, inp["qkv_img"], None, inp["pos"], w.split, w.theta)
    O, _, _ = bs.block_sparse_attention(qe, ke, ve, 0.0, keep=keep)
    got = gather_rows(o, torch.arange(w.S).expand(w.B, w.H, w.S))
    assert rel_l2(got, O) <= BF16_REL_L2


@pytest.mark.slow
def test_block_sparse_full_length(cuda_device):
    """S = 16896 (512 text + 128 x 128 image tokens, the 2048 x 2048 shape),
    4 heads, tau = 1: 512 sampled rows per head against the oracle on the
    kernel's selection; fewer blocks than dense."""
    w = W.custom(B=1, H=4, d=128, S_txt=512, grid=128, n_ref=0)
    inp = W.make_inputs(w, seed=0)
    (q, k, v), o, lse, kl, kc = _run(w, inp, cuda_device, 1.0)
    n_kb = jattn.n_blocks(w.S)
    keep = _keep_mask(kl, kc, n_kb)
    _check_selection(keep, q.double().cpu().numpy(), k.double().cpu().numpy(), 1.0)
    assert keep.mean() < 0.9
    rows = W.sample_rows(w, 512, 1)
    qe, ke, ve = oracle.rotated_qkv(inp["qkv_txt"], inp["qkv_img"], None, inp["pos"], w.split, w.theta)
    O, L, _ = bs.block_sparse_attention(qe, ke, ve, 1.0, rows=rows.numpy(), keep=keep)
    got = gather_rows(o, rows)
    print(f"full length tau 1: kept {keep.mean():.3f}, rel-L2 {rel_l2(got, O):.3e} max-abs {max_abs(got, O):.3e}")
    assert rel_l2(got, O) <= BF16_REL_L2
    assert max_abs(got, O) <= BF16_MAX_ABS
    np.testing.assert_allclose(gather_lse(lse, rows), L, rtol=0, atol=2e-3)
    assert jattn.device_status()[0] == jattn.OK
