"""Pins for the oracle of the FP8 attention with token repair (CPU only).

The repaired attention takes, for the n = ceil(rho * S) tokens with the
largest |k|^2 + |v|^2 of each head, the exact key, value and logit, and the
dequantised e4m3 ones for every other token, under one softmax.  The tests
reduce it to independently pinned cases (nothing repaired, everything
repaired), check the split-and-merge decomposition that a two-pass kernel
uses, and pin the selection and the count by hand.
"""
import math

import numpy as np
import pytest

import oracle
from diffusion_transformer_joint_jattn_b200 import workloads as W

rng = np.random.default_rng(5)


def test_selection_by_hand():
    """Largest scores first, ties to the lower index, result in index
    order.  Catches an ascending sort, an unstable tie-break and an
    unsorted result."""
    assert oracle.repair_select(np.array([3.0, 1.0, 3.0, 2.0, 5.0]), 2).tolist() == [0, 4]
    assert oracle.repair_select(np.array([3.0, 1.0, 3.0, 2.0, 5.0]), 3).tolist() == [0, 2, 4]
    assert oracle.repair_select(np.array([1.0, 1.0, 1.0, 1.0]), 2).tolist() == [0, 1]
    assert oracle.repair_select(np.array([1.0, 2.0]), 0).tolist() == []


@pytest.mark.parametrize("S,rho,n", [(16896, 0.005, 85), (200, 0.005, 1), (1000, 0.005, 5), (7, 0.0, 0),
                                     (7, 1.0, 7), (33280, 0.005, 167), (10, 0.30000001192092896, 3),
                                     (100, 1e-6, 0)])
def test_repair_count(S, rho, n):
    """n = ceil(rho * S - 1e-3): 84.48 -> 85, exactly 5.0 -> 5 (not 6), the
    float32 value of 0.3 on 10 tokens -> 3 (not 4)."""
    assert oracle.repair_count(S, rho) == n


def test_scores_are_rotation_invariant_squared_norms():
    """|k|^2 + |v|^2 of a hand row, and invariance under the (norm-
    preserving) rotary embedding: the score may be taken before or after
    RoPE."""
    assert oracle.repair_scores(np.array([[3.0, 4.0]]), np.array([[1.0, 2.0]]))[0] == 30.0
    k = rng.standard_normal((300, 128))
    v = rng.standard_normal((300, 128))
    pos = np.stack([rng.integers(0, 3, 300), rng.integers(0, 64, 300), rng.integers(0, 64, 300)], 1)
    kr = oracle.rope_rotate(k, pos, (16, 56, 56), 10000.0)
    np.testing.assert_allclose(oracle.repair_scores(kr, v), oracle.repair_scores(k, v), rtol=1e-13)


def _case(seed=3):
    w = W.custom(B=1, H=2, d=64, S_txt=10, grid=7, n_ref=0)
    inp = W.make_inputs(w, seed)
    q, k, v = oracle.rotated_qkv(inp["qkv_txt"], inp["qkv_img"], None, inp["pos"], w.split, w.theta)
    deq = lambda x: oracle.dequantize_blocks(*oracle.quantize_blocks(x.astype(np.float32)))
    return w, inp, (q, k, v), (deq(q), deq(k), deq(v))


def test_everything_repaired_is_the_exact_attention():
    w, inp, (q, k, v), (qd, kd, vd) = _case()
    allr = np.broadcast_to(np.arange(w.S), (w.B, w.H, w.S))
    O, L = oracle.repaired_attention(q, k, v, qd, kd, vd, allr)
    O2, L2 = oracle.joint_attention(inp["qkv_txt"], inp["qkv_img"], None, inp["pos"], w.split, w.theta)
    np.testing.assert_allclose(O, O2, rtol=0, atol=1e-13)
    np.testing.assert_allclose(L, L2, rtol=0, atol=1e-13)


def test_nothing_repaired_is_the_dequantised_operand_attention():
    w, inp, (q, k, v), (qd, kd, vd) = _case()
    none = np.zeros((w.B, w.H, 0), dtype=np.int64)
    O, L = oracle.repaired_attention(q, k, v, qd, kd, vd, none)
    O2, L2 = oracle.attention_on(qd, kd, vd)
    np.testing.assert_allclose(O, O2, rtol=0, atol=1e-13)
    np.testing.assert_allclose(L, L2, rtol=0, atol=1e-13)


def test_split_and_merge_decomposition():
    """Attention over the non-repaired keys (dequantised) and over the
    repaired keys (exact), merged with weights exp(LSE_part - LSE), equals
    the one-softmax definition: the identity the two-pass kernel relies on.
    Catches a repaired key counted twice or a wrong normalisation."""
    w, inp, (q, k, v), (qd, kd, vd) = _case(8)
    scale = 1 / math.sqrt(w.d)
    for h in range(w.H):
        sc = oracle.repair_scores(k[0, h], v[0, h])
        R = oracle.repair_select(sc, 6)
        keep = np.setdiff1d(np.arange(w.S), R)
        O, L = oracle.repaired_attention_rows(q[0, h], qd[0, h], k[0, h], v[0, h], kd[0, h], vd[0, h], R, scale)
        Oa, La = oracle.attention_rows(qd[0, h], kd[0, h][keep], vd[0, h][keep], scale)
        Ob, Lb = oracle.attention_rows(q[0, h], k[0, h][R], v[0, h][R], scale)
        Lm = np.logaddexp(La, Lb)
        Om = np.exp(La - Lm)[:, None] * Oa + np.exp(Lb - Lm)[:, None] * Ob
        np.testing.assert_allclose(O, Om, rtol=0, atol=1e-13)
        np.testing.assert_allclose(L, Lm, rtol=0, atol=1e-13)


def test_dominant_repaired_key_returns_its_exact_value():
    """One repaired key whose exact logit exceeds every other by ~50: the
    output is its exact value row, not the dequantised one."""
    S, d = 40, 64
    q = rng.standard_normal((1, d))
    k = rng.standard_normal((S, d)) * 0.1
    v = rng.standard_normal((S, d))
    k[17] = q[0] * 50 / (q[0] @ q[0]) * math.sqrt(d)        # logit 50 after the 1/sqrt(d) scale
    kd, vd = k * (1 + 1e-2), v + 0.05                         # stand-in "dequantised" operands
    O, L = oracle.repaired_attention_rows(q, q, k, v, kd, vd, [17], 1 / math.sqrt(d))
    np.testing.assert_allclose(O[0], v[17], rtol=0, atol=1e-15 + 1e-18 * S)
    assert L[0] == pytest.approx(50.0, abs=1e-12)
