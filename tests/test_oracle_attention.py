"""Pins for the FP64 attention oracle (CPU only).

Each test checks the oracle against something it does not compute itself: a
closed form, an invariant of softmax attention or of rotary embeddings, a
special case with a known answer, or a 50-digit evaluation on a tiny input.
The docstring of each test names the mistakes it would catch.
"""
import json
import math
import os

import mpmath
import numpy as np
import pytest
import torch

import oracle
from diffusion_transformer_joint_jattn_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
rng = np.random.default_rng(1234)


def _streams(B, H, d, S_txt, grid, n_ref, seed=0):
    w = W.custom(B=B, H=H, d=d, S_txt=S_txt, grid=grid, n_ref=n_ref)
    return w, W.make_inputs(w, seed)


# ----------------------------------------------------------------- RoPE pins

def test_rope_closed_forms():
    """Golden closed forms: unit vectors at chosen positions land on
    (cos a, sin a) of the right channel pair with exactly-known frequencies
    (1, 0.1, 0.01).  Catches a wrong pair convention (half-split vs
    interleaved), axis offsets, the frequency exponent and the rotation sign."""
    fx = json.load(open(os.path.join(GOLDEN, "rope_closed_forms.json")))
    for c in fx["cases"]:
        d = c["d"]
        x = np.zeros((1, d))
        x[0, c["unit"]] = 1.0
        y = oracle.rope_rotate(x, np.array([c["pos"]]), c["split"], 10000.0)[0]
        a = c["angle"]
        i0, i1 = c["pair"]
        if c["unit"] == i0:
            want = (math.cos(a), math.sin(a))
        else:
            want = (-math.sin(a), math.cos(a))
        assert y[i0] == pytest.approx(want[0], abs=1e-14), c
        assert y[i1] == pytest.approx(want[1], abs=1e-14), c
        rest = np.delete(y, [i0, i1])
        assert np.all(rest == 0.0), c


def test_rope_identity_at_origin_and_text_positions():
    """Text tokens sit at (0,0,0): the rotation must be the identity."""
    x = rng.standard_normal((7, 128))
    y = oracle.rope_rotate(x, np.zeros((7, 3), np.int32), (16, 56, 56), 10000.0)
    assert np.array_equal(x, y)


def test_rope_preserves_pair_norms():
    """A rotation keeps the norm of every channel pair (catches a sign error
    that turns the rotation into a shear or reflection-with-scale)."""
    x = rng.standard_normal((64, 128))
    pos = rng.integers(0, 128, size=(64, 3))
    y = oracle.rope_rotate(x, pos, (16, 56, 56), 10000.0)
    nx = x[:, 0::2] ** 2 + x[:, 1::2] ** 2
    ny = y[:, 0::2] ** 2 + y[:, 1::2] ** 2
    np.testing.assert_allclose(ny, nx, rtol=1e-13)


def test_rope_relative_position_property():
    """q_rot(m) . k_rot(n) depends only on m - n on every axis: shifting both
    positions by the same (dt, dr, dc) leaves the dot product unchanged, and
    a different offset changes it."""
    q = rng.standard_normal(128)
    k = rng.standard_normal(128)
    split = (16, 56, 56)

    def dot(pm, pn):
        qr = oracle.rope_rotate(q[None], np.array([pm]), split, 1e4)[0]
        kr = oracle.rope_rotate(k[None], np.array([pn]), split, 1e4)[0]
        return qr @ kr

    base = dot([0, 3, 5], [1, 7, 2])
    assert dot([2, 13, 20], [3, 17, 17]) == pytest.approx(base, rel=1e-12)
    assert abs(dot([0, 3, 5], [1, 8, 2]) - base) > 1e-6


# ------------------------------------------------------------ attention pins

def test_softmax_rows_sum_to_one_and_lse():
    """With V = identity columns, O's rows are the softmax rows: they must sum
    to 1 and be non-negative; LSE must equal log(sum(exp(s))) computed with
    mpmath at 50 digits on the same logits."""
    S, d = 9, 8
    q = rng.standard_normal((S, d))
    k = rng.standard_normal((S, d))
    v = np.eye(S)
    o, lse = oracle.attention_rows(q, k, v, 1 / math.sqrt(d))
    np.testing.assert_allclose(o.sum(1), 1.0, rtol=0, atol=1e-14)
    assert (o >= 0).all()
    mpmath.mp.dps = 50
    for i in range(S):
        s = [mpmath.mpf(float(q[i] @ k[j])) / mpmath.sqrt(d) for j in range(S)]
        want = mpmath.log(mpmath.fsum(mpmath.exp(x) for x in s))
        assert lse[i] == pytest.approx(float(want), rel=1e-13)


def test_constant_values_give_constant_output():
    """If every value row is the same vector c, every output row is c whatever
    the logits (catches a missing or wrong normalisation by l)."""
    S, d = 33, 16
    q = 3 * rng.standard_normal((S, d))
    k = 3 * rng.standard_normal((S, d))
    c = rng.standard_normal(d)
    o, _ = oracle.attention_rows(q, k, np.tile(c, (S, 1)), 1 / math.sqrt(d))
    np.testing.assert_allclose(o, np.tile(c, (S, 1)), rtol=1e-13, atol=1e-13)


def test_single_dominant_logit_returns_that_value_row():
    """q parallel to k_j with a huge norm: the softmax is one-hot on j and the
    output is v_j (catches transposed operands or a query/key index swap)."""
    S, d, j = 12, 16, 7
    k = rng.standard_normal((S, d))
    v = rng.standard_normal((S, d))
    q = 1e3 * k[j][None] / np.linalg.norm(k[j])
    k_scaled = k.copy()
    k_scaled[j] *= 10.0
    o, _ = oracle.attention_rows(q, k_scaled, v, 1 / math.sqrt(d))
    np.testing.assert_allclose(o[0], v[j], rtol=0, atol=1e-12)


def test_single_token_sequence():
    """S = 1: softmax over one key is 1, so O = v and LSE = the one logit."""
    w, inp = _streams(1, 2, 64, 1, 0, 0)
    O, L = oracle.joint_attention(inp["qkv_txt"], None, None, inp["pos"], w.split)
    v = oracle.as_f64(inp["qkv_txt"])[:, 0, 2]          # [B, H, d]
    np.testing.assert_array_equal(O[:, :, 0], v)
    q = oracle.as_f64(inp["qkv_txt"])[:, 0, 0]
    k = oracle.as_f64(inp["qkv_txt"])[:, 0, 1]
    np.testing.assert_allclose(L[:, :, 0], (q * k).sum(-1) / 8.0, rtol=1e-14)


def test_softmax_scale_closed_form():
    """Two keys, logits a/sqrt(d) and 0, values 1 and 0: the output is the
    logistic function sigmoid(a/sqrt(d)).  Pins the 1/sqrt(d) scale (1/d or
    no scale fail) and the exp base."""
    d = 64
    q = np.zeros((1, d)); q[0, 3] = 2.5
    k = np.zeros((2, d)); k[0, 3] = 1.0
    v = np.zeros((2, d)); v[0, 0] = 1.0
    o, lse = oracle.attention_rows(q, k, v, 1 / math.sqrt(d))
    z = 2.5 / 8.0
    assert o[0, 0] == pytest.approx(1 / (1 + math.exp(-z)), rel=1e-15)
    assert lse[0] == pytest.approx(math.log(math.exp(z) + 1), rel=1e-15)


def test_zero_queries_average_values_and_lse_is_log_s():
    """q = 0: every logit is 0, so O is the mean of V and LSE = ln S."""
    S, d = 50, 32
    k = rng.standard_normal((S, d))
    v = rng.standard_normal((S, d))
    o, lse = oracle.attention_rows(np.zeros((3, d)), k, v, 1 / math.sqrt(d))
    np.testing.assert_allclose(o, np.tile(v.mean(0), (3, 1)), rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(lse, math.log(S), rtol=1e-15)


def test_joint_permutation_invariance():
    """Permuting keys, values and their positions together leaves every output
    row unchanged (catches rotating a key with the wrong token's position or
    pairing K and V rows of different tokens)."""
    w, inp = _streams(1, 2, 64, 8, 4, 1)
    O, _ = oracle.joint_attention(inp["qkv_txt"], inp["qkv_img"], inp["qkv_ref"], inp["pos"], w.split)
    S = w.S
    perm = torch.from_numpy(rng.permutation(S))
    qkv = torch.cat([inp["qkv_txt"], inp["qkv_img"], inp["qkv_ref"]], dim=1)
    O2, _ = oracle.joint_attention(qkv[:, perm], None, None, inp["pos"][perm], w.split)
    inv = torch.argsort(perm).numpy()
    np.testing.assert_allclose(O2[:, :, inv], O, rtol=1e-12, atol=1e-13)


def test_global_translation_invariance():
    """Adding the same (dt, dr, dc) to every position leaves O unchanged:
    RoPE scores depend on position differences only."""
    w, inp = _streams(1, 2, 64, 8, 4, 0)
    O, _ = oracle.joint_attention(inp["qkv_txt"], inp["qkv_img"], None, inp["pos"], w.split)
    pos2 = inp["pos"] + torch.tensor([3, 11, 5], dtype=torch.int32)
    O2, _ = oracle.joint_attention(inp["qkv_txt"], inp["qkv_img"], None, pos2, w.split)
    np.testing.assert_allclose(O2, O, rtol=1e-11, atol=1e-12)


def test_sampled_rows_equal_full_rows():
    """Row sampling only selects outputs: sampled rows equal the same rows of
    the full result, in order (catches rotating a sampled query with the
    position of its sample index instead of its token index)."""
    w, inp = _streams(1, 2, 64, 16, 8, 0)
    full, Lf = oracle.joint_attention(inp["qkv_txt"], inp["qkv_img"], None, inp["pos"], w.split)
    rows = W.sample_rows(w, n=20, seed=3)
    part, Lp = oracle.joint_attention(inp["qkv_txt"], inp["qkv_img"], None, inp["pos"], w.split,
                                      rows=rows)
    for b in range(w.B):
        for h in range(w.H):
            np.testing.assert_allclose(part[b, h], full[b, h, rows[b, h].numpy()], rtol=1e-13, atol=1e-14)
            np.testing.assert_allclose(Lp[b, h], Lf[b, h, rows[b, h].numpy()], rtol=1e-13)


def test_joint_order_and_stream_split():
    """Splitting one sequence into txt | img | ref streams at any boundary and
    joining them back is the identity (the assembly neither reorders nor
    drops tokens)."""
    w, inp = _streams(2, 3, 64, 5, 3, 1)
    q, k, v = oracle.joint_sequence(inp["qkv_txt"], inp["qkv_img"], inp["qkv_ref"])
    allq = torch.cat([inp["qkv_txt"], inp["qkv_img"], inp["qkv_ref"]], dim=1)
    np.testing.assert_array_equal(q, oracle.as_f64(allq[:, :, 0].permute(0, 2, 1, 3)))
    np.testing.assert_array_equal(k, oracle.as_f64(allq[:, :, 1].permute(0, 2, 1, 3)))
    np.testing.assert_array_equal(v, oracle.as_f64(allq[:, :, 2].permute(0, 2, 1, 3)))
    q2, _, _ = oracle.joint_sequence(allq[:, :2], allq[:, 2:], None)
    np.testing.assert_array_equal(q2, q)


def test_brute_force_50_digits_tiny():
    """Whole pipeline on a tiny joint sequence against a 50-digit mpmath
    evaluation (precision check of the float64 arithmetic)."""
    w = W.custom(B=1, H=1, d=8, S_txt=2, grid=2, n_ref=0, split=(2, 2, 4))
    inp = W.make_inputs(w, 5)
    O, L = oracle.joint_attention(inp["qkv_txt"], inp["qkv_img"], None, inp["pos"], w.split)
    mpmath.mp.dps = 50
    qkv = torch.cat([inp["qkv_txt"], inp["qkv_img"]], dim=1)[0].to(torch.float64).numpy()
    pos = inp["pos"].numpy()
    S, d = w.S, w.d

    def rot(x, p):
        out = [mpmath.mpf(0)] * d
        off = 0
        for a, n in enumerate(w.split):
            for i in range(n // 2):
                ang = p[a] * mpmath.power(10000, -mpmath.mpf(2 * i) / n)
                x0, x1 = mpmath.mpf(float(x[off + 2 * i])), mpmath.mpf(float(x[off + 2 * i + 1]))
                out[off + 2 * i] = x0 * mpmath.cos(ang) - x1 * mpmath.sin(ang)
                out[off + 2 * i + 1] = x0 * mpmath.sin(ang) + x1 * mpmath.cos(ang)
            off += n
        return out

    qs = [rot(qkv[i, 0, 0], pos[i]) for i in range(S)]
    ks = [rot(qkv[i, 1, 0], pos[i]) for i in range(S)]
    for i in range(S):
        s = [mpmath.fsum(qs[i][c] * ks[j][c] for c in range(d)) / mpmath.sqrt(d) for j in range(S)]
        e = [mpmath.exp(x) for x in s]
        l = mpmath.fsum(e)
        for c in range(d):
            oc = mpmath.fsum(e[j] * mpmath.mpf(float(qkv[j, 2, 0, c])) for j in range(S)) / l
            assert O[0, 0, i, c] == pytest.approx(float(oc), rel=1e-12, abs=1e-14)
        assert L[0, 0, i] == pytest.approx(float(mpmath.log(l)), rel=1e-13)
