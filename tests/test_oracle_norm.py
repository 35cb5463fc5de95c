"""Pins for the oracle's query/key RMS normalisation (CPU only).

The normalisation is x -> w * x / sqrt(mean(x^2) + eps) over the d channels
of one (token, head), applied to Q and K before the rotation, with one weight
vector per stream and per Q/K.  Each test checks it against something the
oracle does not compute itself (hand arithmetic, a closed form, an
invariant); the docstrings name the mistakes each one catches.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from diffusion_transformer_joint_jattn_b200 import workloads as W

rng = np.random.default_rng(77)


def test_rms_norm_hand_example():
    """x = (3, 4), w = 1, eps = 0: mean(x^2) = 25/2, so x / sqrt(12.5) =
    (3, 4) * sqrt(2) / 5 = (0.6 sqrt 2, 0.8 sqrt 2).  Catches sum instead of
    mean, a missing square root, and RMS vs standard deviation (the mean here
    is 3.5, not 0)."""
    y = oracle.rms_norm(np.array([3.0, 4.0]), np.ones(2), 0.0)
    assert y[0] == pytest.approx(0.6 * math.sqrt(2.0), rel=1e-15)
    assert y[1] == pytest.approx(0.8 * math.sqrt(2.0), rel=1e-15)


@pytest.mark.parametrize("c,eps", [(0.5, 1e-6), (-3.0, 1e-6), (1e-3, 1e-6), (2.0, 0.25)])
def test_rms_norm_constant_vector_with_eps(c, eps):
    """x = c * 1 (d = 128): every output is c / sqrt(c^2 + eps).  Catches eps
    added outside the square root or after it, and a dropped sign."""
    y = oracle.rms_norm(np.full(128, c), np.ones(128), eps)
    np.testing.assert_allclose(y, c / math.sqrt(c * c + eps), rtol=1e-14)


def test_rms_norm_invariants():
    """eps = 0, w = 1: unit RMS output; invariant to a positive scale of x
    and odd in x.  With weights: the weight multiplies channel-wise after the
    normalisation (w * norm(x), not norm(w * x))."""
    x = rng.standard_normal((5, 7, 128)) * rng.uniform(0.1, 30.0, (5, 7, 1))
    y = oracle.rms_norm(x, np.ones(128), 0.0)
    np.testing.assert_allclose(np.mean(y * y, axis=-1), 1.0, rtol=1e-13)
    np.testing.assert_allclose(oracle.rms_norm(7.5 * x, np.ones(128), 0.0), y, rtol=1e-13)
    np.testing.assert_allclose(oracle.rms_norm(-x, np.ones(128), 0.0), -y, rtol=1e-15)
    w = rng.uniform(-2.0, 2.0, 128)
    np.testing.assert_allclose(oracle.rms_norm(x, w, 0.0), y * w, rtol=1e-13)
    # a non-uniform weight changes the result if it were applied before the norm
    assert not np.allclose(oracle.rms_norm(x * w, np.ones(128), 0.0), y * w)


def test_norm_precedes_rotation():
    """A unit vector in channel 0 of Q at time position 1: the first t-axis
    pair turns by exactly 1 rad (frequency theta^0).  Normalising first gives
    channel 0..1 = w0 sqrt(d) (cos 1, sin 1); rotating first would give
    sqrt(d) (w0 cos 1, w1 sin 1).  With w0 != w1 the two orders differ."""
    d = 128
    w = W.custom(B=1, H=1, d=d, S_txt=0, grid=1, n_ref=1)         # S = 2: img (0,0,0), ref (1,0,0)
    qkv_img = torch.zeros(1, 1, 3, 1, d)
    qkv_ref = torch.zeros(1, 1, 3, 1, d)
    qkv_ref[0, 0, 0, 0, 0] = 1.0
    qkv_ref[0, 0, 1, 0, 0] = 1.0
    qkv_img[0, 0, :2, 0, :] = 1.0
    nw = torch.ones(3, 2, d, dtype=torch.float32)
    nw[2, 0, 0], nw[2, 0, 1] = 2.0, 0.5                          # ref stream, Q weights
    nw[2, 1, 0], nw[2, 1, 1] = 3.0, 0.25                         # ref stream, K weights
    pos = W.joint_positions(0, 1, 1)
    q, k, _ = oracle.rotated_qkv(None, qkv_img, qkv_ref, pos, w.split, w.theta, norm_w=nw, eps=0.0)
    r = math.sqrt(d)
    assert q[0, 0, 1, 0] == pytest.approx(2.0 * r * math.cos(1.0), rel=1e-14)
    assert q[0, 0, 1, 1] == pytest.approx(2.0 * r * math.sin(1.0), rel=1e-14)
    assert k[0, 0, 1, 0] == pytest.approx(3.0 * r * math.cos(1.0), rel=1e-14)
    assert k[0, 0, 1, 1] == pytest.approx(3.0 * r * math.sin(1.0), rel=1e-14)
    assert np.all(q[0, 0, 1, 2:] == 0.0)
    np.testing.assert_allclose(q[0, 0, 0], 1.0, rtol=1e-15)       # img token: all-ones row, RMS 1, w = 1


def test_norm_weights_per_stream_and_qk():
    """Stream s and Q/K index j scale by their own weight: constant weights
    (s + 1) * (j + 1) / 2 must show up as that factor on unit-RMS rows.  V is
    never touched.  Catches swapped stream or Q/K indices."""
    w = W.custom(B=2, H=3, d=64, S_txt=5, grid=3, n_ref=1)
    inp = W.make_inputs(w, 4)
    nw = torch.empty(3, 2, 64)
    for s in range(3):
        for j in range(2):
            nw[s, j] = (s + 1) * (j + 1) / 2
    out = oracle.qk_norm_streams(inp["qkv_txt"], inp["qkv_img"], inp["qkv_ref"], nw, 0.0)
    for s, (src, got) in enumerate(zip((inp["qkv_txt"], inp["qkv_img"], inp["qkv_ref"]), out)):
        x = src.to(torch.float64).numpy()
        for j in range(2):
            rms = np.sqrt(np.mean(got[:, :, j] ** 2, axis=-1))
            np.testing.assert_allclose(rms, (s + 1) * (j + 1) / 2, rtol=1e-13)
            # direction preserved
            cos = np.sum(got[:, :, j] * x[:, :, j], -1) / np.linalg.norm(got[:, :, j], axis=-1) / np.linalg.norm(x[:, :, j], axis=-1)
            np.testing.assert_allclose(cos, 1.0, rtol=1e-13)
        assert np.array_equal(got[:, :, 2], x[:, :, 2])


def test_attention_with_norm_is_attention_on_normalised_inputs():
    """The full oracle with norm_w equals the oracle without it fed the
    normalised streams (the norm enters only through Q and K), and with unit
    weights and eps = 0 the logits of every row are bounded by d (Cauchy-
    Schwarz on unit-RMS vectors) so LSE <= sqrt(d) + ln S."""
    w = W.custom(B=1, H=2, d=64, S_txt=6, grid=4, n_ref=0)
    inp = W.make_inputs(w, 2)
    nw = W.norm_weights(64, 2)
    O1, L1 = oracle.joint_attention(inp["qkv_txt"], inp["qkv_img"], None, inp["pos"], w.split, w.theta,
                                    norm_w=nw, eps=1e-6)
    t, i, _ = oracle.qk_norm_streams(inp["qkv_txt"], inp["qkv_img"], None, nw, 1e-6)
    O2, L2 = oracle.joint_attention(t, i, None, inp["pos"], w.split, w.theta)
    np.testing.assert_array_equal(O1, O2)
    np.testing.assert_array_equal(L1, L2)
    _, L = oracle.joint_attention(inp["qkv_txt"], inp["qkv_img"], None, inp["pos"], w.split, w.theta,
                                  norm_w=torch.ones(3, 2, 64), eps=0.0)
    assert np.all(L <= math.sqrt(64) + math.log(w.S) + 1e-12)
