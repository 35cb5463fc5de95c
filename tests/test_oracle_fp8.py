"""Pins for the oracle's E4M3 encoder and per-block quantiser (CPU only).

The encoder is checked against the OCP E4M3 table (golden fixture), against an
exhaustive round trip of every finite code, against torch's own
``float8_e4m3fn`` cast (a library routine, for in-range values) and against
round-to-nearest-even tie cases.  The block quantiser is checked against the
properties its definition fixes (the block maximum maps to 448, the
dequantisation error bound, zero blocks, block boundaries).
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
rng = np.random.default_rng(7)


def test_decode_table_golden():
    fx = json.load(open(os.path.join(GOLDEN, "e4m3_codes.json")))
    for c in fx["decode"]:
        assert oracle.e4m3_decode(np.uint8(int(c["code"], 16))) == c["value"], c
    assert np.isnan(oracle.e4m3_decode(np.uint8(0x7F)))
    assert np.isnan(oracle.e4m3_decode(np.uint8(0xFF)))


def test_encode_rne_and_saturation_golden():
    fx = json.load(open(os.path.join(GOLDEN, "e4m3_codes.json")))
    for c in fx["encode_rne"]:
        assert int(oracle.e4m3_encode(np.float64(c["x"]))) == int(c["code"], 16), c


def test_every_finite_code_round_trips():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    vals = oracle.e4m3_decode(codes)
    back = oracle.e4m3_encode(vals)
    np.testing.assert_array_equal(back, codes)


def test_encode_matches_torch_cast_in_range():
    """torch's float8_e4m3fn cast (RNE) agrees on finite in-range values,
    including subnormals, ties and values just around every code."""
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    vals = oracle.e4m3_decode(codes)
    mids = []
    svals = np.sort(np.unique(vals))
    for a, b in zip(svals[:-1], svals[1:]):
        m = 0.5 * (a + b)
        mids += [m, np.nextafter(m, -np.inf), np.nextafter(m, np.inf)]
    x = np.concatenate([vals, np.array(mids), rng.uniform(-448, 448, 20000),
                        rng.standard_normal(20000) * 0.01]).astype(np.float32)
    x = x[np.abs(x) <= 448]
    mine = oracle.e4m3_encode(x)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(mine, ref)


def test_quantize_block_max_maps_to_448_and_error_bound():
    """scale = amax/448 puts each block's largest |x| on code +-448 (0x7E/0xFE),
    and every dequantised value is within half a step of x: relative error
    <= 2^-4 in the normal range, absolute <= 2^-10 * scale below it."""
    x = (rng.standard_normal((2, 3, 300, 64)) * rng.uniform(0.01, 100, (2, 3, 1, 1))).astype(np.float32)
    codes, scale = oracle.quantize_blocks(x)
    assert scale.shape == (2, 3, 3)
    for b in range(2):
        for h in range(3):
            for j in range(3):
                blk = x[b, h, 128 * j:128 * (j + 1)]
                cb = codes[b, h, 128 * j:128 * (j + 1)]
                i = np.unravel_index(np.argmax(np.abs(blk)), blk.shape)
                assert cb[i] & 0x7F == 0x7E
                assert scale[b, h, j] == np.float32(np.float64(np.abs(blk).max()) / 448.0)
    dq = oracle.dequantize_blocks(codes, scale)
    s = np.repeat(scale.astype(np.float64), 128, axis=2)[:, :, :300, None]
    y = np.abs(x.astype(np.float64)) / s
    err = np.abs(dq - x)
    normal = y >= 2.0 ** -6
    assert np.all(err[normal] <= 2.0 ** -4 * np.abs(x[normal]) * (1 + 1e-6))
    assert np.all(err[~normal] <= 2.0 ** -10 * s.repeat(64, -1)[~normal] * (1 + 1e-6))


def test_quantize_zero_block_and_tail():
    """An all-zero block gets scale 1 and code 0; a ragged tail block is its
    own block (its scale ignores the previous block)."""
    x = np.zeros((1, 1, 130, 8), np.float32)
    x[0, 0, 129, 3] = -2.0
    codes, scale = oracle.quantize_blocks(x)
    assert scale[0, 0, 0] == 1.0
    assert np.all(codes[0, 0, :128] == 0)
    assert scale[0, 0, 1] == np.float32(2.0 / 448.0)
    assert codes[0, 0, 129, 3] == 0xFE
