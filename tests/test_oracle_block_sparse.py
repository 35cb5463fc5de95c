"""Pins of the block-sparse oracle (oracle/block_sparse.py), none of which
re-uses its own formulas:
  * block means of a hand-made sequence, including a short last block;
  * block shares of a hand-built 2 x 3 case, each value worked out with
    math.exp here, and rows summing to 1;
  * the selection rule on hand-picked shares (threshold tau / n_kb, the
    largest share always kept, ties to the lower block);
  * special cases that reduce to already-pinned functions: tau = 0 is the
    dense attention (oracle.attention_on), one kept block per query block is
    the dense attention over that block's keys (oracle.attention_rows on the
    sliced keys);
  * invariances: shuffling the tokens inside a key block changes neither the
    selection nor the output."""
import math

import numpy as np
import pytest

import oracle
from oracle import block_sparse as bs


def test_block_means_hand_example():
    x = np.arange(10, dtype=np.float64).reshape(5, 2)        # rows (0,1), (2,3), (4,5), (6,7), (8,9)
    m = bs.block_means(x, 2)
    np.testing.assert_array_equal(m, [[1.0, 2.0], [5.0, 6.0], [8.0, 9.0]])
    np.testing.assert_array_equal(bs.block_means(x, 5), [[4.0, 5.0]])
    np.testing.assert_array_equal(bs.block_means(x, 8), [[4.0, 5.0]])


def test_block_shares_hand_example():
    # d = 2, scale 1: query block means (1, 0) and (0, 2); key blocks of 2
    # with means (1, 1), (0, -1), (2, 0)
    q = np.array([[1.0, 0.0], [1.0, 0.0], [0.0, 2.0], [0.0, 2.0]])
    k = np.array([[1.0, 2.0], [1.0, 0.0], [0.0, -1.0], [0.0, -1.0], [3.0, 0.0], [1.0, 0.0]])
    sh = bs.block_shares(q, k, bq=2, bk=2, softmax_scale=1.0)
    e = [math.exp(1.0), math.exp(0.0), math.exp(2.0)]        # logits 1, 0, 2
    np.testing.assert_allclose(sh[0], [x / sum(e) for x in e], rtol=1e-15)
    e = [math.exp(2.0), math.exp(-2.0), math.exp(0.0)]       # logits 2, -2, 0
    np.testing.assert_allclose(sh[1], [x / sum(e) for x in e], rtol=1e-15)
    rng = np.random.default_rng(0)
    sh = bs.block_shares(rng.standard_normal((300, 8)), rng.standard_normal((500, 8)))
    np.testing.assert_allclose(sh.sum(axis=1), 1.0, rtol=1e-14)
    assert sh.shape == (2, 4)


def test_block_select_rule():
    sh = np.array([[0.5, 0.3, 0.2], [0.2, 0.2, 0.6], [1 / 3, 1 / 3, 1 / 3]])
    assert bs.block_select(sh, 0.0).all()
    np.testing.assert_array_equal(bs.block_select(sh, 1.0), [[1, 0, 0], [0, 0, 1], [1, 1, 1]])
    np.testing.assert_array_equal(bs.block_select(sh, 0.9), [[1, 1, 0], [0, 0, 1], [1, 1, 1]])
    # tau so large that no share reaches it: only the largest share (ties -> lower index)
    np.testing.assert_array_equal(bs.block_select(sh, 10.0), [[1, 0, 0], [0, 0, 1], [1, 0, 0]])


def _case(S=300, d=16, H=2, seed=1):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((1, H, S, d)), rng.standard_normal((1, H, S, d)) * 1.5,
            rng.standard_normal((1, H, S, d)))


def test_tau_zero_is_dense_attention():
    q, k, v = _case()
    O, L, keep = bs.block_sparse_attention(q, k, v, 0.0, bq=64, bk=32)
    assert keep.all()
    O2, L2 = oracle.attention_on(q, k, v)
    np.testing.assert_allclose(O, O2, rtol=0, atol=1e-13)
    np.testing.assert_allclose(L, L2, rtol=0, atol=1e-13)


def test_one_kept_block_is_attention_over_its_keys():
    """Query block I keeps only key block J: the output equals dense
    attention over that block's keys alone (the last key block is short)."""
    q, k, v = _case(S=300)
    bq, bk = 64, 32
    n_qb, n_kb = -(-300 // bq), -(-300 // bk)
    keep = np.zeros((1, 2, n_qb, n_kb), dtype=bool)
    choice = [[3, 9, 0, 5, 9], [1, 1, 8, 2, 9]]               # block 9 holds tokens 288..299
    for h in range(2):
        for I in range(n_qb):
            keep[0, h, I, choice[h][I]] = True
    O, _, _ = bs.block_sparse_attention(q, k, v, 0.0, bq=bq, bk=bk, keep=keep)
    scale = 1 / math.sqrt(16)
    for h in range(2):
        for I in range(n_qb):
            J = choice[h][I]
            r = slice(I * bq, min(300, (I + 1) * bq))
            ks = slice(J * bk, min(300, (J + 1) * bk))
            want, _ = oracle.attention_rows(q[0, h, r], k[0, h, ks], v[0, h, ks], scale)
            np.testing.assert_allclose(O[0, h, r], want, rtol=0, atol=1e-13)


def test_shuffling_inside_a_key_block_changes_nothing():
    q, k, v = _case(S=256, d=8)
    O, _, keep = bs.block_sparse_attention(q, k, v, 1.0, bq=64, bk=32)
    assert not keep.all() and keep.any(axis=-1).all()
    perm = np.arange(256)
    rng = np.random.default_rng(5)
    for J in range(8):
        perm[J * 32:(J + 1) * 32] = J * 32 + rng.permutation(32)
    O2, _, keep2 = bs.block_sparse_attention(q, k[:, :, perm], v[:, :, perm], 1.0, bq=64, bk=32)
    np.testing.assert_array_equal(keep, keep2)
    np.testing.assert_allclose(O, O2, rtol=0, atol=1e-13)


def test_higher_tau_keeps_fewer_blocks():
    q, k, v = _case(S=512, d=8)
    sh = bs.block_shares(q[0, 0], k[0, 0], bq=64, bk=32)
    kept = [bs.block_select(sh, t).sum() for t in (0.0, 0.5, 1.0, 1.5, 3.0)]
    assert kept == sorted(kept, reverse=True) and kept[0] == sh.size and kept[-1] >= sh.shape[0]
