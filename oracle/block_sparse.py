"""FP64 oracle of the block-sparse joint attention.

TEST INFRASTRUCTURE ONLY.  Only the tests, the package's smoke check and the
benchmark's CPU-baseline leg may import this module; the product path never
calls it and has no CPU fallback.

Source ("Speed Up Image Generation with FLUX 3 Image Klein on NVIDIA Blackwell
GPUs", sections "Quantized and sparse attention" and "Optimized single-GPU
deployment"): Sol-Attention cuts the DiT's attention work with a block-sparse
kernel whose sparsity a parameter tau controls -- a higher tau lowers the
image quality for little further speed, i.e. drops more blocks -- and which
runs dense until a noise-level cutoff (a sampler setting, outside this
operation: tau = 0 is the dense attention).  The page names no selection
rule; the reading taken here (also listed in the design notes):

  * queries are grouped in blocks of ``bq`` = 256 consecutive joint tokens,
    keys in blocks of ``bk`` = 128 (the last block of each may be shorter);
  * each block is represented by the mean of its rotated query (key) rows;
  * for query block I the estimated attention share of key block J is the
    softmax over J of  qbar_I . kbar_J * scale  (scale = 1/sqrt(d));
  * key block J is kept for query block I iff its share is at least
    tau / n_kb (tau times the share of a uniform attention), and the block
    with the largest share is always kept, so every query block attends to
    at least one key block;
  * every query row of block I then attends, with an exact softmax, to the
    keys of its kept blocks only.
"""
from __future__ import annotations

import math

import numpy as np

BQ = 256
BK = 128


def block_means(x: np.ndarray, block: int) -> np.ndarray:
    """Mean over consecutive token blocks of ``x [..., S, d]`` -> ``[..., nb, d]``;
    the last block averages only its own (possibly fewer) tokens."""
    x = np.asarray(x, dtype=np.float64)
    S = x.shape[-2]
    nb = -(-S // block)
    out = np.empty(x.shape[:-2] + (nb, x.shape[-1]))
    for i in range(nb):
        out[..., i, :] = x[..., i * block:min(S, (i + 1) * block), :].mean(axis=-2)
    return out


def block_shares(q_rot: np.ndarray, k_rot: np.ndarray, bq: int = BQ, bk: int = BK, softmax_scale=None):
    """Estimated attention share of every key block for every query block of
    one head: ``q_rot, k_rot [S, d]`` -> ``[n_qb, n_kb]``, rows summing to 1."""
    d = q_rot.shape[-1]
    scale = 1.0 / math.sqrt(d) if softmax_scale is None else float(softmax_scale)
    s = block_means(q_rot, bq) @ block_means(k_rot, bk).T * scale
    s = s - s.max(axis=1, keepdims=True)
    p = np.exp(s)
    return p / p.sum(axis=1, keepdims=True)


def block_select(shares: np.ndarray, tau: float) -> np.ndarray:
    """Kept key blocks ``[n_qb, n_kb]`` (bool): share >= tau / n_kb, plus each
    row's largest share (ties to the lower block index)."""
    n_kb = shares.shape[1]
    keep = shares >= tau / n_kb
    keep[np.arange(shares.shape[0]), np.argmax(shares, axis=1)] = True
    return keep


def block_sparse_attention_rows(q_rows, rows, k, v, keep, bq: int = BQ, bk: int = BK, softmax_scale=None):
    """Attention of query rows (indices ``rows`` into the sequence, values
    ``q_rows [m, d]``) of one head over the keys of their query block's kept
    key blocks, two-pass softmax.  Returns (O [m, d], LSE [m])."""
    S, d = k.shape
    scale = 1.0 / math.sqrt(d) if softmax_scale is None else float(softmax_scale)
    rows = np.asarray(rows)
    O = np.empty((len(rows), d))
    L = np.empty(len(rows))
    key_block = np.arange(S) // bk
    for I in np.unique(rows // bq):
        sel = rows // bq == I
        kmask = keep[I][key_block]
        s = (q_rows[sel] @ k[kmask].T) * scale
        m = s.max(axis=1, keepdims=True)
        p = np.exp(s - m)
        l = p.sum(axis=1, keepdims=True)
        O[sel] = (p @ v[kmask]) / l
        L[sel] = (m + np.log(l))[:, 0]
    return O, L


def block_sparse_attention(q_rot, k_rot, v, tau: float, rows=None, bq: int = BQ, bk: int = BK,
                           softmax_scale=None, keep=None):
    """All (b, h) of rotated ``[B, H, S, d]`` operands: select (unless ``keep``
    ``[B, H, n_qb, n_kb]`` is given) and attend.  Returns (O [B, H, m, d],
    LSE [B, H, m], keep [B, H, n_qb, n_kb])."""
    B, H, S, d = q_rot.shape
    if rows is None:
        rows = np.broadcast_to(np.arange(S), (B, H, S))
    rows = np.asarray(rows)
    m = rows.shape[-1]
    O = np.empty((B, H, m, d))
    L = np.empty((B, H, m))
    keeps = np.empty((B, H, -(-S // bq), -(-S // bk)), dtype=bool)
    for b in range(B):
        for h in range(H):
            kp = keep[b, h] if keep is not None else block_select(
                block_shares(q_rot[b, h], k_rot[b, h], bq, bk, softmax_scale), tau)
            keeps[b, h] = kp
            O[b, h], L[b, h] = block_sparse_attention_rows(q_rot[b, h][rows[b, h]], rows[b, h], k_rot[b, h],
                                                            v[b, h], kp, bq, bk, softmax_scale)
    return O, L, keeps
