"""FP64 oracle of the FP8 attention with token repair.

TEST INFRASTRUCTURE ONLY.  Only the tests, the package's smoke check and the
benchmark's CPU-baseline leg may import this module; the product path never
calls it and has no CPU fallback.

Source ("Speed Up Image Generation with FLUX 3 Image Klein on NVIDIA Blackwell
GPUs", section "Quantized and sparse attention"): the FP8 attention variant
that the page recommends at 2048x2048 selects, with a repair budget rho
(0.005 in the tested configuration), the fraction of tokens with the highest
quantisation error and corrects them with a residual computed at higher
precision.  The page names neither the error measure nor the form of the
correction; the readings taken here (also listed in the design notes) are:

  * per (batch, head), n = min(S, ceil(rho * S - 1e-3)) tokens are repaired
    (the 1e-3 keeps a budget that lands a rounding error above an integer,
    e.g. a float32 rho of 0.3 on 10 tokens, from taking one more token);
  * a token's quantisation error is measured by the e4m3 error bound of its
    key and value rows, which for a floating-point format is proportional to
    their magnitude: score_j = |k_j|^2 + |v_j|^2 (rotated, unquantised k);
    the n largest scores are taken, ties to the lower token index;
  * a repaired token enters the attention with its exact key and value and an
    exact logit q_i . k_j; every other token with the dequantised e4m3 key and
    value and the logit qd_i . kd_j of the dequantised operands.  One softmax
    runs over all S keys.
"""
from __future__ import annotations

import math

import numpy as np


def repair_count(S: int, rho: float) -> int:
    """n = ceil(rho * S - 1e-3), within [0, S] (0 when rho == 0)."""
    return max(0, min(S, int(math.ceil(rho * S - 1e-3)))) if rho > 0 else 0


def repair_scores(k_rot: np.ndarray, v: np.ndarray) -> np.ndarray:
    """|k_j|^2 + |v_j|^2 over the last axis: ``[..., S, d]`` -> ``[..., S]``."""
    k_rot = np.asarray(k_rot, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    return np.sum(k_rot * k_rot, axis=-1) + np.sum(v * v, axis=-1)


def repair_select(scores: np.ndarray, n: int) -> np.ndarray:
    """Indices of the n largest scores of a 1-D array (ties to the lower
    index), returned in ascending index order."""
    scores = np.asarray(scores, dtype=np.float64)
    order = np.lexsort((np.arange(scores.shape[0]), -scores))
    return np.sort(order[:n])


def repaired_attention_rows(q_rows, qd_rows, k, v, kd, vd, repaired, scale: float):
    """Attention of some query rows of one head with a repaired key set.

    q_rows / qd_rows [m, d]: exact / dequantised query rows; k, v, kd, vd
    [S, d]; ``repaired``: token indices.  Logit of key j: q_i . k_j * scale if
    j is repaired, else qd_i . kd_j * scale; value v_j or vd_j alike.
    Two-pass softmax over all keys.  Returns (O [m, d], LSE [m])."""
    S = k.shape[0]
    rep = np.zeros(S, dtype=bool)
    rep[np.asarray(repaired, dtype=np.int64)] = True
    s = np.where(rep[None, :], q_rows @ k.T, qd_rows @ kd.T) * scale
    vv = np.where(rep[:, None], v, vd)
    m = s.max(axis=1, keepdims=True)
    p = np.exp(s - m)
    l = p.sum(axis=1, keepdims=True)
    return (p @ vv) / l, (m + np.log(l))[:, 0]


def repaired_attention(q, k, v, qd, kd, vd, repaired, rows=None, softmax_scale=None, row_chunk=1024):
    """All (b, h): exact operands q, k, v and dequantised qd, kd, vd, each
    ``[B, H, S, d]`` float64; repaired ``[B, H, n]`` token indices.
    Returns (O [B, H, m, d], LSE [B, H, m])."""
    B, H, S, d = q.shape
    scale = 1.0 / math.sqrt(d) if softmax_scale is None else float(softmax_scale)
    if rows is None:
        rows = np.broadcast_to(np.arange(S), (B, H, S))
    rows = np.asarray(rows)
    m = rows.shape[-1]
    O = np.empty((B, H, m, d))
    L = np.empty((B, H, m))
    for b in range(B):
        for h in range(H):
            r = rows[b, h]
            for i in range(0, m, row_chunk):
                rr = r[i:i + row_chunk]
                O[b, h, i:i + row_chunk], L[b, h, i:i + row_chunk] = repaired_attention_rows(
                    q[b, h][rr], qd[b, h][rr], k[b, h], v[b, h], kd[b, h], vd[b, h], repaired[b, h], scale)
    return O, L
