"""FP64 oracle for DiT joint attention with 2D axial RoPE.

TEST INFRASTRUCTURE ONLY.  Only the tests, the package's smoke check and the
benchmark's CPU-baseline leg may import this module.  The product path never
calls it and has no CPU fallback.

What it computes is the plain definition of the method, written out in float64
with numpy: joint-sequence assembly, rotary position embedding on Q and K, and
softmax(Q K^T / sqrt(d)) V over the whole joint sequence, with a two-pass
(not online) softmax.  Flash attention reaches the same result up to rounding,
so the definition is the oracle.

Sources ("Speed Up Image Generation with FLUX 3 Image Klein on NVIDIA Blackwell
GPUs"):
  * section "FLUX 3 inference with TensorRT LLM VisualGen": text, noisy
    target-image and optional reference-image streams are combined through
    joint attention -> ``joint_sequence``;
  * section "GEMM kernel optimization": rotary position embeddings are applied
    to the query and key projections -> ``rope_rotate``; the same fused
    projection also normalises the query and key -> ``rms_norm`` /
    ``qk_norm_streams`` (optional);
  * section "Quantized and sparse attention": the dense (VANILLA) attention the
    quantised variants are compared against -> ``attention_rows``.

Readings where the page is silent (each is listed in the design notes):
  * the joint order is txt | img | ref, no mask, every row is an output row;
  * RoPE is 2D axial over (t, row, col) with per-axis channel spans
    ``split = (n_t, n_r, n_c)`` laid out in that order; inside a span of n
    channels, pair p = channels (2p, 2p+1) rotates by pos_axis * theta^(-2p/n);
  * the softmax scale is exactly 1/sqrt(d);
  * query/key normalisation (when used) is RMSNorm over the d channels of
    one (token, head), with a learned per-channel weight, one weight vector
    per stream and per Q/K, applied before the rotation:
    x -> w * x / sqrt(mean(x^2) + eps).
"""
from __future__ import annotations

import math
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import torch


def as_f64(t) -> np.ndarray:
    """Exact float64 copy of a (bf16 / fp16 / fp32) torch tensor or array."""
    if isinstance(t, torch.Tensor):
        return t.detach().to("cpu").to(torch.float64).numpy()
    return np.asarray(t, dtype=np.float64)


# --------------------------------------------------------------------------
# Rotary position embedding (2D axial: t, row, col)
# --------------------------------------------------------------------------

def rope_frequencies(n: int, theta: float) -> np.ndarray:
    """omega_p = theta^(-2p/n) for p = 0 .. n/2-1 (one axis of n channels)."""
    p = np.arange(n // 2, dtype=np.float64)
    return np.power(np.float64(theta), -2.0 * p / n)


def rope_angles(pos: np.ndarray, split, theta: float) -> np.ndarray:
    """Angle of every channel pair: ``[S, d/2]`` float64.

    Pair index runs over the axes in order t, row, col; pair p of axis a turns
    by pos[:, a] * omega_{a,p}.
    """
    pos = np.asarray(pos, dtype=np.float64)
    cols = []
    for a, n in enumerate(split):
        if n:
            cols.append(pos[:, a:a + 1] * rope_frequencies(n, theta)[None, :])
    return np.concatenate(cols, axis=1)


def rope_rotate(x: np.ndarray, pos: np.ndarray, split, theta: float) -> np.ndarray:
    """Rotate each interleaved channel pair (2i, 2i+1) of ``x[..., S, d]``.

    (x0, x1) -> (x0 cos a - x1 sin a,  x0 sin a + x1 cos a).
    """
    ang = rope_angles(pos, split, theta)
    c, s = np.cos(ang), np.sin(ang)
    x0, x1 = x[..., 0::2], x[..., 1::2]
    out = np.empty_like(x, dtype=np.float64)
    out[..., 0::2] = x0 * c - x1 * s
    out[..., 1::2] = x0 * s + x1 * c
    return out


# --------------------------------------------------------------------------
# Query / key RMS normalisation
# --------------------------------------------------------------------------

def rms_norm(x, w, eps: float) -> np.ndarray:
    """w * x / sqrt(mean(x^2) + eps) over the last axis of ``x[..., d]``;
    ``w`` is ``[d]``."""
    x = np.asarray(x, dtype=np.float64)
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * np.asarray(w, dtype=np.float64)


def qk_norm_streams(qkv_txt, qkv_img, qkv_ref, norm_w, eps: float):
    """Normalise Q and K of each stream ``[B, S_s, 3, H, d]`` with that
    stream's weights: ``norm_w[s][0]`` for Q and ``norm_w[s][1]`` for K, s = 0
    (txt), 1 (img), 2 (ref).  V is untouched.  Returns float64 streams
    (``None`` stays ``None``)."""
    w = as_f64(norm_w)
    out = []
    for s, t in enumerate((qkv_txt, qkv_img, qkv_ref)):
        if t is None:
            out.append(None)
            continue
        x = as_f64(t).copy()
        x[:, :, 0] = rms_norm(x[:, :, 0], w[s, 0], eps)
        x[:, :, 1] = rms_norm(x[:, :, 1], w[s, 1], eps)
        out.append(x)
    return out


# --------------------------------------------------------------------------
# Joint sequence assembly
# --------------------------------------------------------------------------

def joint_sequence(qkv_txt, qkv_img, qkv_ref):
    """Concatenate the per-stream ``[B, S_s, 3, H, d]`` QKV tensors along the
    token axis in the order txt | img | ref and return float64 Q, K, V, each
    ``[B, H, S, d]``.  Absent streams are ``None``."""
    parts = [as_f64(t) for t in (qkv_txt, qkv_img, qkv_ref) if t is not None and t.shape[1] > 0]
    qkv = np.concatenate(parts, axis=1)                  # [B, S, 3, H, d]
    qkv = np.transpose(qkv, (2, 0, 3, 1, 4))             # [3, B, H, S, d]
    return qkv[0], qkv[1], qkv[2]


# --------------------------------------------------------------------------
# Attention
# --------------------------------------------------------------------------

def attention_rows(q_rows: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float):
    """Dense softmax attention of some query rows against all keys of one head.

    q_rows [n, d], k [S, d], v [S, d] (float64).  Two-pass softmax:
      s_ij = scale * q_i . k_j;  m_i = max_j s_ij;  p_ij = exp(s_ij - m_i);
      l_i = sum_j p_ij;  O_i = sum_j p_ij v_j / l_i;  LSE_i = m_i + ln l_i.
    Returns (O [n, d], LSE [n]).
    """
    s = (q_rows @ k.T) * scale
    m = s.max(axis=1, keepdims=True)
    p = np.exp(s - m)
    l = p.sum(axis=1, keepdims=True)
    o = (p @ v) / l
    return o, (m + np.log(l))[:, 0]


def joint_attention(qkv_txt, qkv_img, qkv_ref, pos, split, theta=10000.0, rows=None,
                    softmax_scale=None, row_chunk=1024, workers=None, norm_w=None, eps=1e-6):
    """The whole hot path in FP64: (normalise Q/K,) assemble, rotate Q/K,
    attend.

    rows: None for every row, else int ``[B, H, m]`` query-row indices.
    norm_w: None, or ``[3, 2, d]`` query/key RMSNorm weights per stream.
    Returns (O [B, H, m, d], LSE [B, H, m]) in float64.
    """
    if norm_w is not None:
        qkv_txt, qkv_img, qkv_ref = qk_norm_streams(qkv_txt, qkv_img, qkv_ref, norm_w, eps)
    q, k, v = joint_sequence(qkv_txt, qkv_img, qkv_ref)
    pos = np.asarray(pos.numpy() if isinstance(pos, torch.Tensor) else pos)
    B, H, S, d = q.shape
    scale = 1.0 / math.sqrt(d) if softmax_scale is None else float(softmax_scale)
    if rows is None:
        rows = np.broadcast_to(np.arange(S), (B, H, S))
    rows = np.asarray(rows.numpy() if isinstance(rows, torch.Tensor) else rows)
    m = rows.shape[-1]
    O = np.empty((B, H, m, d))
    L = np.empty((B, H, m))

    def one_head(bh):
        b, h = divmod(bh, H)
        r = rows[b, h]
        kh = rope_rotate(k[b, h], pos, split, theta)
        qh = rope_rotate(q[b, h][r], pos[r], split, theta)
        for i in range(0, m, row_chunk):
            O[b, h, i:i + row_chunk], L[b, h, i:i + row_chunk] = attention_rows(
                qh[i:i + row_chunk], kh, v[b, h], scale)

    if workers is None or workers <= 1 or B * H == 1:
        for bh in range(B * H):
            one_head(bh)
    else:
        with ThreadPoolExecutor(workers) as ex:
            list(ex.map(one_head, range(B * H)))
    return O, L


def rotated_qkv(qkv_txt, qkv_img, qkv_ref, pos, split, theta=10000.0, norm_w=None, eps=1e-6):
    """FP64 rotated Q, K and plain V, each ``[B, H, S, d]`` (the prologue's
    exact result before rounding to a storage type); Q and K normalised
    first when ``norm_w`` is given."""
    if norm_w is not None:
        qkv_txt, qkv_img, qkv_ref = qk_norm_streams(qkv_txt, qkv_img, qkv_ref, norm_w, eps)
    q, k, v = joint_sequence(qkv_txt, qkv_img, qkv_ref)
    pos = np.asarray(pos.numpy() if isinstance(pos, torch.Tensor) else pos)
    return rope_rotate(q, pos, split, theta), rope_rotate(k, pos, split, theta), v


def attention_on(q_rot, k_rot, v, rows=None, softmax_scale=None, row_chunk=1024):
    """Attention on given (already rotated) float64 ``[B, H, S, d]`` operands.

    Used for error attribution: feeding operands rounded to a storage format
    separates the format's own error from the rest of a kernel's error."""
    B, H, S, d = q_rot.shape
    scale = 1.0 / math.sqrt(d) if softmax_scale is None else float(softmax_scale)
    if rows is None:
        rows = np.broadcast_to(np.arange(S), (B, H, S))
    rows = np.asarray(rows.numpy() if isinstance(rows, torch.Tensor) else rows)
    m = rows.shape[-1]
    O = np.empty((B, H, m, d))
    L = np.empty((B, H, m))
    for b in range(B):
        for h in range(H):
            qh = q_rot[b, h][rows[b, h]]
            for i in range(0, m, row_chunk):
                O[b, h, i:i + row_chunk], L[b, h, i:i + row_chunk] = attention_rows(
                    qh[i:i + row_chunk], k_rot[b, h], v[b, h], scale)
    return O, L


def flops(B, H, S, d) -> int:
    """4 * B * H * S^2 * d: Q.K^T and P.V, 2*S^2*d each per (b, h)."""
    return 4 * B * H * S * S * d
