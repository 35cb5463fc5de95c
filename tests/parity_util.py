"""Helpers shared by the GPU parity tests: oracle results per workload (cached
for the session), row gathering and the error metrics.

Error metrics (the plain reading of the tolerance statement): rel-L2 =
||O_gpu - O_ref||_F / ||O_ref||_F over all sampled rows of all (b, h) at
once; max-abs over the same set.
"""
from __future__ import annotations

import functools
import os

import numpy as np
import torch

import oracle
from diffusion_transformer_joint_jattn_b200 import workloads as W

# Tolerances for the BF16 path and the FP8 path (fixed by the method's
# accuracy target for this workload family).
BF16_REL_L2 = 5e-3
BF16_MAX_ABS = 2e-2
FP8_REL_L2 = 3e-2

ORACLE_WORKERS = max(1, min(8, (os.cpu_count() or 2) // 2))


def rel_l2(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


def max_abs(a, b) -> float:
    return float(np.max(np.abs(np.asarray(a, np.float64) - np.asarray(b, np.float64))))


def gather_rows(o_bshd: torch.Tensor, rows: torch.Tensor) -> np.ndarray:
    """O [B, S, H, d] (any device) -> float64 [B, H, m, d] at rows [B, H, m]."""
    o = o_bshd.to("cpu")
    B, S, H, d = o.shape
    out = np.empty((B, H, rows.shape[-1], d))
    for b in range(B):
        for h in range(H):
            out[b, h] = o[b, rows[b, h], h].to(torch.float64).numpy()
    return out


def gather_lse(lse_bhs: torch.Tensor, rows: torch.Tensor) -> np.ndarray:
    l = lse_bhs.to("cpu").to(torch.float64)
    B, H, _ = l.shape
    return np.stack([np.stack([l[b, h, rows[b, h]].numpy() for h in range(H)]) for b in range(B)])


@functools.lru_cache(maxsize=2)
def workload_case(name: str, n_rows: int = 4096, seed: int = 0):
    """(workload, inputs, rows, O_ref [B,H,m,d], LSE_ref [B,H,m]) on the CPU."""
    w = W.BY_NAME[name]
    inp = W.make_inputs(w, seed)
    rows = W.sample_rows(w, n_rows, seed)
    O, L = oracle.joint_attention(inp["qkv_txt"], inp["qkv_img"], inp["qkv_ref"], inp["pos"], w.split,
                                  w.theta, rows=rows, workers=ORACLE_WORKERS)
    return w, inp, rows, O, L


def fp16_operand_floor(w, inp, rows) -> np.ndarray:
    """The oracle's attention (float64) on the sampled rows after rounding the
    rotated Q and K to fp16 (V is exact in fp16 for these inputs): with the
    result rounded to bf16 on top, the error any kernel with 16-bit
    tensor-core operands and a bf16 output carries by format alone."""
    import math
    from concurrent.futures import ThreadPoolExecutor
    q, k, v = oracle.joint_sequence(inp["qkv_txt"], inp["qkv_img"], inp["qkv_ref"])
    pos = inp["pos"].numpy()
    rows = rows.numpy()
    out = np.empty((w.B, w.H, rows.shape[-1], w.d))

    def head(bh):
        b, h = divmod(bh, w.H)
        r = rows[b, h]
        kr = oracle.rope_rotate(k[b, h], pos, w.split, w.theta).astype(np.float16).astype(np.float64)
        qr = oracle.rope_rotate(q[b, h][r], pos[r], w.split, w.theta).astype(np.float16).astype(np.float64)
        for i in range(0, len(r), 1024):
            out[b, h, i:i + 1024], _ = oracle.attention_rows(qr[i:i + 1024], kr, v[b, h], 1 / math.sqrt(w.d))

    with ThreadPoolExecutor(ORACLE_WORKERS) as ex:
        list(ex.map(head, range(w.B * w.H)))
    return out


def round_bf16(x: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(x)).to(torch.bfloat16).to(torch.float64).numpy()


def to_device(inp, dev):
    return {k: (None if v is None else v.to(dev)) for k, v in inp.items()}
