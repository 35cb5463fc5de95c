"""Seeded synthetic workloads for DiT joint attention.

This module only draws random numbers and lays them out; it holds none of the
method's arithmetic (no rotation, no softmax, no quantisation).  Both the CUDA
path and the FP64 oracle consume what it produces, so that a parity test feeds
byte-identical inputs to both sides.

Workload shapes follow the joint-attention setting of "Speed Up Image
Generation with FLUX 3 Image Klein on NVIDIA Blackwell GPUs" (section "FLUX 3
inference with TensorRT LLM VisualGen": text, noisy target-image and optional
reference-image streams combined through joint attention; section "Quantized
and sparse attention": 2048x2048 generation on one B200, where attention is
the dominant DiT kernel).  The page gives no head count, head dimension, text
length or RoPE layout; those come from the five workload definitions below.

Layout conventions (shared with the C ABI):

* A stream ``qkv_s`` is ``[B, S_s, 3, H, d]`` bf16 -- the natural output of a
  fused QKV projection for that stream (index 0 = Q, 1 = K, 2 = V).
* ``pos`` is ``[S, 3]`` int32 holding (t, row, col) per joint token, in the
  joint order txt | img | ref, shared across the batch.
* Text tokens sit at (0, 0, 0); image token (r, c) of a G x G grid at
  (0, r, c) in row-major order; reference image k (k = 1..n_ref) token (r, c)
  at (k, r, c).
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional, Tuple

import torch


@dataclass(frozen=True)
class JointAttentionWorkload:
    """One joint-attention problem: shapes, RoPE layout and value recipe."""

    name: str
    B: int
    H: int
    d: int
    S_txt: int
    grid: int                      # image tokens form a grid x grid patch grid
    n_ref: int                     # reference images, each grid x grid tokens
    split: Tuple[int, int, int]    # rotary channels per axis (t, row, col)
    theta: float = 10000.0
    outlier_frac: float = 0.0      # fraction of head channels scaled in Q and K
    outlier_mult: float = 1.0
    paths: Tuple[str, ...] = ("bf16",)
    description: str = field(default="", compare=False)

    @property
    def S_img(self) -> int:
        return self.grid * self.grid

    @property
    def S_ref(self) -> int:
        return self.n_ref * self.grid * self.grid

    @property
    def S(self) -> int:
        return self.S_txt + self.S_img + self.S_ref

    @property
    def n_outlier(self) -> int:
        return int(round(self.outlier_frac * self.d))

    @property
    def flops(self) -> int:
        """Algorithmic FLOPs of one call: 2*S^2*d for Q.K^T plus 2*S^2*d for P.V,
        per (batch, head)."""
        return 4 * self.B * self.H * self.S * self.S * self.d

    def with_batch_heads(self, B: Optional[int] = None, H: Optional[int] = None):
        from dataclasses import replace
        return replace(self, B=self.B if B is None else B, H=self.H if H is None else H)


WORKLOADS = (
    JointAttentionWorkload(
        "tiny", B=1, H=2, d=64, S_txt=32, grid=16, n_ref=0, split=(16, 24, 24),
        description="tiny joint attention: 32 text + 16x16 image tokens, d=64"),
    JointAttentionWorkload(
        "t2i_1024_base", B=2, H=24, d=128, S_txt=512, grid=64, n_ref=0, split=(16, 56, 56),
        outlier_frac=0.01, outlier_mult=8.0,
        description="1024x1024 Base T2I (CFG batch 2): 512 text + 64x64 image tokens"),
    JointAttentionWorkload(
        "t2i_2048_base", B=2, H=24, d=128, S_txt=512, grid=128, n_ref=0, split=(16, 56, 56),
        outlier_frac=0.01, outlier_mult=8.0, paths=("bf16", "fp8"),
        description="2048x2048 Base T2I (CFG batch 2): 512 text + 128x128 image tokens"),
    JointAttentionWorkload(
        "t2i_2048_distilled", B=1, H=24, d=128, S_txt=512, grid=128, n_ref=0, split=(16, 56, 56),
        outlier_frac=0.02, outlier_mult=16.0, paths=("fp8",),
        description="2048x2048 distilled T2I (no CFG): 512 text + 128x128 image tokens"),
    JointAttentionWorkload(
        "i2i_2048_base", B=2, H=24, d=128, S_txt=512, grid=128, n_ref=1, split=(16, 56, 56),
        outlier_frac=0.01, outlier_mult=8.0, paths=("bf16", "fp8"),
        description="2048x2048 Base I2I: 512 text + 128x128 target + 128x128 reference tokens"),
)

BY_NAME = {w.name: w for w in WORKLOADS}


def joint_positions(S_txt: int, grid: int, n_ref: int) -> torch.Tensor:
    """(t, row, col) int32 positions of the joint sequence txt | img | ref."""
    G = grid
    r = torch.arange(G, dtype=torch.int32).repeat_interleave(G)
    c = torch.arange(G, dtype=torch.int32).repeat(G)
    parts = [torch.zeros(S_txt, 3, dtype=torch.int32)]
    for t in range(n_ref + 1):
        parts.append(torch.stack([torch.full((G * G,), t, dtype=torch.int32), r, c], dim=1))
    return torch.cat(parts, dim=0).contiguous()


def outlier_channels(w: JointAttentionWorkload, seed: int, shared: bool = True):
    """Per-head outlier channel sets for Q and K (int64 [H, n_outlier] each).

    ``shared=True`` scales the same channels in Q and K (the plain reading of
    "1% of head channels in Q and K scaled"); ``shared=False`` draws K's set
    independently.
    """
    g = torch.Generator().manual_seed(seed + 1)
    n = w.n_outlier
    q_idx = torch.empty(w.H, n, dtype=torch.int64)
    k_idx = torch.empty(w.H, n, dtype=torch.int64)
    for h in range(w.H):
        q_idx[h] = torch.randperm(w.d, generator=g)[:n]
        k_idx[h] = q_idx[h] if shared else torch.randperm(w.d, generator=g)[:n]
    return q_idx, k_idx


def _draw(w: JointAttentionWorkload, g: torch.Generator, idx: Optional[torch.Tensor]):
    x = torch.randn(w.B, w.S, w.H, w.d, generator=g, dtype=torch.float32)
    if idx is not None and idx.numel():
        for h in range(w.H):
            x[:, :, h, idx[h]] *= w.outlier_mult   # powers of two: exact in bf16
    return x.to(torch.bfloat16)


def make_inputs(w: JointAttentionWorkload, seed: int = 0, shared_outliers: bool = True):
    """Draw Q, K, V ~ N(0, 1) (each ``[B, S, H, d]`` fp32, txt | img | ref order,
    from one generator seeded ``seed``), scale the outlier channels, round to
    bf16 and pack per stream.

    Returns ``dict(qkv_txt, qkv_img, qkv_ref, pos)``; a stream with no tokens is
    ``None``.  Everything is on the CPU.
    """
    g = torch.Generator().manual_seed(seed)
    q_idx, k_idx = outlier_channels(w, seed, shared_outliers) if w.n_outlier else (None, None)
    q = _draw(w, g, q_idx)
    k = _draw(w, g, k_idx)
    v = _draw(w, g, None)
    bounds = [0, w.S_txt, w.S_txt + w.S_img, w.S]
    streams = []
    for a, b in zip(bounds[:-1], bounds[1:]):
        if b == a:
            streams.append(None)
        else:
            streams.append(torch.stack([q[:, a:b], k[:, a:b], v[:, a:b]], dim=2).contiguous())
    del q, k, v
    return dict(qkv_txt=streams[0], qkv_img=streams[1], qkv_ref=streams[2],
                pos=joint_positions(w.S_txt, w.grid, w.n_ref))


def norm_weights(d: int, seed: int = 0, spread: float = 0.25) -> torch.Tensor:
    """Synthetic query/key RMSNorm weights: fp32 ``[3, 2, d]`` (stream txt /
    img / ref, then Q / K), drawn as 1 + spread * N(0, 1) from a generator
    seeded ``seed + 3``.  (Trained weights are not needed: the normalisation's
    arithmetic is the same for any weight vector.)"""
    g = torch.Generator().manual_seed(seed + 3)
    return (1.0 + spread * torch.randn(3, 2, d, generator=g, dtype=torch.float32)).contiguous()


def sample_rows(w: JointAttentionWorkload, n: int = 4096, seed: int = 0) -> torch.Tensor:
    """Sorted distinct query rows per (b, h): int64 ``[B, H, m]`` with
    m = min(n, S); every row when S <= n."""
    g = torch.Generator().manual_seed(seed + 2)
    m = min(n, w.S)
    out = torch.empty(w.B, w.H, m, dtype=torch.int64)
    for b in range(w.B):
        for h in range(w.H):
            if m == w.S:
                out[b, h] = torch.arange(w.S)
            else:
                out[b, h] = torch.sort(torch.randperm(w.S, generator=g)[:m]).values
    return out


def custom(name="custom", **kw) -> JointAttentionWorkload:
    """A workload with explicit shapes (edge cases, small parity cases)."""
    kw.setdefault("split", (16, 56, 56) if kw.get("d", 128) == 128 else (16, 24, 24))
    return JointAttentionWorkload(name, **kw)
