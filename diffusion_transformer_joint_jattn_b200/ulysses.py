"""Sequence-parallel joint attention (Ulysses) over a process group.

"Speed Up Image Generation with FLUX 3 Image Klein on NVIDIA Blackwell GPUs",
section "Multi-GPU inference": the runtime partitions each branch's sequence
across GPUs with Ulysses sequence parallelism (and puts the two classifier-
free-guidance branches on separate GPU groups, which is plain data
parallelism over the batch entries and needs no exchange).

Ulysses turns a sequence-sharded input into a head-sharded one and back:

* every rank holds, for each stream (txt, img, ref), its contiguous 1/P of
  the stream's tokens with all H heads: ``[B, S_s/P, 3, H, d]``;
* one all-to-all gives every rank all S tokens for its H/P heads (rank j gets
  heads [j*H/P, (j+1)*H/P)); the joint attention then runs locally, unchanged
  (every head is independent);
* a second all-to-all returns each rank's tokens with all heads:
  ``[B, S_s/P, H, d]`` per stream.

Both exchanges are single ``all_to_all_single`` calls (NCCL over NVLink on
GPUs) that carry all three streams at once: per destination rank the
payload is [txt block, img block, ref block].  The attention itself is the
library's device path (``jattn.joint_attention``, the high-precision pair
unless ``precise=False`` is passed); it is a parameter only so
that the exchange logic can be exercised on CPU process groups.
"""
from __future__ import annotations

from typing import Callable, Optional, Sequence, Tuple

import torch
import torch.distributed as dist


def _world(group) -> Tuple[int, int]:
    return dist.get_world_size(group), dist.get_rank(group)


def _check_shards(shards, P: int):
    ref = next(t for t in shards if t is not None)
    B, _, three, H, d = ref.shape
    if three != 3:
        raise ValueError("streams must be [B, S_s/P, 3, H, d]")
    if H % P:
        raise ValueError(f"H = {H} is not divisible by the group size {P}")
    for t in shards:
        if t is not None and (t.shape[0] != B or t.shape[2:] != ref.shape[2:] or not t.is_contiguous()):
            raise ValueError("all streams must be contiguous [B, S_s/P, 3, H, d] with the same B, H, d")
    return B, H, d


def ulysses_attention(shards: Sequence[Optional[torch.Tensor]], pos: torch.Tensor, split, theta: float = 10000.0,
                      group=None, attention: Optional[Callable] = None, **attention_kw):
    """Sequence-sharded joint attention.

    shards: (txt, img, ref) local shards ``[B, S_s/P, 3, H, d]`` (None for an
    absent stream), rank r holding tokens [r*S_s/P, (r+1)*S_s/P) of stream s;
    pos: ``[S, 3]`` int32 positions of the whole joint sequence (txt | img |
    ref), the same on every rank.  Returns the local output shards
    ``[B, S_s/P, H, d]`` per stream (None for absent streams).
    ``attention(qkv_txt, qkv_img, qkv_ref, pos, split, theta, **kw)`` computes
    O ``[B, S, H', d]`` for full-sequence streams of H' heads; by default the
    library's device path."""
    if attention is None:
        from . import jattn
        attention = jattn.joint_attention
    P, r = _world(group)
    B, H, d = _check_shards(shards, P)
    Hg = H // P
    lens = [0 if t is None else t.shape[1] for t in shards]          # local tokens per stream
    ref = next(t for t in shards if t is not None)

    # 1. sequence-sharded -> head-sharded: per destination j, each stream's
    #    local tokens for heads [j*Hg, (j+1)*Hg).
    send = []
    for t in shards:
        if t is None:
            continue
        S_loc = t.shape[1]
        blk = t.view(B, S_loc, 3, P, Hg, d).permute(3, 0, 1, 2, 4, 5)         # [P, B, S_loc, 3, Hg, d]
        send.append(blk.reshape(P, -1))
    send = torch.cat(send, dim=1).contiguous()                              # [P, L]
    recv = torch.empty_like(send)
    dist.all_to_all_single(recv, send, group=group)
    full = []
    off = 0
    for t, S_loc in zip(shards, lens):
        if t is None:
            full.append(None)
            continue
        n = B * S_loc * 3 * Hg * d
        blk = recv[:, off:off + n].view(P, B, S_loc, 3, Hg, d)               # block i: rank i's tokens
        full.append(blk.permute(1, 0, 2, 3, 4, 5).reshape(B, P * S_loc, 3, Hg, d).contiguous())
        off += n

    # 2. the joint attention of this rank's heads over the whole sequence
    o = attention(full[0], full[1], full[2], pos, split, theta, **attention_kw)   # [B, S, Hg, d]
    if isinstance(o, tuple):
        o = o[0]

    # 3. head-sharded -> sequence-sharded: per destination j, rank j's tokens
    #    of each stream, for this rank's heads.
    send_o = []
    start = 0
    for t, S_loc in zip(shards, lens):
        if t is None:
            continue
        S_s = P * S_loc
        seg = o[:, start:start + S_s].reshape(B, P, S_loc, Hg, d).permute(1, 0, 2, 3, 4)  # [P, B, S_loc, Hg, d]
        send_o.append(seg.reshape(P, -1))
        start += S_s
    send_o = torch.cat(send_o, dim=1).contiguous()
    recv_o = torch.empty_like(send_o)
    dist.all_to_all_single(recv_o, send_o, group=group)
    out = []
    off = 0
    for t, S_loc in zip(shards, lens):
        if t is None:
            out.append(None)
            continue
        n = B * S_loc * Hg * d
        blk = recv_o[:, off:off + n].view(P, B, S_loc, Hg, d)               # block i: heads of rank i
        out.append(blk.permute(1, 2, 0, 3, 4).reshape(B, S_loc, H, d).contiguous())
        off += n
    return tuple(out)


def shard_streams(streams: Sequence[Optional[torch.Tensor]], P: int, r: int):
    """Rank r's contiguous 1/P of each stream's tokens (streams [B, S_s, 3, H, d];
    every S_s must be divisible by P)."""
    out = []
    for t in streams:
        if t is None:
            out.append(None)
            continue
        S_s = t.shape[1]
        if S_s % P:
            raise ValueError(f"a stream of {S_s} tokens does not split over {P} ranks")
        n = S_s // P
        out.append(t[:, r * n:(r + 1) * n].contiguous())
    return out


def cfg_ulysses_layout(world: int, B: int, H: int, lens: Sequence[int]) -> Tuple[int, int]:
    """(cfg_size, ulysses_size) for ``world`` ranks, as the page's multi-GPU
    mode arranges them: the classifier-free-guidance branches (batch entries)
    on separate rank groups when the batch splits evenly, the sequence of
    each branch over the ranks of its group.  ulysses_size must divide H and
    every stream's token count."""
    cfg = 2 if world % 2 == 0 and B % 2 == 0 else 1
    uly = world // cfg
    if H % uly or any(n % uly for n in lens):
        raise ValueError(f"{world} ranks: ulysses size {uly} must divide H = {H} and the stream lengths {list(lens)}")
    return cfg, uly


def cfg_ulysses_groups(world: int, cfg: int, uly: int):
    """Rank lists of the Ulysses groups: group g holds ranks [g*uly, (g+1)*uly)
    and serves batch entries [g*B/cfg, (g+1)*B/cfg)."""
    if cfg * uly != world:
        raise ValueError("cfg_size * ulysses_size must equal the world size")
    return [list(range(g * uly, (g + 1) * uly)) for g in range(cfg)]


def rank_work(rank: int, B: int, cfg: int, uly: int) -> Tuple[slice, int, int]:
    """(batch slice, Ulysses group index, rank inside the group) of ``rank``."""
    g, r = divmod(rank, uly)
    nb = B // cfg
    return slice(g * nb, (g + 1) * nb), g, r
