"""Head-sharded VSA forward across the GPUs of one node.

Sequence-parallel DiT layers hold, on each rank, a contiguous shard of the
tokens for every head.  VSA needs a head's whole token grid (the cube tiling,
the coarse stage and the key selection span the sequence), so the forward
exchanges the shards once into head shards (every rank: all tokens of H / P
heads), runs the VSA kernels on them, and exchanges the outputs back into the
token shards: two all-to-alls around a per-head computation.  At 720p the
Wan-14B sequence is 75.6k tokens (the FastWan article, section "一张卡，秒生
视频", names sequences beyond 80k tokens for 720p video and attention as more
than 85 % of the inference time), which one B200 holds, so this is the
scaling path for longer sequences or more frames, not a need at 720p.

The exchanges are ``torch.distributed.all_to_all_single`` calls (NCCL on the
GPUs, gloo on the CPU for the tests), with uneven token shards allowed; no
collective reads another GPU's memory through a TMA load.
"""

from __future__ import annotations

from typing import Callable, Optional, Sequence

import torch
import torch.distributed as dist


def token_shards(n_tokens: int, world: int) -> list[tuple[int, int]]:
    """Contiguous token ranges of the ranks: the first n % world ranks get one more."""
    base, extra = divmod(n_tokens, world)
    out, start = [], 0
    for r in range(world):
        size = base + (1 if r < extra else 0)
        out.append((start, start + size))
        start += size
    return out


def _world(group) -> tuple[int, int]:
    if group is None and not dist.is_initialized():
        return 0, 1
    return dist.get_rank(group), dist.get_world_size(group)


def seq_to_heads(x: torch.Tensor, shards: Sequence[tuple[int, int]], group=None) -> torch.Tensor:
    """[B, H, n_r, ...] token shard -> [B, H / P, N, ...] head shard (all tokens)."""
    rank, world = _world(group)
    if world == 1:
        return x.contiguous()
    B, H = x.shape[:2]
    hp = H // world
    tail = x.shape[3:]
    per = int(torch.tensor(tail).prod().item()) if tail else 1
    # to rank j: heads j*hp .. (j+1)*hp of this rank's tokens
    send = torch.cat([x[:, j * hp:(j + 1) * hp].contiguous().reshape(-1) for j in range(world)])
    sizes_in = [B * hp * (shards[rank][1] - shards[rank][0]) * per] * world
    sizes_out = [B * hp * (e - s) * per for s, e in shards]
    recv = torch.empty(sum(sizes_out), dtype=x.dtype, device=x.device)
    dist.all_to_all_single(recv, send, sizes_out, sizes_in, group=group)
    parts, off = [], 0
    for (s, e), n in zip(shards, sizes_out):
        parts.append(recv[off:off + n].reshape(B, hp, e - s, *tail))
        off += n
    return torch.cat(parts, dim=2)


def heads_to_seq(y: torch.Tensor, shards: Sequence[tuple[int, int]], group=None) -> torch.Tensor:
    """[B, H / P, N, ...] head shard -> [B, H, n_r, ...] token shard."""
    rank, world = _world(group)
    if world == 1:
        return y.contiguous()
    B, hp = y.shape[:2]
    tail = y.shape[3:]
    per = int(torch.tensor(tail).prod().item()) if tail else 1
    # to rank j: this rank's heads at rank j's tokens
    send = torch.cat([y[:, :, s:e].contiguous().reshape(-1) for s, e in shards])
    sizes_in = [B * hp * (e - s) * per for s, e in shards]
    n_r = shards[rank][1] - shards[rank][0]
    sizes_out = [B * hp * n_r * per] * world
    recv = torch.empty(sum(sizes_out), dtype=y.dtype, device=y.device)
    dist.all_to_all_single(recv, send, sizes_out, sizes_in, group=group)
    return torch.cat([recv[i * sizes_out[0]:(i + 1) * sizes_out[0]].reshape(B, hp, n_r, *tail)
                      for i in range(world)], dim=1)


Attention = Callable[..., torch.Tensor]


def _vsa_attention(batch, heads, head_dim, grid, topk, q, k, v, g_f, g_c):
    """The VSA forward on one head shard: the three launches of the benchmark."""
    from . import vsa

    shape = vsa.make_shape(batch, heads, head_dim, grid)
    out = torch.empty_like(q)
    vsa.vsa_forward_fused(shape, q, k, v, topk, out, g_f, g_c)
    return out


def vsa_forward_head_parallel(grid, topk, q, k, v, g_f=None, g_c=None, group=None,
                              attention: Optional[Attention] = None) -> torch.Tensor:
    """The VSA forward of a sequence-parallel layer.

    q, k, v: this rank's token shard [B, H, n_r, d] (``token_shards`` of the
    grid's N tokens over the group's ranks, in rank order); g_f, g_c: the
    gates' shard [B, H, n_r] or None.  H must be a multiple of the world size.
    Returns this rank's shard of the output, [B, H, n_r, d].  ``attention``
    replaces the VSA kernels (same arguments as the default, which runs the
    CUDA path on the head shard)."""
    rank, world = _world(group)
    B, H, _, d = q.shape
    if H % world:
        raise ValueError(f"{H} heads do not split over {world} ranks")
    n_tokens = grid[0] * grid[1] * grid[2]
    shards = token_shards(n_tokens, world)
    if q.shape[2] != shards[rank][1] - shards[rank][0]:
        raise ValueError("q does not hold this rank's token shard")
    qh, kh, vh = (seq_to_heads(t, shards, group) for t in (q, k, v))
    gfh = seq_to_heads(g_f, shards, group) if g_f is not None else None
    gch = seq_to_heads(g_c, shards, group) if g_c is not None else None
    fn = attention or _vsa_attention
    oh = fn(B, H // world, d, grid, topk, qh, kh, vh, gfh, gch)
    return heads_to_seq(oh, shards, group)
