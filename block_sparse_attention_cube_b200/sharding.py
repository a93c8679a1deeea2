"""Multi-GPU partitions of the attention call, one process per GPU.

Every (batch element, head) pair is independent from the pooling to the merge: the coarse
scores, the selection and the fine attention never mix heads or batch elements.  So:

* head-sharded inputs (each rank holds all tokens of its heads): each rank runs the call on its
  heads, with no collective (`head_range` gives a rank's heads);
* token-sharded inputs (sequence parallelism in the Ulysses style, where each rank holds a shard of
  the tokens for every head, padded so that the shards are equal): one all-to-all turns the token
  shards of all heads into all tokens of this rank's heads before the call, and one turns the
  output back (`seq_to_heads`, `heads_to_seq`, `sharded_forward`).  The pre-attention pass
  (Q/K RMSNorm over all H*D channels of a token, then 3D RoPE) runs on the token shard first,
  where each token's whole row is present, at the shard's token offset;
* classifier-free-guidance branches are batch elements: with the batch split across ranks
  (`batch_range`) the ranks run independent calls.

Sources: WorldFoundry inference-optimisation guide (openenvision.org, "推理优化"), fused_rope row
(the fused RoPE takes the rank's token offset and padding under Ulysses sequence parallelism);
Wan2.2 teardown (zharfai.com), section "Video sparse attention selects cubes" (attention per head).

The collectives are torch.distributed all_to_all_single calls (NCCL on GPUs, gloo on CPU); with
one rank, or no process group, they are the identity.  The attention itself always runs in the
library's kernels; `attend` exists so that a test can put a reference in its place on CPU ranks.
"""
from __future__ import annotations

from typing import Callable, List, Optional, Tuple

import torch

from . import Shape, forward, qk_norm_rope


def _world(group) -> Tuple[int, int]:
    import torch.distributed as dist
    if not dist.is_available() or not dist.is_initialized():
        return 1, 0
    return dist.get_world_size(group), dist.get_rank(group)


def head_range(heads: int, world: int, rank: int) -> Tuple[int, int]:
    """Contiguous heads [h0, h1) of a rank; shares differ by at most one head."""
    base, extra = divmod(heads, world)
    h0 = rank * base + min(rank, extra)
    return h0, h0 + base + (1 if rank < extra else 0)


def batch_range(batch: int, world: int, rank: int) -> Tuple[int, int]:
    """Contiguous batch elements [b0, b1) of a rank (CFG branches, independent requests)."""
    return head_range(batch, world, rank)


def token_shard(tokens: int, world: int, rank: int) -> Tuple[int, int]:
    """(token_offset, n) of a rank's shard: n = ceil(N / world) rows; rows past N are padding."""
    n = -(-tokens // world)
    return rank * n, n


def _all_to_all(send: List[torch.Tensor], recv_shapes: List[Tuple[int, ...]], group) -> List[torch.Tensor]:
    """Send send[r] to rank r; receive one tensor of recv_shapes[s] from every rank s."""
    import torch.distributed as dist
    flat = torch.cat([t.reshape(-1) for t in send])
    sizes_in = [t.numel() for t in send]
    sizes_out = [int(torch.Size(s).numel()) for s in recv_shapes]
    out = torch.empty(sum(sizes_out), dtype=flat.dtype, device=flat.device)
    dist.all_to_all_single(out, flat, sizes_out, sizes_in, group=group)
    return [c.view(s) for c, s in zip(out.split(sizes_out), recv_shapes)]


def seq_to_heads(x: torch.Tensor, heads: int, tokens: int, group=None) -> torch.Tensor:
    """Token shard [B, n, H, ...] of every head -> all tokens [B, N, H_r, ...] of this rank's heads."""
    world, rank = _world(group)
    if world == 1:
        return x[:, :tokens]
    B, n = x.shape[0], x.shape[1]
    rest = tuple(x.shape[3:])
    send, shapes = [], []
    h0, h1 = head_range(heads, world, rank)
    for r in range(world):
        a, b = head_range(heads, world, r)
        send.append(x[:, :, a:b].contiguous())
        shapes.append((B, n, h1 - h0) + rest)
    parts = _all_to_all(send, shapes, group)
    return torch.cat(parts, dim=1)[:, :tokens].contiguous()


def heads_to_seq(o: torch.Tensor, heads: int, tokens: int, group=None) -> torch.Tensor:
    """All tokens [B, N, H_r, ...] of this rank's heads -> its token shard [B, n, H, ...] of every head
    (rows past N are zeros)."""
    world, rank = _world(group)
    if world == 1:
        return o
    B = o.shape[0]
    rest = tuple(o.shape[3:])
    _, n = token_shard(tokens, world, rank)
    padded = o.new_zeros((B, n * world) + tuple(o.shape[2:]))
    padded[:, :tokens] = o
    send, shapes = [], []
    for r in range(world):
        a, b = head_range(heads, world, r)
        send.append(padded[:, r * n:(r + 1) * n].contiguous())
        shapes.append((B, n, b - a) + rest)
    return torch.cat(_all_to_all(send, shapes, group), dim=2).contiguous()


def sharded_forward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, shape: Shape, topk_k: int,
                    scale: Optional[float] = None, g_coarse: Optional[torch.Tensor] = None,
                    g_fine: Optional[torch.Tensor] = None, group=None,
                    norm_rope: Optional[dict] = None,
                    attend: Optional[Callable] = None) -> torch.Tensor:
    """The attention call on token-sharded inputs (sequence parallelism).

    q, k, v: this rank's token shard [B, n, H, D] (n = ceil(N / world), rows past N are padding);
    gates [B, n, H] or None; `shape` describes the whole sequence.  `norm_rope`, if given, holds
    the keyword arguments of qk_norm_rope (w_q, w_k, eps, theta) and the pre-attention pass runs
    on the shard first.  Returns this rank's token shard [B, n, H, D] of the output."""
    world, rank = _world(group)
    H, N = shape.heads, shape.tokens
    offset, _ = token_shard(N, world, rank)
    if norm_rope is not None:
        q, k = qk_norm_rope(q, k, shape, token_offset=offset, **norm_rope)
    h0, h1 = head_range(H, world, rank)
    qh, kh, vh = (seq_to_heads(t, H, N, group) for t in (q, k, v))
    gc = seq_to_heads(g_coarse, H, N, group) if g_coarse is not None else None
    gf = seq_to_heads(g_fine, H, N, group) if g_fine is not None else None
    local = Shape(shape.batch, h1 - h0, shape.head_dim, shape.grid)
    if h1 > h0:
        run = attend if attend is not None else forward
        o = run(qh, kh, vh, local, topk_k, scale, gc, gf)
    else:   # more ranks than heads: this rank attends over nothing
        o = qh.new_zeros(qh.shape)
    return heads_to_seq(o, H, N, group)
