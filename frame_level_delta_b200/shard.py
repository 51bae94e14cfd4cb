"""Head sharding across GPUs: which heads each rank serves.

Heads of the linear branch are independent (every step of the path works per
(batch, head)), so a batch's heads can be split across ranks with no exchange:
each rank runs a context over its head slice of the shared token tensors
(vda_config.H_total, h0). The pages shard their attention by heads across GPUs
(Ulysses style), with an uneven split between the two branches (VDN-H3 post,
section "benchmark": a 5:3 split); ``weights`` gives such uneven shares.
"""
from __future__ import annotations

from typing import List, Optional, Sequence, Tuple


def head_partition(H: int, world: int, weights: Optional[Sequence[float]] = None) -> List[Tuple[int, int]]:
    """Split heads 0..H-1 into `world` contiguous slices (h0, n), in rank order.

    Even by default (the first H % world ranks take one head more). With
    `weights`, rank r's share is proportional to weights[r] (largest remainders
    get the leftover heads). Every rank gets at least one head, so H >= world.
    """
    if world < 1 or H < world:
        raise ValueError(f"cannot split {H} heads over {world} ranks with at least one head each")
    if weights is None:
        weights = [1.0] * world
    if len(weights) != world or any(w <= 0 for w in weights):
        raise ValueError("weights: one positive share per rank")
    total = float(sum(weights))
    exact = [H * w / total for w in weights]
    counts = [max(1, int(x)) for x in exact]
    while sum(counts) > H:  # the max(1, .) floors can overshoot when shares are tiny
        i = max((r for r in range(world) if counts[r] > 1), key=lambda r: (counts[r] - exact[r], counts[r]))
        counts[i] -= 1
    order = sorted(range(world), key=lambda r: (exact[r] - counts[r], -r), reverse=True)
    k = 0
    while sum(counts) < H:
        counts[order[k % world]] += 1
        k += 1
    out, h0 = [], 0
    for n in counts:
        out.append((h0, n))
        h0 += n
    return out


def seq_to_heads(x_seq, parts, group=None):
    """Ulysses exchange, sequence shards to head shards: every rank holds its
    contiguous token range of all heads, x_seq [B, n, H, d] (the same n on every
    rank); afterwards each rank holds every token of its own heads,
    [B, world * n, n_r, d] with (h0_r, n_r) = parts[rank] (uneven splits allowed).
    One all_to_all_single over the process group (NCCL between GPUs)."""
    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    B, n, H, d = x_seq.shape
    send = torch.cat([x_seq[:, :, h0:h0 + k].reshape(-1) for (h0, k) in parts])
    n_r = parts[rank][1]
    recv = torch.empty(world * B * n * n_r * d, dtype=x_seq.dtype, device=x_seq.device)
    dist.all_to_all_single(recv, send, output_split_sizes=[B * n * n_r * d] * world,
                           input_split_sizes=[B * n * k * d for (_, k) in parts], group=group)
    # recv holds, source rank by source rank, [B, n, n_r, d]: token order is rank order.
    return recv.view(world, B, n, n_r, d).permute(1, 0, 2, 3, 4).reshape(B, world * n, n_r, d)


def heads_to_seq(x_heads, parts, group=None):
    """The inverse exchange: [B, world * n, n_r, d] (every token, this rank's
    heads) back to [B, n, H, d] (this rank's tokens, every head)."""
    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group)
    B, N, n_r, d = x_heads.shape
    n = N // world
    H = sum(k for _, k in parts)
    send = x_heads.view(B, world, n, n_r, d).permute(1, 0, 2, 3, 4).reshape(-1)
    recv = torch.empty(B * n * H * d, dtype=x_heads.dtype, device=x_heads.device)
    dist.all_to_all_single(recv, send, output_split_sizes=[B * n * k * d for (_, k) in parts],
                           input_split_sizes=[B * n * n_r * d] * world, group=group)
    out = torch.empty(B, n, H, d, dtype=x_heads.dtype, device=x_heads.device)
    off = 0
    for (h0, k) in parts:
        sz = B * n * k * d
        out[:, :, h0:h0 + k] = recv[off:off + sz].view(B, n, k, d)
        off += sz
    return out
