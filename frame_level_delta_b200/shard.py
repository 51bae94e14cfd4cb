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
