"""Head sharding of one stream across ranks (one process per GPU).

Every step of the path is independent across heads: the 3D RoPE, the append,
the re-rotations, the attention and the per-head score pass. Rank r of G
therefore owns the contiguous head range head_ranges(H, G)[r] of every
layer's cache and runs the whole step on it; the integer cache state is
computed identically on every rank, so nothing about it is exchanged. The one
exchange is Deep-Forcing top-C (rCM length-extrapolation guide, strategy 4):
a token's score sums over all heads, so the ranks all-reduce (sum) their score
vectors and each selects top-C from the sum with rc_select_topc.
"""
from typing import List, Tuple


def head_ranges(heads: int, world: int) -> List[Tuple[int, int]]:
    """Contiguous, balanced head ranges [h0, h1) for ranks 0..world-1.

    The first heads % world ranks get one head more; a rank may get none when
    world > heads.
    """
    if heads < 0 or world < 1:
        raise ValueError("heads >= 0 and world >= 1 required")
    base, extra = divmod(heads, world)
    out, h = [], 0
    for r in range(world):
        n = base + (1 if r < extra else 0)
        out.append((h, h + n))
        h += n
    return out


def sharded_scores_topc(cache, layer: int, scores_local, C: int, topc=None, group=None):
    """Sum this rank's token-score vector over the process group (in place,
    its first n_candidates entries) and select top-C from the sum.
    scores_local: fp32 on this rank's device, as rc_step wrote it for the
    rank's heads. Every rank calls this at the same step (one collective)."""
    import torch.distributed as dist
    n = cache.state(layer).n_candidates
    if n > 0 and dist.is_available() and dist.is_initialized():
        dist.all_reduce(scores_local[:n], op=dist.ReduceOp.SUM, group=group)
    return cache.select_topc(layer, scores_local, C, topc)
