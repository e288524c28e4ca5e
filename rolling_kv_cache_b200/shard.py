"""Head sharding of one stream across ranks (one process per GPU).

Every step of the path is independent across heads: the 3D RoPE, the append,
the re-rotations, the attention and the per-head score pass. Rank r of G
therefore owns the contiguous head range head_ranges(H, G)[r] of every
layer's cache and runs the whole step on it; the integer cache state is
computed identically on every rank, so nothing about it is exchanged. The one
exchange is Deep-Forcing top-C (rCM length-extrapolation guide, strategy 4):
a token's score sums over all heads, so the ranks all-reduce (sum) their score
vectors and each selects top-C from the sum with rc_select_topc.

Callers whose activations are sharded by sequence instead (each rank holds a
block of the chunk's tokens with every head, as the LingBot explainer's
Ulysses-style sequence parallelism does) swap them with one all-to-all before
the step (seq_to_heads) and one after it (heads_to_seq); both move
n_tokens * H * d / world elements per rank over NCCL.
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


def token_ranges(n_tokens: int, world: int) -> List[Tuple[int, int]]:
    """Contiguous token blocks of a sequence-sharded chunk (same rule as heads)."""
    return head_ranges(n_tokens, world)


def seq_to_heads(x_seq, heads: int, group=None):
    """Ulysses swap before the step: this rank's token block with every head,
    [n_local, H, d], becomes every token of this rank's head range,
    [n_tokens, h1 - h0, d] (token blocks in rank order). One all-to-all."""
    import torch
    import torch.distributed as dist
    world, rank = dist.get_world_size(group), dist.get_rank(group)
    hr = head_ranges(heads, world)
    n_loc, d = x_seq.shape[0], x_seq.shape[2]
    sizes = torch.tensor([n_loc], dtype=torch.int64)
    counts = [torch.zeros(1, dtype=torch.int64) for _ in range(world)]
    dist.all_gather(counts, sizes, group=group)
    n_by_rank = [int(c.item()) for c in counts]
    h0, h1 = hr[rank]
    send = torch.cat([x_seq[:, a:b].reshape(-1) for a, b in hr]).contiguous()
    recv = torch.empty(sum(n_by_rank) * (h1 - h0) * d, dtype=x_seq.dtype, device=x_seq.device)
    dist.all_to_all_single(recv, send, output_split_sizes=[n * (h1 - h0) * d for n in n_by_rank],
                           input_split_sizes=[n_loc * (b - a) * d for a, b in hr], group=group)
    return recv.view(sum(n_by_rank), h1 - h0, d)


def heads_to_seq(x_heads, heads: int, n_local: int, group=None):
    """Ulysses swap after the step: every token of this rank's head range,
    [n_tokens, h1 - h0, d], back to this rank's token block with every head,
    [n_local, H, d]. One all-to-all."""
    import torch
    import torch.distributed as dist
    world, rank = dist.get_world_size(group), dist.get_rank(group)
    hr = head_ranges(heads, world)
    h0, h1 = hr[rank]
    d = x_heads.shape[2]
    sizes = torch.tensor([n_local], dtype=torch.int64)
    counts = [torch.zeros(1, dtype=torch.int64) for _ in range(world)]
    dist.all_gather(counts, sizes, group=group)
    n_by_rank = [int(c.item()) for c in counts]
    send = x_heads.contiguous().view(-1)
    recv = torch.empty(n_local * heads * d, dtype=x_heads.dtype, device=x_heads.device)
    dist.all_to_all_single(recv, send, output_split_sizes=[n_local * (b - a) * d for a, b in hr],
                           input_split_sizes=[n * (h1 - h0) * d for n in n_by_rank], group=group)
    parts, off = [], 0
    for a, b in hr:
        sz = n_local * (b - a) * d
        parts.append(recv[off:off + sz].view(n_local, b - a, d))
        off += sz
    return torch.cat(parts, dim=1)
