"""Head sharding of the packed attention forward across ranks.

The forward has no exchange step: every (segment, head) unit is independent.
With the tensor-parallel layout of the upstream QKV projection, rank r of N
holds heads [r*H/N, (r+1)*H/N) of q, k, v as its own contiguous
``[T, H/N, d]`` tensors and calls ``pa_varlen_attn_fwd`` on them with the full
``cu_seqlens`` — no collective is needed.  ``gather_heads`` is the one
collective a caller may want afterwards (the full ``[T, H, d]`` output on every
rank); it is plumbing (torch.distributed), not part of the attention path.
"""


def head_range(heads, world, rank):
    """[start, stop) of the heads owned by ``rank``; balanced to within one head."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("invalid rank / world")
    base, extra = divmod(int(heads), int(world))
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def gather_heads(local, heads, group=None):
    """All-gather per-rank ``[T, h_r, ...]`` shards into the full ``[T, heads, ...]`` tensor.

    Shards differ by at most one head; each is padded to the largest shard for the
    collective (which needs equal sizes) and trimmed afterwards.
    """
    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group)
    ranges = [head_range(heads, world, r) for r in range(world)]
    width = max(b - a for a, b in ranges)
    shape = (local.shape[0], width) + tuple(local.shape[2:])
    send = torch.zeros(shape, dtype=local.dtype, device=local.device)
    send[:, :local.shape[1]] = local
    parts = [torch.empty(shape, dtype=local.dtype, device=local.device) for _ in range(world)]
    dist.all_gather(parts, send, group=group)
    return torch.cat([part[:, :b - a] for part, (a, b) in zip(parts, ranges)], dim=1)
