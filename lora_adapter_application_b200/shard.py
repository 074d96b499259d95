"""Row sharding across data-parallel ranks.

Every row of a batch is computed on its own (page "Multi-LoRA Serving",
section 2: the delta of row i depends only on x_i and its adapter), so a batch
splits across ranks by contiguous row ranges with no exchange between ranks.
"""


def shard_rows(T: int, world: int, rank: int):
    """Contiguous [lo, hi) rows of a T-row batch owned by `rank` of `world`."""
    if not (0 <= rank < world) or T < 0:
        raise ValueError("bad shard request")
    base, extra = divmod(T, world)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)
