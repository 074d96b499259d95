"""World-size-2 data-parallel path on CPU (gloo): row sharding reproduces the
single-process result, and the bench's rank reductions (max / sum) work."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from lora_adapter_application_b200.shard import shard_rows


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    import oracle
    import workloads
    d = bench.Dist()
    d.init(backend="gloo")
    try:
        w = workloads.random_case(3, 37, 5, 48, [16, 8], 8, dtype=torch.bfloat16)
        lay = w.layers[0]
        lo, hi = shard_rows(w.T, world, rank)
        mine = oracle.lora_apply(lay.x, lay.A, lay.B, lay.col_off, w.ranks, w.alpha, w.ids, lay.y0,
                                 rows=np.arange(lo, hi, dtype=np.int32))
        parts = [None] * world
        torch.distributed.all_gather_object(parts, (lo, hi, mine))
        d.barrier()
        q.put((rank, parts, d.max(rank + 1.5), d.sum(rank + 1)))
    finally:
        d.close()


def test_shard_rows_partition():
    for T in (0, 1, 7, 64, 1000):
        for world in (1, 2, 3, 8):
            got = [shard_rows(T, world, r) for r in range(world)]
            assert got[0][0] == 0 and got[-1][1] == T
            assert all(a[1] == b[0] for a, b in zip(got, got[1:]))
            assert max(h - l for l, h in got) - min(h - l for l, h in got) <= 1
    with pytest.raises(ValueError):
        shard_rows(4, 2, 2)


def test_two_rank_gloo_matches_single_process():
    import oracle
    import workloads
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = [q.get(timeout=180) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    w = workloads.random_case(3, 37, 5, 48, [16, 8], 8, dtype=torch.bfloat16)
    lay = w.layers[0]
    full = oracle.lora_apply(lay.x, lay.A, lay.B, lay.col_off, w.ranks, w.alpha, w.ids, lay.y0)
    for rank, parts, mx, sm in results:
        assert mx == 2.5 and sm == 3.0
        stitched = np.concatenate([p[2] for p in sorted(parts, key=lambda p: p[0])])
        np.testing.assert_array_equal(stitched, full)
