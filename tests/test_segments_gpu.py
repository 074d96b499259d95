"""lora_build_segments on the GPU against the oracle's grouping: bit-exact."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_helpers import build_meta

pytestmark = pytest.mark.gpu


def _compare(ids, N, R, min_run, expect_status=None):
    ids_t = torch.as_tensor(np.asarray(ids, dtype=np.int32))
    meta, status = build_meta(ids_t, N, R, min_run)
    got = meta.host()
    ref = oracle.build_segments(ids_t.numpy(), N, R, min_run, 128,
                                meta.c.max_gather_tiles, meta.c.max_contig_tiles)
    np.testing.assert_array_equal(got["perm"], ref["perm"])
    np.testing.assert_array_equal(got["seg_start"], ref["seg_start"])
    np.testing.assert_array_equal(got["seg_adapter"], ref["seg_adapter"])
    for k in ["n_seg", "n_gather", "n_contig", "n_short"]:
        assert got[k] == ref[k], k
    np.testing.assert_array_equal(got["grow"], ref["grow"])
    np.testing.assert_array_equal(got["gather_tiles"], ref["gather_tiles"])
    np.testing.assert_array_equal(got["contig_tiles"], ref["contig_tiles"])
    st = int(status.item())
    assert st == ref["status"]
    if expect_status is not None:
        assert st == expect_status
    return got


@pytest.mark.parametrize("seed", range(12))
def test_random_batches(cuda_lib, seed):
    rng = np.random.default_rng(100 + seed)
    T = int(rng.choice([1, 5, 31, 64, 300, 1000, 2047, 2048, 2049, 4100, 9000, 20000]))
    N = int(rng.choice([1, 3, 17, 100, 1000]))
    if seed % 3 == 0:
        ids = rng.integers(-1, N, size=T)
    elif seed % 3 == 1:      # prompt-like runs
        lens = rng.integers(1, 300, size=max(1, T // 100))
        ids = np.repeat(rng.integers(-1, N, size=lens.shape[0]), lens)[:T]
        if ids.shape[0] < T:
            ids = np.concatenate([ids, rng.integers(-1, N, size=T - ids.shape[0])])
    else:                    # Zipf-like skew
        p = np.arange(1, N + 1, dtype=np.float64) ** -1.1
        ids = rng.choice(N, size=T, p=p / p.sum())
    _compare(ids, N, int(rng.choice([1, 7, 16])), int(rng.choice([0, 8, 64])), 0)


@pytest.mark.parametrize("ids,N", [
    ([], 3), ([-1] * 7, 2), ([1] * 5000, 2), ([0], 1), ([-1] * 3000 + [0] + [-1] * 3000, 1),
    ([3, -1, -1, 3], 4), ([0] * 2048, 1), ([0] * 2049, 1)])
def test_edge_cases(cuda_lib, ids, N):
    _compare(ids, N, 16, 64, 0)


def test_bad_ids_are_flagged_and_skipped(cuda_lib):
    ids = [0, 1, 7, -3, 1, 1, -1, 2]
    got = _compare(ids, 3, 2, 0, expect_status=1)
    assert 2 not in got["grow"] and 3 not in got["grow"]
    big = np.random.default_rng(3).integers(-1, 5, size=5000)
    big[[17, 4000]] = [9, -2]
    _compare(big, 5, 16, 8, expect_status=1)


@pytest.mark.parametrize("name", ["tiny", "decode_qproj", "prefill", "multislice_8b", "mixed_70b"])
def test_workload_ids(cuda_lib, name):
    gen = {"tiny": lambda: workloads.tiny(),
           "decode_qproj": lambda: workloads.decode_qproj(),
           "prefill": lambda: workloads.prefill(d=8),
           "multislice_8b": lambda: workloads.multislice_8b(N=100, hidden=8, kv=8, inter=8),
           "mixed_70b": lambda: workloads.mixed_70b(hidden=8, inter=8)}[name]
    w = gen()
    _compare(w.ids.numpy(), w.N, 16, 64, 0)


def test_deterministic(cuda_lib):
    ids = torch.as_tensor(np.random.default_rng(9).integers(-1, 50, size=30000).astype(np.int32))
    a, _ = build_meta(ids, 50, 16, 8)
    b, _ = build_meta(ids, 50, 16, 8)
    ha, hb = a.host(), b.host()
    for k in ha:
        np.testing.assert_array_equal(np.asarray(ha[k]), np.asarray(hb[k]))


@pytest.mark.parametrize("T,N,min_run,seed", [
    (5000, 3, 64, 1), (20000, 7, 1000, 2), (50000, 40, 64, 3), (131072, 4096, 128, 4),
    (131072, 9, 1, 5), (70000, 2, 2048, 6)])
def test_long_runs_across_blocks(cuda_lib, T, N, min_run, seed):
    """Runs of up to 6000 rows: many straddle or span the 2048-position blocks
    of the multi-block tile passes; ids -1 and short runs in between."""
    rng = np.random.default_rng(500 + seed)
    parts = []
    while sum(len(p) for p in parts) < T:
        L = int(rng.choice([1, 3, 40, 129, 700, 2047, 2049, 6000]))
        parts.append(np.full(L, int(rng.integers(-1, N)), dtype=np.int32))
    ids = np.concatenate(parts)[:T]
    _compare(ids, N, int(rng.choice([1, 16])), min_run, 0)


@pytest.mark.parametrize("T,N", [(2049, 24), (4100, 24), (8192, 24), (8192, 1023),
                                 (5000, 2000), (8192, 4096)])
def test_grouping_one_block_and_multi_block_bounds(cuda_lib, T, N):
    """Around the bounds of the one-block grouping (up to 8192 rows when N <= 1023)
    and the multi-block passes (more ids): decode-like ids, prompt runs, -1 rows."""
    rng = np.random.default_rng(T + N)
    parts, n = [], 0
    while n < T:
        L = int(rng.choice([1, 2, 70, 300, 129]))
        parts.append(np.full(L, int(rng.integers(-1, N)), dtype=np.int32))
        n += L
    ids = np.concatenate(parts)[:T]
    for min_run in (0, 64):
        _compare(ids, N, 16, min_run, 0)
