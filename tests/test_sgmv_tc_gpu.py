"""Tensor-core SGMV (contiguous tiles of prompt-like runs) against the fp64 oracle.

Runs of at least min_run rows with one adapter become contiguous tiles of up to
128 rows; lora_add_linear, lora_sgmv_shrink and lora_sgmv_expand send those to
the tcgen05 kernel (page "Multi-LoRA Serving", sections 3.2 and 3.4).  Every
row of every case is compared with the oracle; rows without an adapter must
come back bit-identical.  LORA_TC_CLUSTER forces the number of thread blocks
per tile, so the distributed-shared-memory exchange runs with 1, 2, 4 and 8
blocks.
"""
import numpy as np
import pytest
import torch

import lora_adapter_application_b200 as lora
import oracle
import workloads
from gpu_helpers import DeviceLayer, assert_within, build_meta, kernels_of, oracle_rows, run_fused

pytestmark = pytest.mark.gpu

RUNS = [(300, 0), (129, 1), (9, -1), (128, 2), (20, 3), (3, 1), (64, -1), (47, 2)]
RUNS3 = [(300, 0), (129, 1), (9, -1), (128, 2), (20, 0), (3, 1), (64, -1), (47, 2)]

# name, seed, T, N, d_in, d_out, r_max, ranks, runs, clusters (the sizes whose exchange
# buffers still fit shared memory with the ring: 2 x C x n_slices x r_max x 512 bytes)
CASES = [
    ("q_proj", 1, 800, 4, 512, 512, 16, [16, 16, 16, 16], RUNS, (1, 2, 4)),
    ("qkv_masked_ranks", 2, 700, 3, 256, [128, 64, 64], 16, [16, 5, 12], RUNS3, (1, 2)),
    ("ragged_r32", 3, 760, 4, 200, [200, 72], 32, [32, 17, 9, 24], RUNS, (1,)),
    ("ragged_r16", 9, 760, 4, 200, [200, 72], 16, [16, 11, 9, 3], RUNS, (1, 2)),
    ("two_slices_r64", 4, 760, 4, 1024, [256, 256], 64, [64, 8, 40, 33], RUNS, (1,)),
    ("rank128", 5, 700, 2, 384, 136, 128, [128, 100], [(400, 0), (150, 1), (150, -1)], (1,)),
    ("narrow", 6, 300, 2, 64, 8, 16, [16, 7], [(200, 0), (100, 1)], (1,)),
    ("tail_at_T", 7, 333, 3, 256, 256, 16, None, [(40, -1), (293, 2)], (1, 2)),
    ("cluster8", 8, 600, 3, 1024, 1024, 16, [16, 16, 11], [(260, 0), (200, 1), (140, 2)], (8, 4)),
]


def _case(c):
    name, seed, T, N, d_in, d_out, r_max, ranks, runs, _ = c
    return workloads.random_case(seed, T, N, d_in, d_out, r_max, ranks=ranks, runs=runs,
                                 dtype=torch.bfloat16)


def _ids(c):
    return c[0]


def _kernels_of(fn):
    """Names of the CUDA kernels fn launches (fn may run more than once)."""
    out, kernels, _ = kernels_of(fn)
    return out, set(kernels)


def _on_tensor_cores(names):
    return any("sgmv_tc_kernel" in n for n in names)


@pytest.mark.parametrize("case", CASES, ids=_ids)
def test_add_linear_contiguous_tiles(cuda_lib, case, monkeypatch):
    w = _case(case)
    lay = w.layers[0]
    dl = DeviceLayer(lay)
    ref = oracle_rows(w, lay, None)
    none = (w.ids < 0)
    for C in case[-1]:
        monkeypatch.setenv("LORA_TC_CLUSTER", str(C))
        meta, status = build_meta(w.ids, w.N, 16, 16)
        y, names = _kernels_of(lambda: run_fused(w, dl, meta, status).cpu())
        assert _on_tensor_cores(names), f"C={C}: no tensor-core launch in {sorted(names)}"
        assert int(status.item()) == 0, f"status {int(status.item())} with C={C}"
        assert_within(y.double().numpy(), ref, torch.bfloat16, f"{case[0]} C={C}")
        assert torch.equal(y[none], lay.y0[none])


@pytest.mark.parametrize("C", [1, 2])
def test_shrink_expand_contiguous_tiles(cuda_lib, C, monkeypatch):
    monkeypatch.setenv("LORA_TC_CLUSTER", str(C))
    w = workloads.random_case(11, 500, 4, 384, [128, 64], 16, ranks=[16, 12, 9, 16],
                              runs=[(200, 0), (130, 1), (40, 2), (100, 3), (30, -1)],
                              dtype=torch.bfloat16)
    lay = w.layers[0]
    dl = DeviceLayer(lay)
    meta, status = build_meta(w.ids, w.N, 16, 16)
    ranks, alphas = w.ranks.cuda(), lora.alphas_full(w.alpha, w.N)
    v = torch.full((2, w.T, w.r_max), float("nan"), device="cuda")
    _, names = _kernels_of(lambda: lora.lora_sgmv_shrink(v, dl.x, dl.A, ranks, meta, status))
    assert _on_tensor_cores(names), sorted(names)
    assert int(status.item()) == 0
    vref = oracle.lora_shrink(lay.x, lay.A, w.ranks, w.ids)            # [T, S, r_max]
    vg = v.cpu().double().permute(1, 0, 2).numpy()
    for i in range(w.T):
        n = int(w.ids[i])
        if n < 0:
            assert np.isnan(vg[i]).all()
            continue
        r = int(w.ranks[n])
        assert_within(vg[i, :, :r], vref[i, :, :r], torch.float32, f"v row {i}")
        assert np.isnan(vg[i, :, r:]).all()                            # k >= r_n not written
    vin = torch.as_tensor(vref, dtype=torch.float32).permute(1, 0, 2).contiguous().cuda()
    y = dl.y0.clone()

    def expand():                                     # y += ...: start from y0 on every run
        y.copy_(dl.y0)
        lora.lora_sgmv_expand(y, vin, dl.B, dl.col_off, ranks, alphas, meta, status)

    _, names = _kernels_of(expand)
    assert _on_tensor_cores(names), sorted(names)
    assert int(status.item()) == 0
    assert_within(y.cpu().double().numpy(), oracle_rows(w, lay, None), torch.bfloat16, "expand")


def test_contiguous_bad_rank_flagged(cuda_lib):
    w = workloads.random_case(12, 400, 3, 256, 256, 16, ranks=[16, 16, 16],
                              runs=[(150, 0), (150, 1), (100, 2)], dtype=torch.bfloat16)
    lay = w.layers[0]
    dl = DeviceLayer(lay)
    meta, status = build_meta(w.ids, w.N, 16, 16)
    ranks = torch.tensor([16, 17, 16], dtype=torch.int32).cuda()      # 17 > r_max
    alphas = lora.alphas_full(w.alpha, w.N)
    y = dl.y0.clone()
    lora.lora_add_linear(y, dl.x, dl.A, dl.B, dl.col_off, ranks, alphas, meta, status)
    torch.cuda.synchronize()
    assert int(status.item()) & lora.DEV_BAD_RANK
    rows1 = (w.ids == 1)
    assert torch.equal(y.cpu()[rows1], lay.y0[rows1])
    ok = (~rows1).numpy()
    ref = oracle_rows(w, lay, None)
    assert_within(y.cpu().double().numpy()[ok], ref[ok], torch.bfloat16, "bad rank")


def test_contiguous_deterministic(cuda_lib):
    w = _case(CASES[0])
    dl = DeviceLayer(w.layers[0])
    meta, status = build_meta(w.ids, w.N, 16, 16)
    a = run_fused(w, dl, meta, status)
    b = run_fused(w, dl, meta, status)
    assert torch.equal(a, b)


def test_tensor_core_kernel_runs(cuda_lib):
    """The contiguous tiles really take the tcgen05 kernel (kernel names from the profiler)."""
    w = _case(CASES[0])
    dl = DeviceLayer(w.layers[0])
    meta, status = build_meta(w.ids, w.N, 16, 16)
    run_fused(w, dl, meta, status)
    _, names = _kernels_of(lambda: run_fused(w, dl, meta, status))
    assert _on_tensor_cores(names), sorted(names)
    # a decode-only grouping (min_run = 0) never launches it
    meta0, status0 = build_meta(w.ids, w.N, 16, 0)
    _, names = _kernels_of(lambda: run_fused(w, dl, meta0, status0))
    assert not _on_tensor_cores(names), sorted(names)


def test_captured_graph_matches_eager(cuda_lib):
    """lora_add_linear inside a CUDA graph (the side-stream fork and join are captured
    too) gives bit-identical results to eager calls, replay after replay."""
    w = _case(CASES[0])          # prompt runs and decode rows: both kernels, both streams
    dl = DeviceLayer(w.layers[0])
    meta, status = build_meta(w.ids, w.N, 16, 16)
    ranks, alphas = w.ranks.cuda(), lora.alphas_full(w.alpha, w.N)
    eager = dl.y0.clone()
    lora.lora_add_linear(eager, dl.x, dl.A, dl.B, dl.col_off, ranks, alphas, meta, status)
    torch.cuda.synchronize()
    y = dl.y0.clone()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        lora.lora_add_linear(y, dl.x, dl.A, dl.B, dl.col_off, ranks, alphas, meta, status,
                             stream=s)
    for _ in range(2):
        y.copy_(dl.y0)
        g.replay()
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert torch.equal(y, eager)
    del g
