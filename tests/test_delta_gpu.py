"""Delta application on the GPU against the fp64 oracle, element by element.

Tolerances (the method's): bf16 in / fp32 accumulate: |gpu - oracle| <=
1e-2 * max(1, |oracle|); fp32: 1e-4 * max(1, |oracle|).  Rows without an
adapter must come back bit-identical.
"""
import numpy as np
import pytest
import torch

import lora_adapter_application_b200 as lora
import oracle
import workloads
from gpu_helpers import DeviceLayer, assert_within, build_meta, oracle_rows, run_fused

pytestmark = pytest.mark.gpu

ENTRY = {"add_linear": lora.lora_add_linear, "bgmv_fused": lora.lora_bgmv_fused}


def _check_full(w, layer_idx=0, fn="add_linear", R=16, min_run=64):
    lay = w.layers[layer_idx]
    dl = DeviceLayer(lay)
    meta, status = build_meta(w.ids, w.N, R, min_run)
    y = run_fused(w, dl, meta, status, ENTRY[fn]).cpu()
    assert int(status.item()) == 0
    ref = oracle_rows(w, lay, None)
    assert_within(y.to(torch.float64).numpy(), ref, w.dtype, f"{w.name}/{fn}")
    none = (w.ids < 0).numpy()
    assert torch.equal(y[none], lay.y0[none])
    return y


SMALL = [
    # seed, T, N, d_in, d_out, r_max, ranks
    (1, 37, 5, 200, [96, 40], 16, [16, 3, 5, 8, 1]),
    (2, 130, 3, 64, 64, 8, None),
    (3, 64, 7, 1000, [24, 8, 8], 32, None),
    (4, 300, 4, 512, 384, 64, [64, 8, 33, 17]),
    (5, 17, 2, 8, 2, 4, [1, 4]),
]


@pytest.mark.parametrize("case", SMALL)
@pytest.mark.parametrize("fn", ["add_linear", "bgmv_fused"])
@pytest.mark.parametrize("R", [16, 64])
def test_small_bf16_cases(cuda_lib, case, fn, R):
    seed, T, N, d_in, d_out, r_max, ranks = case
    w = workloads.random_case(seed, T, N, d_in, d_out, r_max, ranks=ranks, dtype=torch.bfloat16)
    _check_full(w, fn=fn, R=R, min_run=0)


@pytest.mark.parametrize("r_max", [24, 32, 64])
@pytest.mark.parametrize("blocks", ["1", "3", "0"])
def test_ranks_17_to_24(cuda_lib, r_max, blocks, monkeypatch):
    """Ranks 17-24 (24 loaded ranks, the tail past r_n zero-filled: two m16 rank
    tiles in the shrink, one 32-rank chunk with a partly read lane in the expand)
    over 4096 columns, on one block, three blocks and the full grid."""
    monkeypatch.setenv("LORA_BG_BLOCKS", blocks)
    ranks = [17 + (i % 8) for i in range(12)]
    w = workloads.random_case(41, 256, 12, 4096, [4096], r_max, ranks=ranks, none_frac=0.05,
                              dtype=torch.bfloat16)
    _check_full(w, fn="bgmv_fused", R=64, min_run=0)


@pytest.mark.parametrize("R,min_run", [(16, 8), (5, 0), (1, 0), (16, 200), (64, 0), (64, 8), (37, 16)])
def test_tiles_and_runs(cuda_lib, R, min_run):
    """Long same-adapter segments over several tiles, prompt-like runs that become
    contiguous tiles, and ragged tails."""
    w = workloads.random_case(21, 400, 6, 136, [72, 24], 16,
                              runs=[(70, 2), (9, -1), (130, 5), (3, 2), (40, 0)],
                              dtype=torch.bfloat16)
    _check_full(w, R=R, min_run=min_run)


def test_fp32_tiny_workload(cuda_lib):
    w = workloads.tiny()
    _check_full(w)
    _check_full(w, fn="bgmv_fused", R=3, min_run=4)


def test_bf16_unaligned_takes_general_kernel(cuda_lib):
    w = workloads.random_case(31, 45, 3, 203, 77, 6, dtype=torch.bfloat16)
    _check_full(w, min_run=0)


def test_rank_above_64(cuda_lib):
    w = workloads.random_case(32, 40, 3, 128, 64, 128, ranks=[128, 100, 7],
                              dtype=torch.bfloat16)
    _check_full(w, min_run=0)


def test_strided_rows_and_offsets(cuda_lib):
    """x and y rows wider than the data (ld > width), slices at column offsets."""
    w = workloads.random_case(33, 50, 4, 96, [32, 16], 8, dtype=torch.bfloat16)
    lay = w.layers[0]
    g = torch.Generator().manual_seed(5)
    xw = torch.randn(w.T, 120, generator=g).to(torch.bfloat16)
    xw[:, :96] = lay.x
    yw = torch.randn(w.T, 72, generator=g).to(torch.bfloat16)
    col_off = [8, 48]
    meta, status = build_meta(w.ids, w.N, 16, 0)
    ranks, alphas = w.ranks.cuda(), lora.alphas_full(w.alpha, w.N)
    y = yw.cuda()
    lora.lora_add_linear(y, xw.cuda()[:, :96], [a.cuda() for a in lay.A],
                         [b.cuda() for b in lay.B], col_off, ranks, alphas, meta, status)
    torch.cuda.synchronize()
    ref = oracle.lora_apply(xw, lay.A, lay.B, col_off, w.ranks, w.alpha, w.ids, yw)
    assert_within(y.cpu().double().numpy(), ref, torch.bfloat16, "strided")
    # columns outside the slices are untouched
    untouched = [c for c in range(72) if not (8 <= c < 40 or 48 <= c < 64)]
    assert torch.equal(y.cpu()[:, untouched], yw[:, untouched])


def test_bad_rank_is_flagged_and_rows_untouched(cuda_lib):
    w = workloads.random_case(34, 30, 3, 64, 32, 8, ranks=[8, 8, 8], none_frac=0.0,
                              dtype=torch.bfloat16)
    lay = w.layers[0]
    dl = DeviceLayer(lay)
    meta, status = build_meta(w.ids, w.N, 16, 0)
    ranks = torch.tensor([8, 9, 8], dtype=torch.int32).cuda()   # 9 > r_max
    alphas = lora.alphas_full(w.alpha, w.N)
    y = dl.y0.clone()
    lora.lora_add_linear(y, dl.x, dl.A, dl.B, dl.col_off, ranks, alphas, meta, status)
    torch.cuda.synchronize()
    assert int(status.item()) & lora.DEV_BAD_RANK
    rows1 = (w.ids == 1)
    assert torch.equal(y.cpu()[rows1], lay.y0[rows1])
    ref = oracle_rows(w, lay, None)
    ok = (~rows1).numpy()
    assert_within(y.cpu().double().numpy()[ok], ref[ok], torch.bfloat16, "bad rank")


def test_shrink_then_expand_matches_oracle(cuda_lib):
    w = workloads.random_case(35, 90, 5, 256, [64, 32, 32], 16, ranks=[16, 8, 3, 16, 12],
                              runs=[(70, 1)], dtype=torch.bfloat16)
    lay = w.layers[0]
    dl = DeviceLayer(lay)
    for min_run in (0, 16):
        meta, status = build_meta(w.ids, w.N, 16, min_run)
        v = torch.full((3, w.T, w.r_max), float("nan"), device="cuda")
        ranks, alphas = w.ranks.cuda(), lora.alphas_full(w.alpha, w.N)
        lora.lora_sgmv_shrink(v, dl.x, dl.A, ranks, meta, status)
        torch.cuda.synchronize()
        vref = oracle.lora_shrink(lay.x, lay.A, w.ranks, w.ids)          # [T, S, r_max]
        vg = v.cpu().double().permute(1, 0, 2).numpy()
        for i in range(w.T):
            n = int(w.ids[i])
            if n < 0:
                assert np.isnan(vg[i]).all()        # rows without an adapter: not written
                continue
            r = int(w.ranks[n])
            assert_within(vg[i, :, :r], vref[i, :, :r], torch.float32, f"v row {i}")
        # expand from the oracle's v gives the oracle's y
        vin = torch.as_tensor(vref, dtype=torch.float32).permute(1, 0, 2).contiguous().cuda()
        y = dl.y0.clone()
        lora.lora_sgmv_expand(y, vin, dl.B, dl.col_off, ranks, alphas, meta, status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert_within(y.cpu().double().numpy(), oracle_rows(w, lay, None), torch.bfloat16, "expand")
        # and shrink -> expand on the GPU equals the fused kernel within tolerance
        y2 = dl.y0.clone()
        lora.lora_sgmv_expand(y2, v, dl.B, dl.col_off, ranks, alphas, meta, status)
        torch.cuda.synchronize()
        assert_within(y2.cpu().double().numpy(), oracle_rows(w, lay, None), torch.bfloat16, "pair")


def test_fused_is_deterministic(cuda_lib):
    w = workloads.random_case(36, 500, 9, 512, 256, 16, dtype=torch.bfloat16)
    dl = DeviceLayer(w.layers[0])
    meta, status = build_meta(w.ids, w.N, 16, 0)
    a = run_fused(w, dl, meta, status)
    b = run_fused(w, dl, meta, status)
    assert torch.equal(a, b)


# ------------------------------------------------------------------ full-size workloads

def _full_size(w, layer_idx, R=64, min_run=64):
    """Every row of a full-size workload layer against the oracle (fp64, OpenMP over
    the host cores); rows without an adapter bit-identical."""
    lay = w.layers[layer_idx]
    dl = DeviceLayer(lay)
    meta, status = build_meta(w.ids, w.N, R, min_run)
    y = run_fused(w, dl, meta, status).cpu()
    assert int(status.item()) == 0
    ref = oracle_rows(w, lay, None)
    assert_within(y.double().numpy(), ref, w.dtype, f"{w.name}/{lay.name}")
    none = (w.ids < 0)
    assert torch.equal(y[none], lay.y0[none])
    return y, dl, meta, status


def test_decode_qproj_full(cuda_lib):
    w = workloads.decode_qproj()
    _check_full(w, R=64, min_run=0)
    _check_full(w, R=16, min_run=0)


def _launch(w, launch, min_run):
    """Segment parameters: the ones bench.py times the workload with, or 64-row
    gathered tiles with the given shortest run."""
    if launch == "bench":
        import bench
        return bench.segment_params(w)
    return 64, min_run


@pytest.mark.parametrize("launch", ["bench", "R64"])
def test_prefill_full(cuda_lib, launch):
    w = workloads.prefill()
    R, min_run = _launch(w, launch, 64)
    _full_size(w, 0, R=R, min_run=min_run)


@pytest.mark.parametrize("launch", ["bench", "R64"])
@pytest.mark.parametrize("layer_idx", [0, 1, 2, 3])
def test_multislice_8b_full(cuda_lib, layer_idx, launch):
    w = workloads.multislice_8b()
    R, min_run = _launch(w, launch, 0)
    _full_size(w, layer_idx, R=R, min_run=min_run)


@pytest.mark.parametrize("launch", ["bench", "R64"])
@pytest.mark.parametrize("layer_idx", [0, 1])
def test_mixed_70b_full(cuda_lib, layer_idx, launch):
    """bench.py's launch: 32-row tiles without contiguous runs, every row of both
    layers on the gathered-tile kernel in one launch; R64: 64-row tiles with the
    prompts as contiguous tiles."""
    w = workloads.mixed_70b()
    R, min_run = _launch(w, launch, 64)
    _full_size(w, layer_idx, R=R, min_run=min_run)
