"""Contracts of the fused delta path on the GPU, each against the fp64 oracle:

* padding ranks (A rows and B columns k >= r_n, and v entries k >= r_n given to
  the expand) may hold anything, NaN included, without changing the result;
* each adapter's delta is scaled by its own alpha_n / r_n, computed on the device;
* one workspace serves call after call (its head is back at zero after each);
* tiles whose partial sums exceed one exchange are reduced in several passes,
  and wide layers stream their slices in groups;
* the launch-shape overrides change nothing beyond rounding order;
* calls on two streams, and a CUDA graph replayed with new ids, stay exact.

Tolerance (the method's): bf16 |gpu - oracle| <= 1e-2 * max(1, |oracle|), fp32 1e-4.
"""
import threading

import numpy as np
import pytest
import torch

import lora_adapter_application_b200 as lora
import oracle
import workloads
from gpu_helpers import DeviceLayer, assert_within, build_meta, oracle_rows

pytestmark = pytest.mark.gpu


def _poisoned(lay, ranks, value=float("nan")):
    """Device copies of a layer's adapters with every padding rank set to `value`."""
    A = [a.clone() for a in lay.A]
    B = [b.clone() for b in lay.B]
    for n, r in enumerate(ranks.tolist()):
        for a in A:
            a[n, r:, :] = value
        for b in B:
            b[n, :, r:] = value
    return [a.cuda() for a in A], [b.cuda() for b in B]


def _apply(fn, w, lay, A, B, meta, status, alphas=None, y0=None):
    y = (lay.y0 if y0 is None else y0).cuda().clone()
    alphas = lora.alphas_full(w.alpha, w.N) if alphas is None else alphas
    fn(y, lay.x.cuda(), A, B, lay.col_off, w.ranks.cuda(), alphas, meta, status)
    torch.cuda.synchronize()
    return y.cpu()


def _check(w, lay, y, status, what):
    assert int(status.item()) == 0, f"{what}: device status {int(status.item())}"
    assert_within(y.double().numpy(), oracle_rows(w, lay, None), w.dtype, what)
    none = (w.ids < 0)
    assert torch.equal(y[none], lay.y0[none]), f"{what}: rows without an adapter changed"


# ------------------------------------------------------------------ padding ranks
@pytest.mark.parametrize("R", [16, 64])
@pytest.mark.parametrize("fn", ["add_linear", "bgmv_fused"])
@pytest.mark.parametrize("value", [float("nan"), 1e30])
def test_fused_padding_never_affects_result(cuda_lib, R, fn, value):
    """r_max 64 slots holding ranks 8, 17, 33, 64, 12, 1: the fused kernel loads
    A / B boxes up to r_n rounded to 8 (17 -> 24, 33 -> 40, 12 -> 16, 1 -> 8) and
    masks the loaded padding out of both products."""
    ranks = [8, 17, 33, 64, 12, 1]
    w = workloads.random_case(51, 300, 6, 512, [384, 128], 64, ranks=ranks, none_frac=0.1)
    lay = w.layers[0]
    A, B = _poisoned(lay, w.ranks, value)
    meta, status = build_meta(w.ids, w.N, R, 0)
    f = lora.lora_add_linear if fn == "add_linear" else lora.lora_bgmv_fused
    _check(w, lay, _apply(f, w, lay, A, B, meta, status), status, f"padding {value} R={R} {fn}")


def test_shrink_expand_padding_and_v_padding(cuda_lib):
    """The unfused pair on the fused kernel: shrink never writes v[k >= r_n] (a NaN
    sentinel survives) and ignores A's padding; expand ignores B's padding and
    whatever the caller's v holds at k >= r_n."""
    ranks = [8, 17, 33, 64]
    w = workloads.random_case(52, 200, 4, 256, [192, 64], 64, ranks=ranks, none_frac=0.1)
    lay = w.layers[0]
    A, B = _poisoned(lay, w.ranks)
    meta, status = build_meta(w.ids, w.N, 64, 0)
    ranks_d = w.ranks.cuda()
    v = torch.full((2, w.T, w.r_max), float("nan"), device="cuda")
    lora.lora_sgmv_shrink(v, lay.x.cuda(), A, ranks_d, meta, status)
    torch.cuda.synchronize()
    vref = oracle.lora_shrink(lay.x, lay.A, w.ranks, w.ids)           # [T, S, r_max]
    vg = v.cpu().double().permute(1, 0, 2).numpy()
    for i in range(w.T):
        n = int(w.ids[i])
        if n < 0:
            assert np.isnan(vg[i]).all()
            continue
        r = int(w.ranks[n])
        assert_within(vg[i, :, :r], vref[i, :, :r], torch.float32, f"v row {i}")
        assert np.isnan(vg[i, :, r:]).all(), f"v row {i}: padding written"
    # expand from the oracle's v with NaN beyond r_n
    vin = torch.as_tensor(vref, dtype=torch.float32).permute(1, 0, 2).contiguous()
    for n, r in enumerate(ranks):
        vin[:, (w.ids == n), r:] = float("nan")
    y = lay.y0.cuda().clone()
    lora.lora_sgmv_expand(y, vin.cuda(), B, lay.col_off, ranks_d, lora.alphas_full(w.alpha, w.N),
                          meta, status)
    torch.cuda.synchronize()
    _check(w, lay, y.cpu(), status, "expand with padded v")


def test_tensor_core_path_padding(cuda_lib):
    """Prompt runs on the tensor-core kernel with r_max 32 and ranks 9, 32, 16:
    A boxes are r_max rows, B's padded ranks are zeroed in shared memory."""
    w = workloads.random_case(53, 400, 3, 256, [128, 64], 32, ranks=[9, 32, 16],
                              runs=[(150, 0), (7, -1), (130, 1), (40, 2)])
    lay = w.layers[0]
    A, B = _poisoned(lay, w.ranks)
    meta, status = build_meta(w.ids, w.N, 64, 16)
    assert meta.host()["n_contig"] > 0
    _check(w, lay, _apply(lora.lora_add_linear, w, lay, A, B, meta, status), status, "tc padding")


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_general_kernel_padding(cuda_lib, dtype):
    """fp32, and bf16 with an unaligned width (d_in 203): the general kernel."""
    w = workloads.random_case(54, 90, 3, 203 if dtype == torch.bfloat16 else 96, 77, 16,
                              ranks=[3, 16, 9], dtype=dtype)
    lay = w.layers[0]
    A, B = _poisoned(lay, w.ranks)
    meta, status = build_meta(w.ids, w.N, 64, 0)
    _check(w, lay, _apply(lora.lora_add_linear, w, lay, A, B, meta, status), status,
           f"simt padding {dtype}")


# ------------------------------------------------------------------ per-adapter alpha
@pytest.mark.parametrize("case", ["fused", "tensor_core", "fp32"])
def test_per_adapter_alpha(cuda_lib, case):
    """alphas[n] differs per slot; the library divides by r_n itself.  The oracle
    takes one alpha, so the reference is assembled adapter by adapter."""
    if case == "fp32":
        w = workloads.random_case(55, 120, 5, 64, 48, 16, ranks=[16, 3, 8, 1, 12],
                                  dtype=torch.float32)
        min_run = 0
    elif case == "tensor_core":
        w = workloads.random_case(55, 300, 5, 256, [128, 64], 16, ranks=[16, 3, 8, 1, 12],
                                  runs=[(90, 0), (70, 3)])
        min_run = 16
    else:
        w = workloads.random_case(55, 300, 5, 256, [128, 64], 16, ranks=[16, 3, 8, 1, 12])
        min_run = 0
    alphas = torch.tensor([1.0, 8.0, 32.0, 0.5, 16.0], dtype=torch.float32)
    lay = w.layers[0]
    dl = DeviceLayer(lay)
    meta, status = build_meta(w.ids, w.N, 64, min_run)
    y = _apply(lora.lora_add_linear, w, lay, dl.A, dl.B, meta, status, alphas=alphas.cuda())
    assert int(status.item()) == 0
    ref = lay.y0.double().numpy().copy()
    for n in range(w.N):
        rows = np.nonzero((w.ids == n).numpy())[0].astype(np.int32)
        if len(rows):
            ref[rows] = oracle.lora_apply(lay.x, lay.A, lay.B, lay.col_off, w.ranks,
                                          float(alphas[n]), w.ids, lay.y0, rows=rows)
    assert_within(y.double().numpy(), ref, w.dtype, f"alphas {case}")


# ------------------------------------------------------------------ workspace
def test_workspace_serves_call_after_call(cuda_lib):
    """Three calls on one workspace (the Meta's), another layer shape in between,
    then a caller-provided workspace whose v part holds NaN: every result exact,
    and the workspace head (tickets, exit counter, per-unit counters) is zero
    after every call."""
    w = workloads.random_case(56, 400, 7, 512, [256, 128, 128], 32, ranks=[32, 8, 16, 24, 5, 32, 1])
    lay = w.layers[0]
    dl = DeviceLayer(lay)
    meta, status = build_meta(w.ids, w.N, 64, 0)
    head = 256 + 4 * meta.c.max_gather_tiles
    for _ in range(3):
        _check(w, lay, _apply(lora.lora_add_linear, w, lay, dl.A, dl.B, meta, status), status, "reuse")
        assert int(meta.workspace(3, 32)[:head].count_nonzero()) == 0
    w1 = workloads.random_case(56, 400, 7, 128, [64], 32, ranks=[32, 8, 16, 24, 5, 32, 1])
    w1.ids = w.ids
    l1 = w1.layers[0]
    d1 = DeviceLayer(l1)
    _check(w1, l1, _apply(lora.lora_add_linear, w1, l1, d1.A, d1.B, meta, status), status, "other shape")
    need = lora.lora_linear_workspace_bytes(meta, 3, 32)
    ws = torch.full((need,), 255, dtype=torch.uint8, device="cuda")
    ws[:head].zero_()
    y = lay.y0.cuda().clone()
    lora.lora_add_linear(y, dl.x, dl.A, dl.B, dl.col_off, w.ranks.cuda(),
                         lora.alphas_full(w.alpha, w.N), meta, status, workspace=ws)
    torch.cuda.synchronize()
    _check(w, lay, y.cpu(), status, "own workspace")
    assert int(ws[:head].count_nonzero()) == 0


# ------------------------------------------------------------------ passes and slice groups
@pytest.mark.parametrize("blocks", ["1", "0"])
def test_eight_slices_rank_64_multi_pass(cuda_lib, blocks, monkeypatch):
    """8 slices of rank 64 and 64-row tiles: 16 shrink items per unit (8 slices x two
    32-rank groups), expand items in two 32-row passes, on one block and on the
    full grid."""
    monkeypatch.setenv("LORA_BG_BLOCKS", blocks)
    w = workloads.random_case(57, 260, 3, 256, [64] * 8, 64, ranks=[64, 64, 40], none_frac=0.0)
    lay = w.layers[0]
    dl = DeviceLayer(lay)
    meta, status = build_meta(w.ids, w.N, 64, 0)
    _check(w, lay, _apply(lora.lora_bgmv_fused, w, lay, dl.A, dl.B, meta, status), status,
           f"8 slices blocks={blocks}")


# ------------------------------------------------------------------ launch-shape overrides
@pytest.mark.parametrize("env", [
    {"LORA_BG_ITEM_COLS": "32"}, {"LORA_BG_ITEM_COLS": "96"}, {"LORA_BG_ITEM_COLS": "192"},
    {"LORA_BG_ITEM_COLS": "4096"}, {"LORA_BG_ITEM_COLS": "8192"},
    {"LORA_BG_BLOCKS": "1"}, {"LORA_BG_BLOCKS": "2"}, {"LORA_BG_BLOCKS": "7"},
    {"LORA_BG_KSPLIT": "1"}, {"LORA_BG_KSPLIT": "2"}, {"LORA_BG_KSPLIT": "2", "LORA_BG_BLOCKS": "3"},
])
def test_overrides_keep_parity(cuda_lib, env, monkeypatch):
    for k, v in env.items():
        monkeypatch.setenv(k, v)
    w = workloads.random_case(58, 700, 9, 1024, [512, 256], 64, ranks=[64, 8, 16, 32, 24, 1, 48, 64, 16])
    lay = w.layers[0]
    dl = DeviceLayer(lay)
    meta, status = build_meta(w.ids, w.N, 64, 0)
    _check(w, lay, _apply(lora.lora_add_linear, w, lay, dl.A, dl.B, meta, status), status, str(env))


def test_fixed_shape_is_bit_reproducible(cuda_lib):
    w = workloads.random_case(59, 700, 9, 1024, [512, 256], 64)
    lay = w.layers[0]
    dl = DeviceLayer(lay)
    meta, status = build_meta(w.ids, w.N, 64, 0)
    a = _apply(lora.lora_add_linear, w, lay, dl.A, dl.B, meta, status)
    b = _apply(lora.lora_add_linear, w, lay, dl.A, dl.B, meta, status)
    assert torch.equal(a, b)


# ------------------------------------------------------------------ concurrency and graphs
def test_two_streams_at_once(cuda_lib):
    """Two batches on two streams, launched without a synchronisation between them
    (each Meta has its own workspace): both exact."""
    cases = [workloads.random_case(60 + i, 600, 8, 1024, [1024], 64) for i in range(2)]
    streams = [torch.cuda.Stream() for _ in cases]
    outs = []
    for w, st in zip(cases, streams):
        lay = w.layers[0]
        dl = DeviceLayer(lay)
        meta, status = build_meta(w.ids, w.N, 64, 0)
        meta.workspace(1, w.r_max)
        torch.cuda.synchronize()
        y = dl.y0.clone()
        outs.append((w, lay, y, status, dl, meta, w.ranks.cuda(), lora.alphas_full(w.alpha, w.N)))
    for (w, lay, y, status, dl, meta, rk, al), st in zip(outs, streams):
        lora.lora_add_linear(y, dl.x, dl.A, dl.B, dl.col_off, rk, al, meta, status, stream=st)
    torch.cuda.synchronize()
    for w, lay, y, status, *_ in outs:
        _check(w, lay, y.cpu(), status, "two streams")


def test_graph_replays_with_new_ids(cuda_lib):
    """Grouping and the layer captured once into a CUDA graph; each replay reads a
    new set of ids (different adapter mix, row counts and tile counts) from the
    same device buffer, so the adapter mix changes without a new capture."""
    T, N = 512, 12
    base = workloads.random_case(61, T, N, 512, [256, 256], 32)
    lay = base.layers[0]
    dl = DeviceLayer(lay)
    ids_d = base.ids.cuda().clone()
    meta = lora.Meta(T, N, 64, 0, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    rk, al = base.ranks.cuda(), lora.alphas_full(base.alpha, N)
    y = dl.y0.clone()
    st = torch.cuda.Stream()
    st.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(st):   # warm-up: workspace and side resources before capture
        lora.lora_build_segments(ids_d, meta, status, stream=st)
        lora.lora_add_linear(y, dl.x, dl.A, dl.B, dl.col_off, rk, al, meta, status, stream=st)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=st):
        lora.lora_build_segments(ids_d, meta, status, stream=st)
        lora.lora_add_linear(y, dl.x, dl.A, dl.B, dl.col_off, rk, al, meta, status, stream=st)
    gen = torch.Generator().manual_seed(5)
    for trial, nact in enumerate([12, 3, 1, 12]):
        ids = torch.randint(0, nact, (T,), generator=gen).to(torch.int32)
        ids[torch.rand(T, generator=gen) < 0.15] = -1
        ids_d.copy_(ids)
        y.copy_(lay.y0)
        status.zero_()
        torch.cuda.synchronize()
        g.replay()
        torch.cuda.synchronize()
        w = workloads.Workload("graph", base.dtype, T, N, base.r_max, base.alpha, ids, base.ranks,
                               [lay])
        _check(w, lay, y.cpu(), status, f"replay {trial}")
    del g


def test_capture_beside_an_eager_caller(cuda_lib):
    """One thread captures a mixed batch (prompt runs on the tensor-core kernel,
    decode rows forked to a side stream) while another thread runs another mixed
    batch eagerly on its own stream: each caller stream has its own side stream,
    so neither disturbs the other; both results exact."""
    def mixed(seed):
        return workloads.random_case(seed, 500, 6, 256, [128, 128], 16,
                                     runs=[(150, 0), (130, 3)], none_frac=0.1)
    wa, wb = mixed(62), mixed(63)
    res = {}

    def prep(w):
        lay = w.layers[0]
        dl = DeviceLayer(lay)
        meta, status = build_meta(w.ids, w.N, 64, 16)
        meta.workspace(2, w.r_max)   # allocated now, not while the other thread captures
        return lay, dl, meta, status, w.ranks.cuda(), lora.alphas_full(w.alpha, w.N)

    pa, pb = prep(wa), prep(wb)
    sa, sb = torch.cuda.Stream(), torch.cuda.Stream()
    ya, yb = pa[1].y0.clone(), pb[1].y0.clone()
    with torch.cuda.stream(sa):   # warm-up on the capturing stream (side stream, workspace)
        lora.lora_add_linear(ya, pa[1].x, pa[1].A, pa[1].B, pa[1].col_off, pa[4], pa[5], pa[2],
                             pa[3], stream=sa)
    torch.cuda.synchronize()
    ya.copy_(pa[1].y0)
    start = threading.Barrier(2)

    def eager():
        start.wait()
        with torch.cuda.stream(sb):
            for _ in range(20):
                yb.copy_(pb[1].y0)
                lora.lora_add_linear(yb, pb[1].x, pb[1].A, pb[1].B, pb[1].col_off, pb[4], pb[5],
                                     pb[2], pb[3], stream=sb)
        sb.synchronize()
        res["eager"] = yb.cpu()

    th = threading.Thread(target=eager)
    th.start()
    g = torch.cuda.CUDAGraph()
    start.wait()
    with torch.cuda.graph(g, stream=sa, capture_error_mode="thread_local"):
        lora.lora_add_linear(ya, pa[1].x, pa[1].A, pa[1].B, pa[1].col_off, pa[4], pa[5], pa[2],
                             pa[3], stream=sa)
    th.join()
    torch.cuda.synchronize()
    ya.copy_(pa[1].y0)
    g.replay()
    torch.cuda.synchronize()
    _check(wa, pa[0], ya.cpu(), pa[3], "captured")
    _check(wb, pb[0], res["eager"], pb[3], "eager beside a capture")
    del g


# ------------------------------------------------------------------ bounded waits
def test_stalled_stage_times_out_and_the_context_survives(cuda_lib, monkeypatch):
    """LORA_DEBUG_STALL=1: every expand item waits for one shrink signal more than
    its unit ever gives; the bounded wait runs out (a few ms), LORA_DEV_TIMEOUT is
    set and the call returns.  The same workspace then serves a normal call,
    exactly."""
    w = workloads.random_case(64, 300, 5, 512, [256], 32)
    lay = w.layers[0]
    dl = DeviceLayer(lay)
    meta, status = build_meta(w.ids, w.N, 64, 0)
    monkeypatch.setenv("LORA_DEBUG_STALL", "1")
    _apply(lora.lora_add_linear, w, lay, dl.A, dl.B, meta, status)
    assert int(status.item()) & lora.DEV_TIMEOUT
    head = 256 + 4 * meta.c.max_gather_tiles
    assert int(meta.workspace(1, w.r_max)[:head].count_nonzero()) == 0
    monkeypatch.delenv("LORA_DEBUG_STALL")
    status.zero_()
    _check(w, lay, _apply(lora.lora_add_linear, w, lay, dl.A, dl.B, meta, status), status,
           "after a timed-out call")


# ------------------------------------------------------------------ tile row counts
@pytest.mark.parametrize("rows", [1, 7, 8, 9, 15, 16, 17, 24, 31, 32, 33, 40, 47, 48, 49, 63, 64])
@pytest.mark.parametrize("S,ranks", [(1, [8, 64]), (3, [16, 40]), (2, [8, 33])])
def test_every_tile_row_count(cuda_lib, rows, S, ranks):
    """Two adapters with `rows` rows each, in 64-row tiles: every count of n8 row
    tiles in the shrink (1, 2, 4 or 8 loaded, the rest zero-filled), one or two
    32-row expand passes of one or two m16 tiles, and ranks that use one or two
    m16 rank tiles and the 16-, 32- and 64-rank expand loads."""
    T = 2 * rows + 5
    ids = [0] * rows + [1] * rows + [-1] * 5
    perm = torch.randperm(T, generator=torch.Generator().manual_seed(rows))
    w = workloads.random_case(70 + rows, T, 2, 384, [256] * S if S > 1 else [512], 64, ranks=ranks)
    w.ids = torch.tensor(ids, dtype=torch.int32)[perm]
    lay = w.layers[0]
    dl = DeviceLayer(lay)
    meta, status = build_meta(w.ids, w.N, 64, 0)
    _check(w, lay, _apply(lora.lora_add_linear, w, lay, dl.A, dl.B, meta, status), status,
           f"rows {rows} S={S}")
