"""The tensor-core gathered-tile kernel (units of at most 16 rows, fused calls,
selected with LORA_BG_TC=1) against the fp64 oracle:

* every unit row count 1..16 (the MMA's N = 16, rows past the count unused), with
  ranks whose 8-rank groups are odd in number (the zero buffer pairs the last
  group) or not whole (padding ranks zeroed in shared memory);
* padding ranks holding NaN or 1e30 never reach a sum;
* input widths that end inside a 64-column chunk, output slices that end inside
  a 128-column tile, and several slices;
* every expand item width and small grids (the persistent loop, tickets);
* the same results as the mma.sync kernel up to rounding order;
* the bounded wait: an expand item whose unit never finishes times out, and the
  workspace then serves a normal call.

Tolerance (the method's): bf16 |gpu - oracle| <= 1e-2 * max(1, |oracle|).
"""
import pytest
import torch

import lora_adapter_application_b200 as lora
import workloads
from gpu_helpers import DeviceLayer, assert_within, build_meta, oracle_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _tensor_core_kernel(monkeypatch):
    """Every fused call in this file goes to the tensor-core kernel (opt-in)."""
    monkeypatch.setenv("LORA_BG_TC", "1")


def _poisoned(lay, ranks, value):
    A = [a.clone() for a in lay.A]
    B = [b.clone() for b in lay.B]
    for n, r in enumerate(ranks.tolist()):
        for a in A:
            a[n, r:, :] = value
        for b in B:
            b[n, :, r:] = value
    return [a.cuda() for a in A], [b.cuda() for b in B]


def _run(w, lay, A, B, meta, status, fn=None):
    y = lay.y0.cuda().clone()
    f = fn or lora.lora_add_linear
    f(y, lay.x.cuda(), A, B, lay.col_off, w.ranks.cuda(), lora.alphas_full(w.alpha, w.N), meta, status)
    torch.cuda.synchronize()
    return y.cpu()


def _check(w, lay, y, status, what):
    assert int(status.item()) == 0, f"{what}: device status {int(status.item())}"
    assert_within(y.double().numpy(), oracle_rows(w, lay, None), w.dtype, what)
    none = w.ids < 0
    assert torch.equal(y[none], lay.y0[none]), f"{what}: rows without an adapter changed"


@pytest.mark.parametrize("rows", list(range(1, 17)))
def test_every_unit_row_count(cuda_lib, rows):
    """Three adapters with `rows` rows each (ranks 8, 24, 64: one, three and eight
    8-rank groups), 16-row tiles, three slices of 200, 72 and 384 columns, d_in 200."""
    T = 3 * rows + 3
    ids = [0] * rows + [1] * rows + [2] * rows + [-1] * 3
    perm = torch.randperm(T, generator=torch.Generator().manual_seed(rows))
    w = workloads.random_case(300 + rows, T, 3, 200, [200, 72, 384], 64, ranks=[8, 24, 64])
    w.ids = torch.tensor(ids, dtype=torch.int32)[perm]
    lay = w.layers[0]
    dl = DeviceLayer(lay)
    meta, status = build_meta(w.ids, w.N, 16, 0)
    _check(w, lay, _run(w, lay, dl.A, dl.B, meta, status), status, f"rows {rows}")


@pytest.mark.parametrize("value", [float("nan"), 1e30])
@pytest.mark.parametrize("fn", ["add_linear", "bgmv_fused"])
def test_padding_never_affects_result(cuda_lib, value, fn):
    """Ranks 1, 8, 12, 17, 33, 40, 63, 64 in 64-rank slots with every padding rank
    poisoned: not whole 8-rank groups (1, 12, 17, 33, 63), odd group counts (1, 8,
    17, 33, 40), and whole ones."""
    ranks = [1, 8, 12, 17, 33, 40, 63, 64]
    w = workloads.random_case(311, 400, 8, 320, [512, 136], 64, ranks=ranks, none_frac=0.1)
    lay = w.layers[0]
    A, B = _poisoned(lay, w.ranks, value)
    meta, status = build_meta(w.ids, w.N, 16, 0)
    f = lora.lora_add_linear if fn == "add_linear" else lora.lora_bgmv_fused
    _check(w, lay, _run(w, lay, A, B, meta, status, f), status, f"padding {value} {fn}")


@pytest.mark.parametrize("env", [
    {"LORA_BT_COLS": "128"}, {"LORA_BT_COLS": "256"}, {"LORA_BT_COLS": "384"},
    {"LORA_BG_BLOCKS": "1"}, {"LORA_BG_BLOCKS": "2"}, {"LORA_BG_BLOCKS": "7"},
])
def test_item_widths_and_grids(cuda_lib, env, monkeypatch):
    """The expand item width and the grid size change nothing beyond rounding order."""
    for k, v in env.items():
        monkeypatch.setenv(k, v)
    w = workloads.random_case(312, 700, 24, 1024, [1024, 256, 256], 64, ranks=[8, 16, 32, 64] * 6)
    lay = w.layers[0]
    dl = DeviceLayer(lay)
    meta, status = build_meta(w.ids, w.N, 16, 0)
    _check(w, lay, _run(w, lay, dl.A, dl.B, meta, status), status, f"env {env}")


def test_agrees_with_the_mma_sync_kernel(cuda_lib, monkeypatch):
    """The tensor-core kernel and the mma.sync kernel on one decode layer (uniform
    ids over 40 adapters, ranks 8-64): both within tolerance of the oracle, and of
    each other."""
    w = workloads.random_case(313, 512, 40, 2048, [2048], 64, ranks=[8, 16, 32, 64] * 10)
    lay = w.layers[0]
    dl = DeviceLayer(lay)
    meta, status = build_meta(w.ids, w.N, 16, 0)
    y_tc = _run(w, lay, dl.A, dl.B, meta, status)
    _check(w, lay, y_tc, status, "tensor-core kernel")
    monkeypatch.setenv("LORA_BG_TC", "0")
    y_ms = _run(w, lay, dl.A, dl.B, meta, status)
    _check(w, lay, y_ms, status, "mma.sync kernel")
    assert_within(y_tc.double().numpy(), y_ms.double().numpy(), w.dtype, "the two kernels")


def test_workspace_head_returns_to_zero(cuda_lib):
    """Tickets, exit counter and done words are zero after every call, so one
    workspace serves the next call."""
    w = workloads.random_case(314, 300, 12, 512, [256, 256], 32)
    lay = w.layers[0]
    dl = DeviceLayer(lay)
    meta, status = build_meta(w.ids, w.N, 16, 0)
    head = 256 + 4 * meta.c.max_gather_tiles
    for k in range(3):
        _check(w, lay, _run(w, lay, dl.A, dl.B, meta, status), status, f"call {k}")
        assert int(meta.workspace(2, w.r_max)[:head].count_nonzero()) == 0


def test_stalled_unit_times_out_and_the_context_survives(cuda_lib, monkeypatch):
    """LORA_DEBUG_STALL=1: expand items wait for one shrink signal more than a unit
    gives; the bounded wait runs out, LORA_DEV_TIMEOUT is set, the call returns with
    its workspace head at zero, and a normal call on it is exact."""
    w = workloads.random_case(315, 300, 5, 512, [256], 32)
    lay = w.layers[0]
    dl = DeviceLayer(lay)
    meta, status = build_meta(w.ids, w.N, 16, 0)
    monkeypatch.setenv("LORA_DEBUG_STALL", "1")
    _run(w, lay, dl.A, dl.B, meta, status)
    assert int(status.item()) & lora.DEV_TIMEOUT
    head = 256 + 4 * meta.c.max_gather_tiles
    assert int(meta.workspace(1, w.r_max)[:head].count_nonzero()) == 0
    monkeypatch.delenv("LORA_DEBUG_STALL")
    status.zero_()
    _check(w, lay, _run(w, lay, dl.A, dl.B, meta, status), status, "after a timed-out call")
