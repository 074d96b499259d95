"""The C-ABI library loads and exports every entry point its header declares,
and the host-side checks reject bad arguments before anything reaches a GPU.
Runs without a GPU: nothing here launches a kernel."""
import ctypes
import os
import re

import pytest

import lora_adapter_application_b200 as lora

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "lora_delta.h")


def declared_entry_points():
    text = open(HEADER).read()
    return re.findall(r"LORA_API\s+[A-Za-z_][A-Za-z0-9_\s\*]*?\b(lora_[a-z0-9_]+)\s*\(", text)


@pytest.fixture(scope="module")
def lib():
    from lora_adapter_application_b200 import build
    build.build()
    return lora.load()


def test_header_declares_the_boundary():
    names = set(declared_entry_points())
    for required in ["lora_build_segments", "lora_sgmv_shrink", "lora_sgmv_expand",
                     "lora_bgmv_fused", "lora_add_linear"]:
        assert required in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_entry_points():
        assert hasattr(lib, name), name
        assert isinstance(getattr(lib, name), ctypes._CFuncPtr)


def test_binding_names_match_the_abi():
    for name in declared_entry_points():
        if name != "lora_status_string":
            assert hasattr(lora, name), name


def test_capacity_bounds(lib):
    mg, mc = lora.lora_meta_capacity(1024, 100, 16, 64, 128)
    assert mg == 64 + 100 and mc == 8 + 16
    assert lora.lora_meta_capacity(10, 100, 16, 0, 128) == (1 + 10, 0)
    with pytest.raises(lora.LoraError):
        lora.lora_meta_capacity(-1, 4, 16, 0, 128)
    with pytest.raises(lora.LoraError):
        lora.lora_meta_capacity(10, 4, 65, 0, 128)
    assert lora.lora_meta_capacity(1024, 100, 64, 0, 128) == (16 + 100, 0)


def test_segment_plan(lib, monkeypatch):
    """lora_segment_plan: a layer routes every row to the fused kernel when the
    batch has fewer long_tile-row tiles than SMs and the layer is 8192+ columns
    wide; when all layers do and the batch has runs, the plan is 32-row tiles and
    no runs; otherwise the caller's values come back."""
    monkeypatch.delenv("LORA_TC_ROUTE", raising=False)
    plan = lora.lora_segment_plan
    # 8192 rows = 64 tiles of 128 < 148 SMs; both layers wide
    assert plan(8192, [28672, 8192], 16, 64, sms=148) == (32, 0, [True, True])
    # one narrow layer: runs kept; the flags still say which layer routes
    assert plan(8192, [28672, 8191], 16, 64, sms=148) == (16, 64, [True, False])
    # as many tiles as SMs: the tensor-core kernel keeps the runs
    assert plan(148 * 128, [28672], 16, 64, sms=148) == (16, 64, [False])
    assert plan(147 * 128, [28672], 16, 64, sms=148) == (32, 0, [True])
    assert plan(147 * 128 + 1, [28672], 16, 64, sms=148) == (16, 64, [False])
    # a decode batch (no runs) keeps its tile size; no layers: unchanged
    assert plan(8192, [28672, 8192], 16, 0, sms=148) == (16, 0, [True, True])
    assert plan(8192, [], 16, 64, sms=148) == (16, 64, [])
    # the long tile sets the tile count: 8192 rows in 32-row tiles = 256 > 148
    assert plan(8192, [28672], 16, 64, sms=148, long_tile=32) == (16, 64, [False])
    # LORA_TC_ROUTE: 1 = never all-gathered, 2 = always
    monkeypatch.setenv("LORA_TC_ROUTE", "1")
    assert plan(8192, [28672, 8192], 16, 64, sms=148) == (16, 64, [False, False])
    monkeypatch.setenv("LORA_TC_ROUTE", "2")
    assert plan(77000, [4096], 16, 64, sms=148) == (32, 0, [True])
    monkeypatch.delenv("LORA_TC_ROUTE")
    # out-of-range arguments: LORA_ERR_SHAPE, nothing written
    for args, kw in [((-1, [8192], 16, 64), {}), ((lora.MAX_ROWS + 1, [8192], 16, 64), {}),
                     ((8192, [0], 16, 64), {}), ((8192, [8192], 0, 64), {}),
                     ((8192, [8192], 65, 64), {}), ((8192, [8192], 16, -1), {}),
                     ((8192, [8192], 16, 64), {"sms": -1}), ((8192, [8192], 16, 64), {"long_tile": 0}),
                     ((8192, [8192], 16, 64), {"long_tile": 129})]:
        with pytest.raises(lora.LoraError):
            plan(*args, **kw)
    # NULL pointers through the C ABI
    rt, mr = ctypes.c_int32(16), ctypes.c_int32(64)
    cols = (ctypes.c_int64 * 1)(8192)
    assert lib.lora_segment_plan(8192, None, 1, 148, 128, ctypes.byref(rt), ctypes.byref(mr), None) == -1
    assert lib.lora_segment_plan(8192, cols, 1, 148, 128, None, ctypes.byref(mr), None) == -1
    assert lib.lora_segment_plan(8192, cols, 1, 148, 128, ctypes.byref(rt), None, None) == -1
    assert (rt.value, mr.value) == (16, 64)
    # the flag array is optional
    assert lib.lora_segment_plan(8192, cols, 1, 148, 128, ctypes.byref(rt), ctypes.byref(mr), None) == 0
    assert (rt.value, mr.value) == (32, 0)


def test_scratch_and_workspace_sizes(lib):
    assert lora.lora_segments_scratch_bytes(2048, 100) == 0
    # one thread block, no scratch: T <= 2048, or T <= 8192 with N <= 1023
    assert lora.lora_segments_scratch_bytes(2048, 4096) == 0
    assert lora.lora_segments_scratch_bytes(8192, 1023) == 0

    def r256(b):
        return (b + 255) // 256 * 256

    # as the header states: per-chunk id counts, one byte per row, 12 bytes per
    # 32 rows and 16 bytes per 2048 rows, each part rounded up to 256 bytes
    for T, N in [(2049, 1024), (8192, 1024), (8193, 8), (77431, 8), (131072, 4096)]:
        chunks, words, blocks = -(-T // 2048), -(-T // 32), -(-T // 2048)
        want = r256(4 * (N + 1) * chunks) + r256(T) + r256(12 * words) + r256(16 * blocks)
        assert lora.lora_segments_scratch_bytes(T, N) == want, (T, N)
    assert lora.lora_shrink_workspace_bytes(1024, 64, 3) == 3 * 1024 * 64 * 4
    # out-of-range sizes: 0, and no integer overflow on the way
    INT_MAX = 2 ** 31 - 1
    assert lora.lora_segments_scratch_bytes(INT_MAX, 8) == 0
    assert lora.lora_segments_scratch_bytes(1024, INT_MAX) == 0
    assert lora.lora_segments_scratch_bytes(lora.MAX_ROWS + 1, 8) == 0


def test_linear_workspace_size(lib):
    """256-byte head, one int per unit of the meta's tile capacity (rounded up to
    256 bytes), then room for the larger of the two kernels' v: fp32
    [2][n_slices][T][r_max] (a small batch's shrink items may be split in two), or
    per unit and slice a bf16 hi + lo pair of 16 rows by r_max rounded up to 16
    ranks."""
    def r256(b):
        return (b + 255) // 256 * 256
    for T, N, R, min_run, S, r_max in [(1024, 100, 64, 0, 3, 64), (256, 32, 64, 0, 1, 16),
                                       (8192, 16, 64, 64, 1, 16), (77431, 8, 16, 64, 2, 32)]:
        m = _meta(T, N, R, min_run)
        mg, mc = lora.lora_meta_capacity(T, N, R, min_run, 128)
        units = mg + (mc * -(-128 // R) if min_run > 0 else 0)
        want = 256 + r256(4 * units) + max(2 * S * T * r_max * 4, units * S * 2 * 16 * -(-r_max // 16) * 16 * 2)
        assert lib.lora_linear_workspace_bytes(ctypes.byref(m), S, r_max) == want, (T, N, R)
    m = _meta()
    assert lib.lora_linear_workspace_bytes(ctypes.byref(m), 0, 16) == 0
    assert lib.lora_linear_workspace_bytes(ctypes.byref(m), 1, 129) == 0
    assert lib.lora_linear_workspace_bytes(None, 1, 16) == 0


def _meta(T=8, N=4, R=4, min_run=0):
    mg, mc = lora.lora_meta_capacity(T, N, R, min_run, 128)
    fake = 0x1000   # never dereferenced: every call below fails its host check first
    return lora.lora_meta(T, N, R, min_run, 128, mg, mc, fake, fake, fake, fake, fake, fake, fake)


def _codes(lib):
    return {n: v for n, v in [("NULL", -1), ("DTYPE", -2), ("SHAPE", -3), ("RANK", -4),
                              ("WORKSPACE", -6), ("CAPACITY", -7)]}


def test_host_checks(lib):
    c = _codes(lib)
    fake = ctypes.c_void_p(0x1000)
    m = _meta()
    assert lib.lora_build_segments(fake, None, None, 0, fake, None) == c["NULL"]
    assert lib.lora_build_segments(fake, ctypes.byref(m), None, 0, None, None) == c["NULL"]
    small = _meta()
    small.max_gather_tiles = 1
    assert lib.lora_build_segments(fake, ctypes.byref(small), None, 0, fake, None) == c["CAPACITY"]
    bad = _meta()
    bad.rows_per_tile = 0
    assert lib.lora_build_segments(fake, ctypes.byref(bad), None, 0, fake, None) == c["SHAPE"]
    sl = (lora.lora_slice * 1)()
    sl[0].A, sl[0].B, sl[0].d_out, sl[0].col_off = 0x1000, 0x1000, 16, 0
    ws_need = lib.lora_linear_workspace_bytes(ctypes.byref(m), 1, 16)
    args = lambda dtype=0, r_max=16, n=1, ld_y=16, sl=sl, ws=ctypes.c_void_p(0x10000), wsb=ws_need: (
        fake, ld_y, fake, 16, 16, sl, n, r_max, fake, fake, ctypes.byref(m), ws, wsb, dtype, fake,
        None)
    assert lib.lora_add_linear(*args(dtype=7)) == c["DTYPE"]
    assert lib.lora_add_linear(*args(r_max=0)) == c["RANK"]
    assert lib.lora_add_linear(*args(r_max=129)) == c["RANK"]
    assert lib.lora_add_linear(*args(n=0)) == c["SHAPE"]
    assert lib.lora_add_linear(*args(n=9)) == c["SHAPE"]
    assert lib.lora_add_linear(*args(ld_y=8)) == c["SHAPE"]   # slice runs past the row
    assert lib.lora_bgmv_fused(*args(ld_y=8)) == c["SHAPE"]
    two = (lora.lora_slice * 2)()                                  # q [0, 16) and k [8, 24): overlap
    two[0].A, two[0].B, two[0].d_out, two[0].col_off = 0x1000, 0x1000, 16, 0
    two[1].A, two[1].B, two[1].d_out, two[1].col_off = 0x1000, 0x1000, 16, 8
    assert lib.lora_add_linear(*args(n=2, ld_y=32, sl=two)) == c["SHAPE"]
    assert lib.lora_sgmv_expand(fake, 32, fake, two, 2, 16, fake, fake, ctypes.byref(m), 0, fake,
                                None) == c["SHAPE"]
    nul = (lora.lora_slice * 1)()
    nul[0].A, nul[0].B, nul[0].d_out = None, 0x1000, 16
    assert lib.lora_add_linear(*args(sl=nul)) == c["NULL"]
    big = _meta()
    big.T = lora.MAX_ROWS + 1
    assert lib.lora_sgmv_shrink(fake, fake, 16, 16, sl, 1, 16, fake, ctypes.byref(big), 0, fake,
                                None) == c["SHAPE"]
    assert lib.lora_sgmv_expand(fake, 16, None, sl, 1, 16, fake, fake, ctypes.byref(m), 0, fake,
                                None) == c["NULL"]
    # the fused calls' workspace: present, large enough, 256-byte aligned
    for fn in (lib.lora_add_linear, lib.lora_bgmv_fused):
        assert fn(*args(ws=None)) == c["NULL"]
        assert fn(*args(wsb=ws_need - 1)) == c["WORKSPACE"]
        assert fn(*args(ws=ctypes.c_void_p(0x10010))) == c["WORKSPACE"]
    assert lib.lora_status_string(-7) == b"LORA_ERR_CAPACITY"


def test_static_grouping_checks_the_meta_first(lib):
    """lora_build_segments_static refuses an out-of-range meta with the same code as
    lora_build_segments (LORA_ERR_SHAPE), before sizing any scratch: no integer
    overflow, no LORA_ERR_WORKSPACE for sizes that are simply invalid."""
    c = _codes(lib)
    fake = ctypes.c_void_p(0x1000)
    for T, N in [(2 ** 31 - 1, 8), (lora.MAX_ROWS + 1, 8), (1024, 2 ** 31 - 1), (-1, 8)]:
        m = _meta()
        m.T, m.N = T, N
        assert lib.lora_build_segments_static(fake, ctypes.byref(m), fake, None) == c["SHAPE"], (T, N)
        assert lib.lora_build_segments(fake, ctypes.byref(m), None, 0, fake, None) == c["SHAPE"]
    m = _meta()
    assert lib.lora_build_segments_static(fake, ctypes.byref(m), None, None) == c["NULL"]
