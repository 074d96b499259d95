"""fp64 CPU oracle for multi-LoRA delta application.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` are the only users.  The library under
``lora_adapter_application_b200/`` never imports this package, and this package
never imports the library: the two share no code.

The arithmetic lives in ``lora_oracle.c`` (plain C, fp64, no fast-math); this
module compiles it with gcc and marshals torch CPU tensors into it.  What each
function computes, and the passage of the pages it follows, is stated there.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "lora_oracle.c")
_LIB = os.path.join(_HERE, "liblora_oracle.so")
_lib = None

BF16, FP32 = 0, 1


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, OpenMP, no fast-math)."""
    stale = (not os.path.exists(_LIB)) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC)
    if force or stale:
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P, I32, I64, D = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_double
        lib.oracle_lora_apply.restype = ctypes.c_int
        lib.oracle_lora_apply.argtypes = [ctypes.c_int, P, I64, I32, I32, P, P, P, P, I32, I32, P,
                                          D, P, I32, P, I32, P, I64, P]
        lib.oracle_lora_shrink.restype = ctypes.c_int
        lib.oracle_lora_shrink.argtypes = [ctypes.c_int, P, I64, I32, I32, P, I32, I32, P, P, P, I32, P]
        lib.oracle_build_segments.restype = ctypes.c_int
        lib.oracle_build_segments.argtypes = [P, I32, I32, I32, I32, I32, I32, I32,
                                              P, P, P, P, P, P, P]
        lib.oracle_lora_merge.restype = ctypes.c_int
        lib.oracle_lora_merge.argtypes = [ctypes.c_int, P, I64, I32, I32, P, P, I32, I32, D, I32, P]
        lib.oracle_lora_param_count.restype = I64
        lib.oracle_lora_param_count.argtypes = [I64, I64, I64]
        lib.oracle_adapter_bytes.restype = I64
        lib.oracle_adapter_bytes.argtypes = [I64, I64, I64, I64]
        lib.oracle_set_threads.argtypes = [ctypes.c_int]
        lib.oracle_max_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return FP32
    raise TypeError(f"oracle takes bf16 or fp32, got {t.dtype}")


def _cpu(t: torch.Tensor) -> torch.Tensor:
    assert t.device.type == "cpu", "oracle inputs live on the host"
    return t.contiguous()


def set_threads(n: int) -> None:
    _load().oracle_set_threads(int(n))


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def lora_apply(x, A, B, col_off, ranks, alpha, ids, y0, rows=None):
    """Rows of y0 plus the LoRA delta of every slice, unrounded, as float64.

    x [T, ld_x]; A[s] [N, r_max, d_in]; B[s] [N, d_out_s, r_max]; y0 [T, ld_y];
    slice s writes columns col_off[s] .. col_off[s]+d_out_s; ranks[N] int;
    ids[T] int (-1 = no adapter).  ``rows`` (optional) lists the rows to compute;
    the result then has one row per listed row.
    """
    lib = _load()
    x, y0 = _cpu(x), _cpu(y0)
    A = [_cpu(a) for a in A]
    B = [_cpu(b) for b in B]
    code = _dtype_code(x)
    for t in [y0] + A + B:
        assert _dtype_code(t) == code, "all float inputs share one dtype"
    T, ld_x = x.shape
    d_in = A[0].shape[2]
    N, r_max = A[0].shape[0], A[0].shape[1]
    ld_y = y0.shape[1]
    n_slices = len(A)
    d_out = np.array([b.shape[1] for b in B], dtype=np.int32)
    offs = np.array(list(col_off), dtype=np.int32)
    ranks_np = np.ascontiguousarray(np.asarray(ranks, dtype=np.int32))
    ids_np = np.ascontiguousarray(np.asarray(ids, dtype=np.int32))
    assert ids_np.shape == (T,) and ranks_np.shape == (N,)
    A_ptrs = (ctypes.c_void_p * n_slices)(*[a.data_ptr() for a in A])
    B_ptrs = (ctypes.c_void_p * n_slices)(*[b.data_ptr() for b in B])
    if rows is None:
        rows_np, n_rows = None, T
    else:
        rows_np = np.ascontiguousarray(np.asarray(rows, dtype=np.int32))
        n_rows = rows_np.shape[0]
    out = np.empty((n_rows, ld_y), dtype=np.float64)
    rc = lib.oracle_lora_apply(code, x.data_ptr(), ld_x, d_in, n_slices, A_ptrs, B_ptrs,
                               d_out.ctypes.data, offs.ctypes.data, N, r_max,
                               ranks_np.ctypes.data, float(alpha), ids_np.ctypes.data, T,
                               None if rows_np is None else rows_np.ctypes.data, n_rows,
                               y0.data_ptr(), ld_y, out.ctypes.data)
    if rc != 0:
        raise ValueError("oracle_lora_apply rejected its arguments")
    return out


def lora_shrink(x, A, ranks, ids, rows=None):
    """v = A_n x_i per listed row and slice, fp64, shape [n_rows, n_slices, r_max]
    (zeros for rows without an adapter and for k >= r_n)."""
    lib = _load()
    x = _cpu(x)
    A = [_cpu(a) for a in A]
    code = _dtype_code(x)
    T, ld_x = x.shape
    N, r_max, d_in = A[0].shape
    n_slices = len(A)
    ranks_np = np.ascontiguousarray(np.asarray(ranks, dtype=np.int32))
    ids_np = np.ascontiguousarray(np.asarray(ids, dtype=np.int32))
    rows_np = np.arange(T, dtype=np.int32) if rows is None else \
        np.ascontiguousarray(np.asarray(rows, dtype=np.int32))
    A_ptrs = (ctypes.c_void_p * n_slices)(*[a.data_ptr() for a in A])
    out = np.empty((rows_np.shape[0], n_slices, r_max), dtype=np.float64)
    rc = lib.oracle_lora_shrink(code, x.data_ptr(), ld_x, d_in, n_slices, A_ptrs, N, r_max,
                                ranks_np.ctypes.data, ids_np.ctypes.data, rows_np.ctypes.data,
                                rows_np.shape[0], out.ctypes.data)
    if rc != 0:
        raise ValueError("oracle_lora_shrink rejected its arguments")
    return out


def build_segments(ids, N, rows_per_tile, min_run, long_tile=128,
                   max_gather_tiles=None, max_contig_tiles=None):
    """Grouping by adapter id plus the tile lists (see lora_oracle.c)."""
    lib = _load()
    ids_np = np.ascontiguousarray(np.asarray(ids, dtype=np.int32))
    T = ids_np.shape[0]
    if max_gather_tiles is None:
        max_gather_tiles = T + N + 1
    if max_contig_tiles is None:
        max_contig_tiles = T + 1
    perm = np.zeros(max(T, 1), np.int32)
    seg_start = np.zeros(N + 1, np.int32)
    seg_adapter = np.zeros(max(N, 1), np.int32)
    counts = np.zeros(4, np.int32)
    grow = np.zeros(max(T, 1), np.int32)
    gt = np.zeros((max(max_gather_tiles, 1), 4), np.int32)
    ct = np.zeros((max(max_contig_tiles, 1), 4), np.int32)
    status = lib.oracle_build_segments(ids_np.ctypes.data, T, N, rows_per_tile, min_run,
                                       long_tile, max_gather_tiles, max_contig_tiles,
                                       perm.ctypes.data, seg_start.ctypes.data,
                                       seg_adapter.ctypes.data, counts.ctypes.data,
                                       grow.ctypes.data, gt.ctypes.data, ct.ctypes.data)
    n_seg, n_gather, n_contig, n_short = (int(c) for c in counts)
    return {
        "status": int(status),
        "perm": perm[:T].copy(),
        "seg_start": seg_start,
        "seg_adapter": seg_adapter[:n_seg].copy(),
        "n_seg": n_seg,
        "n_gather": n_gather,
        "n_contig": n_contig,
        "n_short": n_short,
        "grow": grow[:n_short].copy(),
        "gather_tiles": gt[:n_gather].copy(),
        "contig_tiles": ct[:n_contig].copy(),
    }


def lora_merge(W, A, B, r, alpha, sign=1):
    """W + sign * (alpha / r) * B[:, :r] A[:r, :] in fp64 for one adapter: W [d_out,
    ld_w] (d_in = A's width used), A [r_max, d_in], B [d_out, r_max]."""
    lib = _load()
    W, A, B = _cpu(W), _cpu(A), _cpu(B)
    code = _dtype_code(W)
    assert _dtype_code(A) == code and _dtype_code(B) == code, "one dtype"
    d_out, ld_w = W.shape
    r_max, d_in = A.shape
    assert B.shape == (d_out, r_max)
    out = np.empty((d_out, d_in), dtype=np.float64)
    rc = lib.oracle_lora_merge(code, W.data_ptr(), ld_w, d_out, d_in, A.data_ptr(), B.data_ptr(),
                               r_max, int(r), float(alpha), int(sign), out.ctypes.data)
    if rc != 0:
        raise ValueError("oracle_lora_merge rejected its arguments")
    return out


def lora_param_count(d: int, k: int, r: int) -> int:
    return int(_load().oracle_lora_param_count(d, k, r))


def adapter_bytes(num_layers: int, r: int, hidden: int, dtype_bytes: int) -> int:
    return int(_load().oracle_adapter_bytes(num_layers, r, hidden, dtype_bytes))
