"""Python binding of the B200 multi-LoRA delta library (``liblora_delta.so``).

Argument marshalling only: every function below turns torch tensors into the
plain pointers, strides and sizes of the C ABI declared in
``include/lora_delta.h`` and calls the entry point of the same name.  All
arithmetic runs in the library's CUDA kernels; PyTorch only owns device memory
and streams.  There is no fallback: if the library is not built, or a call is
made with CPU tensors, these functions raise.

What is computed (page "Multi-LoRA Serving: one base, many adapters", section
3.1 and 3.4; page "LoRA service: multi-adapter dynamic loading", section 2):
for every row i with adapter n = ids[i] != -1,

    y_i[col_off_s : col_off_s + d_out_s] += (alphas[n] / r_n) * B_s[n] (A_s[n] x_i)

with only the first r_n rank rows/columns used; the library computes the
scale alphas[n] / r_n on the device from the two per-slot tensors.
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "load", "LoraError", "Meta", "LORA_BF16", "LORA_FP32", "DEV_BAD_ID", "DEV_TILE_OVERFLOW",
    "DEV_BAD_RANK", "lora_version", "lora_last_error", "lora_meta_capacity", "lora_segments_scratch_bytes",
    "lora_build_segments", "lora_build_segments_static", "lora_shrink_workspace_bytes",
    "lora_linear_workspace_bytes", "lora_sgmv_shrink", "lora_sgmv_expand", "lora_bgmv_fused",
    "lora_add_linear", "alphas_full", "lora_load_adapter", "SlotCache", "lora_slot_cache_create",
    "lora_slot_cache_destroy", "lora_slot_cache_acquire", "lora_slot_cache_release",
    "lora_slot_cache_key", "lora_slot_cache_evict", "lora_merge_adapter", "lora_segment_plan",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liblora_delta.so")

LORA_BF16, LORA_FP32 = 0, 1
DEV_BAD_ID, DEV_TILE_OVERFLOW, DEV_BAD_RANK, DEV_TIMEOUT = 1, 2, 4, 8
ERR_CUDA = -8   # LORA_ERR_CUDA
MAX_ROWS, MAX_ADAPTERS, MAX_RANK, MAX_SLICES, LONG_TILE = 131072, 4096, 128, 8, 128
MAX_TILE_ROWS = 64

_P, _I32, _I64, _SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t


class lora_meta(ctypes.Structure):
    _fields_ = [("T", _I32), ("N", _I32), ("rows_per_tile", _I32), ("min_run", _I32),
                ("long_tile", _I32), ("max_gather_tiles", _I32), ("max_contig_tiles", _I32),
                ("perm", _P), ("seg_start", _P), ("seg_adapter", _P), ("counts", _P),
                ("grow", _P), ("gather_tiles", _P), ("contig_tiles", _P)]


class lora_slice(ctypes.Structure):
    _fields_ = [("A", _P), ("B", _P), ("d_out", _I32), ("col_off", _I32)]


class LoraError(RuntimeError):
    pass


_lib = None

_SIGS = {
    "lora_version": (ctypes.c_int, []),
    "lora_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "lora_last_error": (ctypes.c_char_p, []),
    "lora_meta_capacity": (ctypes.c_int, [_I32, _I32, _I32, _I32, _I32, ctypes.POINTER(_I32),
                                          ctypes.POINTER(_I32)]),
    "lora_segments_scratch_bytes": (_SZ, [_I32, _I32]),
    "lora_segment_plan": (ctypes.c_int, [_I32, ctypes.POINTER(_I64), _I32, _I32, _I32,
                                         ctypes.POINTER(_I32), ctypes.POINTER(_I32),
                                         ctypes.POINTER(ctypes.c_uint8)]),
    "lora_build_segments": (ctypes.c_int, [_P, ctypes.POINTER(lora_meta), _P, _SZ, _P, _P]),
    "lora_build_segments_static": (ctypes.c_int, [_P, ctypes.POINTER(lora_meta), _P, _P]),
    "lora_shrink_workspace_bytes": (_SZ, [_I32, _I32, _I32]),
    "lora_linear_workspace_bytes": (_SZ, [ctypes.POINTER(lora_meta), _I32, _I32]),
    "lora_sgmv_shrink": (ctypes.c_int, [_P, _P, _I64, _I32, ctypes.POINTER(lora_slice), _I32, _I32,
                                        _P, ctypes.POINTER(lora_meta), ctypes.c_int, _P, _P]),
    "lora_sgmv_expand": (ctypes.c_int, [_P, _I64, _P, ctypes.POINTER(lora_slice), _I32, _I32, _P, _P,
                                        ctypes.POINTER(lora_meta), ctypes.c_int, _P, _P]),
    "lora_bgmv_fused": (ctypes.c_int, [_P, _I64, _P, _I64, _I32, ctypes.POINTER(lora_slice), _I32,
                                       _I32, _P, _P, ctypes.POINTER(lora_meta), _P, _SZ, ctypes.c_int,
                                       _P, _P]),
    "lora_add_linear": (ctypes.c_int, [_P, _I64, _P, _I64, _I32, ctypes.POINTER(lora_slice), _I32,
                                       _I32, _P, _P, ctypes.POINTER(lora_meta), _P, _SZ, ctypes.c_int,
                                       _P, _P]),
    "lora_load_adapter": (ctypes.c_int, [ctypes.POINTER(lora_slice), _I32, _I32, _I32, _I32, _I32,
                                         _I32, ctypes.POINTER(_P), ctypes.POINTER(_P),
                                         ctypes.c_float, _P, _P, ctypes.c_int, _P]),
    "lora_merge_adapter": (ctypes.c_int, [_P, _I64, _I32, _I32, _P, _P, _I32, _I32, _I32, _P, _P,
                                          _I32, ctypes.c_int, _P, _P]),
    "lora_slot_cache_create": (_P, [_I32]),
    "lora_slot_cache_destroy": (None, [_P]),
    "lora_slot_cache_acquire": (ctypes.c_int, [_P, _I64, ctypes.POINTER(_I32), ctypes.POINTER(_I32)]),
    "lora_slot_cache_release": (ctypes.c_int, [_P, _I32]),
    "lora_slot_cache_key": (_I64, [_P, _I32]),
    "lora_slot_cache_evict": (ctypes.c_int, [_P, _I64]),
}


def load():
    """Load the CUDA library; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise LoraError(f"{LIB_PATH} is missing: build it with "
                            "`python -m lora_adapter_application_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def lora_last_error() -> str:
    """The CUDA failure behind the last LORA_ERR_CUDA on this thread ('' if none)."""
    return load().lora_last_error().decode()


def _check(rc):
    if rc != 0:
        msg = load().lora_status_string(rc).decode()
        if rc == ERR_CUDA:
            msg += f" ({load().lora_last_error().decode()})"
        raise LoraError(msg)


def _dev(t: torch.Tensor, what: str):
    if not isinstance(t, torch.Tensor) or t.device.type != "cuda":
        raise LoraError(f"{what} must be a CUDA tensor")
    return t


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _dtype_code(t):
    if t.dtype == torch.bfloat16:
        return LORA_BF16
    if t.dtype == torch.float32:
        return LORA_FP32
    raise LoraError(f"unsupported dtype {t.dtype}: bf16 or fp32")


def _rows(t, what):
    _dev(t, what)
    if t.dim() != 2 or t.stride(1) != 1:
        raise LoraError(f"{what} must be 2-D with unit column stride")
    return t.stride(0)


def lora_version():
    return int(load().lora_version())


def lora_meta_capacity(T, N, rows_per_tile=MAX_TILE_ROWS, min_run=64, long_tile=LONG_TILE):
    mg, mc = _I32(), _I32()
    _check(load().lora_meta_capacity(T, N, rows_per_tile, min_run, long_tile, ctypes.byref(mg),
                                     ctypes.byref(mc)))
    return mg.value, mc.value


def lora_segments_scratch_bytes(T, N):
    return int(load().lora_segments_scratch_bytes(T, N))


def lora_segment_plan(T, layer_cols, rows_per_tile, min_run, sms=0, long_tile=LONG_TILE):
    """(rows_per_tile, min_run, all_gathered) for a batch of T rows that will run
    through lora_add_linear once per layer, layer_cols[l] being layer l's total
    output columns (see include/lora_delta.h); host only."""
    n = len(layer_cols)
    cols = (_I64 * max(n, 1))(*[int(c) for c in layer_cols])
    flags = (ctypes.c_uint8 * max(n, 1))()
    rt, mr = _I32(rows_per_tile), _I32(min_run)
    _check(load().lora_segment_plan(T, cols, n, sms, long_tile, ctypes.byref(rt), ctypes.byref(mr),
                                    flags))
    return rt.value, mr.value, [bool(flags[i]) for i in range(n)]


def lora_build_segments_static(ids, meta: Meta, status, stream=None):
    """lora_build_segments with the library's own fixed scratch array instead of
    meta.scratch, for callers that cannot allocate device memory (see
    include/lora_delta.h: first call per device before any stream capture;
    calls must not overlap on the GPU)."""
    _dev(ids, "ids")
    _dev(status, "status")
    if ids.dtype != torch.int32 or ids.numel() != meta.T or not ids.is_contiguous():
        raise LoraError("ids must be a contiguous int32 tensor of T entries")
    _check(load().lora_build_segments_static(_ptr(ids), ctypes.byref(meta.c), _ptr(status),
                                             _stream(stream)))


def lora_shrink_workspace_bytes(T, r_max, n_slices):
    return int(load().lora_shrink_workspace_bytes(T, r_max, n_slices))


def lora_linear_workspace_bytes(meta, n_slices, r_max):
    return int(load().lora_linear_workspace_bytes(ctypes.byref(meta.c), n_slices, r_max))


class Meta:
    """Device buffers of a batch's lora_meta, allocated with torch, plus the
    builder's scratch and the fused calls' workspace.  ``rows_per_tile`` caps a
    gathered tile; ``min_run`` (0 = off) is the shortest run of one id that
    becomes contiguous tiles."""

    def __init__(self, T, N, rows_per_tile=MAX_TILE_ROWS, min_run=64, long_tile=LONG_TILE,
                 device="cuda"):
        mg, mc = lora_meta_capacity(T, N, rows_per_tile, min_run, long_tile)
        i32 = dict(dtype=torch.int32, device=device)
        self.T, self.N = T, N
        self.perm = torch.zeros(max(T, 1), **i32)
        self.seg_start = torch.zeros(N + 1, **i32)
        self.seg_adapter = torch.zeros(N, **i32)
        self.counts = torch.zeros(4, **i32)
        self.grow = torch.zeros(max(T, 1), **i32)
        self.gather_tiles = torch.zeros(max(mg, 1), 4, **i32)
        self.contig_tiles = torch.zeros(max(mc, 1), 4, **i32)
        nbytes = lora_segments_scratch_bytes(T, N)
        self.scratch = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=device)
        self.scratch_bytes = nbytes
        self.c = lora_meta(T, N, rows_per_tile, min_run, long_tile, mg, mc,
                           self.perm.data_ptr(), self.seg_start.data_ptr(),
                           self.seg_adapter.data_ptr(), self.counts.data_ptr(),
                           self.grow.data_ptr(), self.gather_tiles.data_ptr(),
                           self.contig_tiles.data_ptr())
        self.device = device
        self._ws = None

    def workspace(self, n_slices, r_max):
        """The fused calls' workspace for a layer of n_slices slices and rank slots
        r_max: one zero-filled buffer per Meta, grown when a layer needs more (the
        library keeps its head at zero from call to call).  Calls that use one
        Meta's workspace must not overlap on the GPU."""
        need = lora_linear_workspace_bytes(self, n_slices, r_max)
        if self._ws is None or self._ws.numel() < need:
            self._ws = torch.zeros(max(need, 256), dtype=torch.uint8, device=self.device)
        return self._ws

    def host(self):
        """Copy the metadata to the host (synchronises)."""
        counts = self.counts.cpu().tolist()
        n_seg, n_gather, n_contig, n_short = counts
        return {
            "perm": self.perm[:self.T].cpu().numpy(),
            "seg_start": self.seg_start.cpu().numpy(),
            "seg_adapter": self.seg_adapter[:n_seg].cpu().numpy(),
            "n_seg": n_seg, "n_gather": n_gather, "n_contig": n_contig, "n_short": n_short,
            "grow": self.grow[:n_short].cpu().numpy(),
            "gather_tiles": self.gather_tiles[:n_gather].cpu().numpy(),
            "contig_tiles": self.contig_tiles[:n_contig].cpu().numpy(),
        }


def lora_build_segments(ids, meta: Meta, status, stream=None):
    _dev(ids, "ids")
    _dev(status, "status")
    if ids.dtype != torch.int32 or ids.numel() != meta.T or not ids.is_contiguous():
        raise LoraError("ids must be a contiguous int32 tensor of T entries")
    _check(load().lora_build_segments(_ptr(ids), ctypes.byref(meta.c), _ptr(meta.scratch),
                                      meta.scratch_bytes, _ptr(status), _stream(stream)))


def _slices(A, B, d_out, col_off):
    n = len(A) if A is not None else len(B)
    if not 1 <= n <= MAX_SLICES:
        raise LoraError("1 to 8 slices")
    arr = (lora_slice * n)()
    for s in range(n):
        arr[s].A = A[s].data_ptr() if A is not None else None
        arr[s].B = B[s].data_ptr() if B is not None else None
        arr[s].d_out = int(d_out[s]) if d_out is not None else 0
        arr[s].col_off = int(col_off[s]) if col_off is not None else 0
    return arr, n


def _shapes(meta, x=None, y=None, A=None, B=None, col_off=None, ranks=None, alphas=None,
            v=None):
    """Shape, dtype and layout agreement of a call's operands (the library sees
    only pointers, so a mismatch here would be an out-of-bounds read there).
    Runs before any device check.  Returns (N slots, r_max, n_slices)."""
    T = meta.T
    stacks = [t for t in (A or []) + (B or [])]
    if not stacks:
        raise LoraError("at least one adapter slice")
    if A is not None and B is not None and len(A) != len(B):
        raise LoraError("one A and one B per slice")
    n = len(A) if A is not None else len(B)
    if not 1 <= n <= MAX_SLICES:
        raise LoraError("1 to 8 slices")
    ref = stacks[0]
    for t in stacks:
        if not isinstance(t, torch.Tensor) or t.dim() != 3 or not t.is_contiguous() or \
                t.dtype != ref.dtype:
            raise LoraError("stacked adapters must be contiguous 3-D tensors of one dtype")
    N = ref.shape[0]
    r_max = A[0].shape[1] if A is not None else B[0].shape[2]
    if N < meta.N:
        raise LoraError(f"adapter stacks hold {N} slots, the batch metadata {meta.N}")
    if A is not None:
        d_in = A[0].shape[2]
        if any(a.shape != (N, r_max, d_in) for a in A):
            raise LoraError("every A slice is [N, r_max, d_in] with the same N, r_max, d_in")
        if x is not None:
            if not isinstance(x, torch.Tensor) or x.dim() != 2 or x.shape[0] < T or x.shape[1] < d_in:
                raise LoraError("x must be 2-D with at least T rows and d_in columns")
            if x.dtype != ref.dtype:
                raise LoraError("x, y, A and B share one dtype")
    if B is not None:
        if any(b.shape[0] != N or b.shape[2] != r_max for b in B):
            raise LoraError("every B slice is [N, d_out, r_max] with the same N and r_max")
        if col_off is None or len(col_off) != n:
            raise LoraError("one column offset per slice")
        if y is not None:
            if not isinstance(y, torch.Tensor) or y.dim() != 2 or y.shape[0] < T:
                raise LoraError("y must be 2-D with at least T rows")
            if y.dtype != ref.dtype:
                raise LoraError("x, y, A and B share one dtype")
            for b, c in zip(B, col_off):
                if int(c) < 0 or int(c) + b.shape[1] > y.shape[1]:
                    raise LoraError("a slice's columns run past y")
    for t, what, dt in ((ranks, "ranks", torch.int32), (alphas, "alphas", torch.float32)):
        if t is not None and (not isinstance(t, torch.Tensor) or t.dtype != dt or
                              not t.is_contiguous() or t.numel() < meta.N):
            raise LoraError(f"{what} must be a contiguous {dt} tensor of at least N entries")
    if v is not None and (not isinstance(v, torch.Tensor) or v.dtype != torch.float32 or
                          not v.is_contiguous() or v.numel() < n * T * r_max):
        raise LoraError("v must be contiguous fp32 [n_slices, T, r_max]")
    return N, r_max, n


def _adapters(A, B):
    for t in (A or []) + (B or []):
        _dev(t, "adapter tensor")


def alphas_full(alpha, N, device="cuda"):
    """One alpha for all N adapter slots, as the fp32 [N] tensor the calls take."""
    return torch.full((N,), float(alpha), dtype=torch.float32, device=device)


def lora_sgmv_shrink(v, x, A, ranks, meta: Meta, status, stream=None):
    """v[s, i, k] = sum_j A[s][n, k, j] x[i, j] for rows with an adapter, k < r_n."""
    N, r_max, n = _shapes(meta, x=x, A=A, ranks=ranks, v=v)
    ld_x = _rows(x, "x")
    _adapters(A, None)
    sl, n = _slices(A, None, None, None)
    _dev(v, "v")
    _check(load().lora_sgmv_shrink(_ptr(v), _ptr(x), ld_x, A[0].shape[2], sl, n, r_max,
                                   _ptr(_dev(ranks, "ranks")), ctypes.byref(meta.c), _dtype_code(x),
                                   _ptr(status), _stream(stream)))


def lora_sgmv_expand(y, v, B, col_off, ranks, alphas, meta: Meta, status, stream=None):
    """y[i, col_off_s + c] += (alphas[n] / r_n) sum_k B[s][n, c, k] v[s, i, k]."""
    N, r_max, n = _shapes(meta, y=y, B=B, col_off=col_off, ranks=ranks, alphas=alphas, v=v)
    ld_y = _rows(y, "y")
    _adapters(None, B)
    sl, n = _slices(None, B, [b.shape[1] for b in B], col_off)
    _dev(v, "v")
    _check(load().lora_sgmv_expand(_ptr(y), ld_y, _ptr(v), sl, n, r_max, _ptr(_dev(ranks, "ranks")),
                                   _ptr(_dev(alphas, "alphas")), ctypes.byref(meta.c),
                                   _dtype_code(y), _ptr(status), _stream(stream)))


def _fused(fn, y, x, A, B, col_off, ranks, alphas, meta, status, stream, workspace):
    N, r_max, n = _shapes(meta, x=x, y=y, A=A, B=B, col_off=col_off, ranks=ranks, alphas=alphas)
    ld_y = _rows(y, "y")
    ld_x = _rows(x, "x")
    _adapters(A, B)
    sl, n = _slices(A, B, [b.shape[1] for b in B], col_off)
    ws = meta.workspace(n, r_max) if workspace is None else _dev(workspace, "workspace")
    _check(fn(_ptr(y), ld_y, _ptr(x), ld_x, A[0].shape[2], sl, n, r_max, _ptr(_dev(ranks, "ranks")),
              _ptr(_dev(alphas, "alphas")), ctypes.byref(meta.c), _ptr(ws),
              ws.numel() * ws.element_size(), _dtype_code(x), _ptr(status), _stream(stream)))


def lora_bgmv_fused(y, x, A, B, col_off, ranks, alphas, meta: Meta, status, stream=None,
                    workspace=None):
    """Fused shrink + expand of every tile in one launch."""
    _fused(load().lora_bgmv_fused, y, x, A, B, col_off, ranks, alphas, meta, status, stream,
           workspace)


def lora_add_linear(y, x, A, B, col_off, ranks, alphas, meta: Meta, status, stream=None,
                    workspace=None):
    """All slices of one linear layer applied to y in place (add_lora_linear).
    ``workspace`` (optional): a zero-filled uint8 CUDA tensor of at least
    lora_linear_workspace_bytes bytes; by default the Meta's own."""
    _fused(load().lora_add_linear, y, x, A, B, col_off, ranks, alphas, meta, status, stream,
           workspace)


# ---------------------------------------------------------------- adapter slots
def lora_load_adapter(A, B, n, src_A, src_B, alpha, ranks, alphas, stream=None):
    """Copy one adapter (src_A[s] [r, d_in], src_B[s] [d_out_s, r], device or pinned
    host tensors) into slot n of the stacks A[s] [N, r_max, d_in], B[s] [N, d_out_s,
    r_max], zeroing the rank padding, and set ranks[n] = r, alphas[n] = alpha."""
    if len(A) != len(B) or len(src_A) != len(A) or len(src_B) != len(B):
        raise LoraError("one source A and B per slice")
    N, r_max, d_in = A[0].shape
    r = src_A[0].shape[0]
    for a, b, sa, sb in zip(A, B, src_A, src_B):
        _dev(a, "A")
        _dev(b, "B")
        if a.shape != (N, r_max, d_in) or b.shape[0] != N or b.shape[2] != r_max:
            raise LoraError("stacks of one N, r_max, d_in")
        if sa.shape != (r, d_in) or sb.shape != (b.shape[1], r):
            raise LoraError("sources are [r, d_in] and [d_out_s, r]")
        if not (sa.is_contiguous() and sb.is_contiguous()) or sa.dtype != a.dtype or sb.dtype != a.dtype:
            raise LoraError("contiguous sources of the stacks' dtype")
        if sa.device.type == "cpu" and not (sa.is_pinned() and sb.is_pinned()):
            raise LoraError("host sources must be pinned")
    sl, S = _slices(A, B, [b.shape[1] for b in B], [0] * len(B))
    pa = (_P * S)(*[t.data_ptr() for t in src_A])
    pb = (_P * S)(*[t.data_ptr() for t in src_B])
    _check(load().lora_load_adapter(sl, S, d_in, r_max, N, int(n), int(r), pa, pb, float(alpha),
                                    _ptr(_dev(ranks, "ranks")), _ptr(_dev(alphas, "alphas")),
                                    _dtype_code(A[0]), _stream(stream)))


def lora_slot_cache_create(n_slots):
    return load().lora_slot_cache_create(int(n_slots))


def lora_slot_cache_destroy(cache):
    load().lora_slot_cache_destroy(cache)


def lora_slot_cache_acquire(cache, key):
    slot, resident = _I32(), _I32()
    _check(load().lora_slot_cache_acquire(cache, int(key), ctypes.byref(slot), ctypes.byref(resident)))
    return slot.value, bool(resident.value)


def lora_slot_cache_release(cache, slot):
    _check(load().lora_slot_cache_release(cache, int(slot)))


def lora_slot_cache_key(cache, slot):
    return int(load().lora_slot_cache_key(cache, int(slot)))


def lora_slot_cache_evict(cache, key):
    _check(load().lora_slot_cache_evict(cache, int(key)))


class SlotCache:
    """The library's LRU slot policy (lora_slot_cache_*), owned by this object."""

    def __init__(self, n_slots):
        self.h = lora_slot_cache_create(n_slots)
        if not self.h:
            raise LoraError("n_slots must be in [1, 4096]")
        self.n_slots = n_slots

    def acquire(self, key):
        return lora_slot_cache_acquire(self.h, key)

    def release(self, slot):
        lora_slot_cache_release(self.h, slot)

    def key(self, slot):
        return lora_slot_cache_key(self.h, slot)

    def evict(self, key):
        lora_slot_cache_evict(self.h, key)

    def __del__(self):
        if getattr(self, "h", None) and _lib is not None:
            lora_slot_cache_destroy(self.h)
            self.h = None


# ---------------------------------------------------------------- merge / unmerge
def lora_merge_adapter(W, A, B, n, ranks, alphas, status, sign=1, stream=None):
    """W += sign * (alphas[n] / r_n) * B[n] @ A[n] in place (one slice's stacks
    A [N, r_max, d_in], B [N, d_out, r_max]; W [d_out, >= d_in])."""
    ld_w = _rows(W, "W")
    _dev(A, "A")
    _dev(B, "B")
    N, r_max, d_in = A.shape
    if B.dim() != 3 or B.shape[0] != N or B.shape[2] != r_max or not (A.is_contiguous() and B.is_contiguous()):
        raise LoraError("A [N, r_max, d_in] and B [N, d_out, r_max], contiguous")
    d_out = B.shape[1]
    if W.shape[0] < d_out or W.shape[1] < d_in or W.dtype != A.dtype or B.dtype != A.dtype:
        raise LoraError("W is [d_out, >= d_in] of the adapters' dtype")
    for t, what, dt in ((ranks, "ranks", torch.int32), (alphas, "alphas", torch.float32)):
        if t.dtype != dt or t.numel() < N:
            raise LoraError(f"{what} must be {dt} with N entries")
    _check(load().lora_merge_adapter(_ptr(W), ld_w, d_out, d_in, _ptr(A), _ptr(B), N, r_max, int(n),
                                     _ptr(_dev(ranks, "ranks")), _ptr(_dev(alphas, "alphas")),
                                     int(sign), _dtype_code(W), _ptr(_dev(status, "status")),
                                     _stream(stream)))
