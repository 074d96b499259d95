"""Shared helpers of the GPU parity tests: run the library through its binding
on a workload and compare with the fp64 oracle."""
import numpy as np
import torch

import lora_adapter_application_b200 as lora
import oracle

# tolerance stated for the method: bf16 in / fp32 accumulate, and fp32 mode
TOL = {torch.bfloat16: 1e-2, torch.float32: 1e-4}


def assert_within(gpu, ref, dtype, what=""):
    gpu = np.asarray(gpu, dtype=np.float64)
    tol = TOL[dtype] * np.maximum(1.0, np.abs(ref))
    err = np.abs(gpu - ref)
    bad = err > tol
    if bad.any():
        idx = np.argwhere(bad)[:5].tolist()
        raise AssertionError(f"{what}: {int(bad.sum())} of {bad.size} elements beyond tolerance, "
                             f"max err {err.max():.3e}, first at {idx}")


class DeviceLayer:
    def __init__(self, layer, device="cuda"):
        self.x = layer.x.to(device)
        self.A = [a.to(device) for a in layer.A]
        self.B = [b.to(device) for b in layer.B]
        self.y0 = layer.y0.to(device)
        self.col_off = list(layer.col_off)
        self.d_out = list(layer.d_out)


def build_meta(ids_cpu, N, rows_per_tile=16, min_run=64, device="cuda"):
    T = ids_cpu.shape[0]
    meta = lora.Meta(T, N, rows_per_tile, min_run, device=device)
    status = torch.zeros(1, dtype=torch.int32, device=device)
    lora.lora_build_segments(ids_cpu.to(device), meta, status)
    return meta, status


def run_fused(w, dl, meta, status, fn=None):
    fn = fn or lora.lora_add_linear
    ranks = w.ranks.cuda()
    alphas = lora.alphas_full(w.alpha, w.N)
    y = dl.y0.clone()
    fn(y, dl.x, dl.A, dl.B, dl.col_off, ranks, alphas, meta, status)
    torch.cuda.synchronize()
    return y


def oracle_rows(w, layer, rows):
    return oracle.lora_apply(layer.x, layer.A, layer.B, layer.col_off, w.ranks, w.alpha, w.ids,
                             layer.y0, rows=rows)


def sample_rows(w, k, seed=0):
    """k rows spread over the batch, plus the first and last row and rows of each id."""
    g = np.random.default_rng(seed)
    T = w.T
    rows = set(g.choice(T, size=min(k, T), replace=False).tolist())
    rows.update([0, T - 1])
    ids = w.ids.numpy()
    for n in np.unique(ids)[:64]:
        where = np.nonzero(ids == n)[0]
        rows.update([int(where[0]), int(where[-1])])
    return np.array(sorted(rows), dtype=np.int32)


def kernels_of(fn, tries=5):
    """Runs fn under the torch profiler (CUPTI) and returns (fn's result, names of
    the device kernels it launched, in order, and the number of kernel-launch API
    calls).  CUPTI hands kernel records over asynchronously, and after earlier
    sessions in the same process it has been seen to deliver fewer records than
    there were launches; such a session is run again, so fn must be safe to
    repeat."""
    from torch.autograd import DeviceType
    from torch.profiler import ProfilerActivity, profile
    for _ in range(tries):
        torch.cuda.synchronize()
        with profile(activities=[ProfilerActivity.CUDA]) as prof:
            out = fn()
            torch.cuda.synchronize()
        ev = prof.events()
        kernels = [e.name for e in ev if e.device_type == DeviceType.CUDA
                   and not e.name.startswith(("Memcpy", "Memset"))]
        launches = sum(1 for e in ev if e.device_type == DeviceType.CPU and "LaunchKernel" in e.name)
        if len(kernels) == launches:
            return out, kernels, launches
    raise AssertionError(f"kernel records never matched the {launches} launches in {tries} "
                         f"profiler sessions (last: {kernels})")
