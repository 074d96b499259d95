"""Seeded synthetic inputs for multi-LoRA delta application.

This module only draws inputs: ids, request lengths, ranks and the float
tensors.  It holds none of the method's arithmetic, so both the fp64 oracle
and the CUDA library can be fed from it without sharing any computation.

Every workload is drawn from one ``torch.Generator`` on the CPU, seeded, and
consumed in a fixed order: structure first (ids, lengths, ranks), then per
layer x, A, B, y0.  The same bits then go to the oracle and, copied, to the
device.

The five named workloads follow the shapes the pages talk about: a Llama-3-8B
q_proj (4096x4096) with rank 16 (page "Multi-LoRA Serving", section 3.1
example; page "LoRA hot load and adapter routing", weight-structure paragraph),
the full attention+MLP projection set (same page, q/k/v/o and gate/up/down),
and a 70B-shaped MLP with hidden 8192 (page "LoRA service", section 7 example).
Distribution choices the pages leave open:

* x ~ N(0, 1); A and B ~ N(0, std = 1/sqrt(d_in)) of the layer;
* y0 ~ N(0, 1), a stand-in for the shared base output W x;
* rank rows/columns beyond an adapter's own rank r_n are zero padding up to
  r_max (the max-lora-rank slot size of page "Multi-LoRA Serving", 3.2);
* Zipf(s) over N adapters means p(id = k-1) proportional to k^-s, k = 1..N.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch

__all__ = ["Layer", "Workload", "make", "NAMES", "tiny", "decode_qproj", "prefill",
           "multislice_8b", "mixed_70b", "random_case"]


@dataclass
class Layer:
    name: str
    d_in: int
    d_out: list          # per slice
    col_off: list        # per slice, column offset in y
    x: torch.Tensor      # [T, d_in]
    A: list              # per slice [N, r_max, d_in]
    B: list              # per slice [N, d_out_s, r_max]
    y0: torch.Tensor     # [T, sum(d_out)]


@dataclass
class Workload:
    name: str
    dtype: torch.dtype
    T: int
    N: int
    r_max: int
    alpha: float
    ids: torch.Tensor    # [T] int32, -1 = base model only
    ranks: torch.Tensor  # [N] int32
    layers: list
    info: dict = field(default_factory=dict)

    def to(self, device):
        """A copy with every tensor moved to ``device`` (same bits)."""
        layers = [Layer(l.name, l.d_in, list(l.d_out), list(l.col_off), l.x.to(device),
                        [a.to(device) for a in l.A], [b.to(device) for b in l.B],
                        l.y0.to(device)) for l in self.layers]
        return Workload(self.name, self.dtype, self.T, self.N, self.r_max, self.alpha,
                        self.ids.to(device), self.ranks.to(device), layers, dict(self.info))


def _normal(g, shape, std, dtype):
    t = torch.randn(shape, generator=g, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(dtype)


def _zipf_ids(g, T, N, s):
    k = torch.arange(1, N + 1, dtype=torch.float64)
    p = k.pow(-s)
    p = p / p.sum()
    return torch.multinomial(p, T, replacement=True, generator=g).to(torch.int32)


def _layer(g, name, T, N, r_max, ranks, d_in, d_out, dtype):
    std = 1.0 / (d_in ** 0.5)
    x = _normal(g, (T, d_in), 1.0, dtype)
    A, B = [], []
    live_rows = (torch.arange(r_max)[None, :] < ranks[:, None].long())   # [N, r_max]
    for d in d_out:
        a = _normal(g, (N, r_max, d_in), std, dtype)
        b = _normal(g, (N, d, r_max), std, dtype)
        a.mul_(live_rows[:, :, None].to(dtype))
        b.mul_(live_rows[:, None, :].to(dtype))
        A.append(a)
        B.append(b)
    col_off, off = [], 0
    for d in d_out:
        col_off.append(off)
        off += d
    y0 = _normal(g, (T, off), 1.0, dtype)
    return Layer(name, d_in, list(d_out), col_off, x, A, B, y0)


def tiny(seed=0, dtype=torch.float32):
    """64 rows, 256 -> 256, rank 8, 4 adapters, ids uniform over {-1,0,1,2,3}, alpha 16."""
    g = torch.Generator().manual_seed(seed)
    T, N, r = 64, 4, 8
    ids = (torch.randint(0, N + 1, (T,), generator=g) - 1).to(torch.int32)
    ranks = torch.full((N,), r, dtype=torch.int32)
    lay = _layer(g, "proj", T, N, r, ranks, 256, [256], dtype)
    return Workload("tiny", dtype, T, N, r, 16.0, ids, ranks, [lay],
                    {"desc": "T=64 d_in=d_out=256 r=8 N=4 fp32 ids U{-1..3} alpha=16"})


def decode_qproj(seed=0, T=256, N=32, d=4096, r=16, none_frac=0.10, zipf=1.1,
                 dtype=torch.bfloat16):
    """Decode batch on a Llama-3-8B q_proj: one token per row, Zipf ids, 10% none."""
    g = torch.Generator().manual_seed(seed)
    none = torch.rand(T, generator=g) < none_frac
    ids = _zipf_ids(g, T, N, zipf)
    ids[none] = -1
    ranks = torch.full((N,), r, dtype=torch.int32)
    lay = _layer(g, "q_proj", T, N, r, ranks, d, [d], dtype)
    return Workload("decode_qproj", dtype, T, N, r, 32.0, ids, ranks, [lay],
                    {"desc": f"decode BGMV q_proj: T={T} rows d={d} r={r} N={N} "
                             f"Zipf({zipf}) ids, {int(none_frac*100)}% none, alpha=32"})


def prefill(seed=0, n_req=64, len_lo=128, len_hi=2048, d=4096, r=16, n_adapters=8,
            dtype=torch.bfloat16):
    """Prefill batch: contiguous prompts, 8 adapters round-robin plus one base-only request."""
    g = torch.Generator().manual_seed(seed)
    lengths = torch.randint(len_lo, len_hi + 1, (n_req,), generator=g)
    base_req = int(torch.randint(0, n_req, (1,), generator=g))
    order = torch.randperm(n_req - 1, generator=g)
    req_ids = torch.empty(n_req, dtype=torch.int32)
    others = [i for i in range(n_req) if i != base_req]
    for m, pos in enumerate(order.tolist()):
        req_ids[others[pos]] = m % n_adapters
    req_ids[base_req] = -1
    ids = torch.repeat_interleave(req_ids, lengths).to(torch.int32)
    T = int(lengths.sum())
    ranks = torch.full((n_adapters,), r, dtype=torch.int32)
    lay = _layer(g, "q_proj", T, n_adapters, r, ranks, d, [d], dtype)
    return Workload("prefill", dtype, T, n_adapters, r, 32.0, ids, ranks, [lay],
                    {"desc": f"prefill SGMV: {n_req} requests, lengths U[{len_lo},{len_hi}], "
                             f"T={T}, d={d}, r={r}, {n_adapters} adapters + 1 base request",
                     "lengths": lengths.tolist(), "req_ids": req_ids.tolist()})


def multislice_8b(seed=0, T=1024, N=100, ranks_from=(8, 16, 32, 64), r_max=64, zipf=1.1,
                  hidden=4096, kv=1024, inter=14336, dtype=torch.bfloat16):
    """Llama-3-8B layer set at decode: qkv (3 slices), o, gate/up (2 slices), down."""
    g = torch.Generator().manual_seed(seed)
    ids = _zipf_ids(g, T, N, zipf)
    choice = torch.randint(0, len(ranks_from), (N,), generator=g)
    ranks = torch.tensor(ranks_from, dtype=torch.int32)[choice]
    layers = [
        _layer(g, "qkv_proj", T, N, r_max, ranks, hidden, [hidden, kv, kv], dtype),
        _layer(g, "o_proj", T, N, r_max, ranks, hidden, [hidden], dtype),
        _layer(g, "gate_up_proj", T, N, r_max, ranks, hidden, [inter, inter], dtype),
        _layer(g, "down_proj", T, N, r_max, ranks, inter, [hidden], dtype),
    ]
    return Workload("multislice_8b", dtype, T, N, r_max, 32.0, ids, ranks, layers,
                    {"desc": f"Llama-3-8B layer set at decode: T={T} rows, {N} adapters, ranks "
                             f"from {list(ranks_from)} padded to {r_max}, Zipf({zipf}) ids, alpha=32"})


def mixed_70b(seed=0, T=8192, n_req=32, len_lo=64, len_hi=512, hidden=8192, inter=28672,
              r=16, N=16, none_frac=0.15, reserve=256, dtype=torch.bfloat16):
    """70B-shaped MLP batch: 32 prefill prompts plus decode rows filling T tokens."""
    g = torch.Generator().manual_seed(seed)
    draws = 0
    while True:
        draws += 1
        lengths = torch.randint(len_lo, len_hi + 1, (n_req,), generator=g)
        if int(lengths.sum()) <= T - reserve:
            break
    n_decode = T - int(lengths.sum())
    units = n_req + n_decode
    none = torch.rand(units, generator=g) < none_frac
    unit_ids = torch.randint(0, N, (units,), generator=g).to(torch.int32)
    unit_ids[none] = -1
    ids = torch.cat([torch.repeat_interleave(unit_ids[:n_req], lengths),
                     unit_ids[n_req:]]).to(torch.int32)
    ranks = torch.full((N,), r, dtype=torch.int32)
    layers = [
        _layer(g, "up_proj", T, N, r, ranks, hidden, [inter], dtype),
        _layer(g, "down_proj", T, N, r, ranks, inter, [hidden], dtype),
    ]
    return Workload("mixed_70b", dtype, T, N, r, 32.0, ids, ranks, layers,
                    {"desc": f"mixed 70B-shaped batch: {n_req} prompts U[{len_lo},{len_hi}] "
                             f"({int(lengths.sum())} tokens) + {n_decode} decode rows, "
                             f"{hidden}->{inter}->{hidden}, r={r}, {N} adapters, "
                             f"{int(none_frac*100)}% none",
                     "length_draws": draws, "prefill_tokens": int(lengths.sum()),
                     "decode_rows": n_decode, "lengths": lengths.tolist()})


def random_case(seed, T, N, d_in, d_out, r_max, ranks=None, none_frac=0.2, runs=None,
                dtype=torch.bfloat16, alpha=16.0):
    """Small random case for tests.  ``runs``: list of (length, id) blocks laid out in
    order, filling the rest with single rows of random ids."""
    g = torch.Generator().manual_seed(seed)
    if ranks is None:
        ranks = torch.randint(1, r_max + 1, (N,), generator=g).to(torch.int32)
    else:
        ranks = torch.as_tensor(ranks, dtype=torch.int32)
    if runs:
        parts = [torch.full((L,), i, dtype=torch.int32) for (L, i) in runs]
        used = sum(L for (L, _) in runs)
        rest = torch.randint(0, N, (max(T - used, 0),), generator=g).to(torch.int32)
        ids = torch.cat(parts + [rest])[:T]
    else:
        ids = torch.randint(0, N, (T,), generator=g).to(torch.int32)
        none = torch.rand(T, generator=g) < none_frac
        ids[none] = -1
    d_out = list(d_out) if isinstance(d_out, (list, tuple)) else [d_out]
    lay = _layer(g, "proj", T, N, r_max, ranks, d_in, d_out, dtype)
    return Workload("random", dtype, T, N, r_max, alpha, ids, ranks, [lay],
                    {"desc": f"random T={T} N={N} d_in={d_in} d_out={d_out} r_max={r_max}"})


NAMES = {
    "tiny": tiny,
    "decode_qproj": decode_qproj,
    "prefill": prefill,
    "multislice_8b": multislice_8b,
    "mixed_70b": mixed_70b,
}


def make(name, seed=0, **kw):
    return NAMES[name](seed=seed, **kw)
