"""Algorithmic traffic and work of one delta application, the denominators of
the roofline the benchmark reports.

Bytes of one layer call (every byte the method must move once):
    sum over rows with an adapter of  e*d_in (x)  +  2*e*sum_s d_out_s (y read and written)
  + sum over distinct adapters used of  sum_s e*r_n*(d_in + d_out_s)  (the live part of A and B)
Rows without an adapter cost nothing; padding beyond r_n is not algorithmic.
Multiply-adds: per row with an adapter r_n*(S*d_in + sum_s d_out_s), flops = 2x that.
"""
from __future__ import annotations

import numpy as np


def layer_bytes(ids, ranks, N, d_in, d_outs, elem_bytes):
    ids = np.asarray(ids)
    ranks = np.asarray(ranks)
    active = (ids >= 0) & (ids < N)
    n_active = int(active.sum())
    rows = n_active * (elem_bytes * d_in + 2 * elem_bytes * int(sum(d_outs)))
    touched = np.unique(ids[active])
    adapters = 0
    for n in touched:
        r = int(ranks[n])
        adapters += sum(elem_bytes * r * (d_in + d) for d in d_outs)
    return rows + adapters


def layer_flops(ids, ranks, N, d_in, d_outs):
    ids = np.asarray(ids)
    ranks = np.asarray(ranks)
    active = (ids >= 0) & (ids < N)
    r = ranks[ids[active]].astype(np.int64)
    return int(2 * (r * (len(d_outs) * d_in + int(sum(d_outs)))).sum())


def workload_bytes(w, elem_bytes=None):
    e = elem_bytes or (2 if str(w.dtype).endswith("bfloat16") else 4)
    return sum(layer_bytes(w.ids.numpy(), w.ranks.numpy(), w.N, l.d_in, l.d_out, e) for l in w.layers)


def workload_flops(w):
    return sum(layer_flops(w.ids.numpy(), w.ranks.numpy(), w.N, l.d_in, l.d_out) for l in w.layers)
