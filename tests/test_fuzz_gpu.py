"""Seeded random layers against the fp64 oracle: shapes, ranks, tile sizes, prompt
runs and rows without an adapter drawn at random, through the fused entry points
with the launch choices a caller can make (split or unsplit shrink items, the
tensor-core or mma.sync gathered-tile kernel, grid sizes).  Each case is small
enough for the oracle to finish in well under a second.

Tolerance (the method's): bf16 |gpu - oracle| <= 1e-2 * max(1, |oracle|); rows
without an adapter bit-identical.
"""
import random

import pytest
import torch

import lora_adapter_application_b200 as lora
import workloads
from gpu_helpers import DeviceLayer, assert_within, build_meta, oracle_rows

pytestmark = pytest.mark.gpu


def _case(seed):
    g = random.Random(seed)
    T = g.randint(1, 600)
    N = g.randint(1, 40)
    d_in = 8 * g.randint(1, 160)
    S = g.choice([1, 1, 2, 3])
    d_out = [8 * g.randint(1, 96) for _ in range(S)]
    r_max = 8 * g.randint(1, 8)
    ranks = [g.randint(1, r_max) for _ in range(N)]
    rows_per_tile = g.choice([1, 5, 8, 16, 16, 33, 64])
    min_run = g.choice([0, 0, 8, 64])
    runs = None
    if min_run and T >= 2 * min_run:   # a few prompt-like runs, the rest single rows
        runs, left = [], T
        for _ in range(g.randint(1, 4)):
            L = g.randint(min_run, max(min_run, min(left // 2, 300)))
            if L > left:
                break
            runs.append((L, g.randrange(N)))
            left -= L
    env = {}
    ks = g.choice([None, "1", "2"])
    if ks:
        env["LORA_BG_KSPLIT"] = ks
    if rows_per_tile <= 16 and g.random() < 0.35:
        env["LORA_BG_TC"] = "1"
    if g.random() < 0.2:
        env["LORA_BG_BLOCKS"] = str(g.choice([1, 3, 17]))
    fn = g.choice(["add_linear", "bgmv_fused"])
    w = workloads.random_case(900 + seed, T, N, d_in, d_out, r_max, ranks=ranks,
                              none_frac=g.choice([0.0, 0.1, 0.4]), runs=runs)
    return w, rows_per_tile, min_run, env, fn


@pytest.mark.parametrize("seed", list(range(100)))
def test_random_layer_matches_oracle(cuda_lib, seed, monkeypatch):
    w, rows_per_tile, min_run, env, fn = _case(seed)
    for k, v in env.items():
        monkeypatch.setenv(k, v)
    lay = w.layers[0]
    dl = DeviceLayer(lay)
    meta, status = build_meta(w.ids, w.N, rows_per_tile, min_run)
    y = dl.y0.clone()
    f = lora.lora_add_linear if fn == "add_linear" else lora.lora_bgmv_fused
    f(y, dl.x, dl.A, dl.B, dl.col_off, w.ranks.cuda(), lora.alphas_full(w.alpha, w.N), meta, status)
    torch.cuda.synchronize()
    what = (f"seed {seed}: T={w.T} N={w.N} d_in={lay.x.shape[1]} d_out={list(lay.d_out)} r_max={w.r_max} "
            f"tile={rows_per_tile} min_run={min_run} {fn} {env}")
    assert int(status.item()) == 0, f"{what}: device status {int(status.item())}"
    y = y.cpu()
    assert_within(y.double().numpy(), oracle_rows(w, lay, None), w.dtype, what)
    none = w.ids < 0
    assert torch.equal(y[none], lay.y0[none]), f"{what}: rows without an adapter changed"
