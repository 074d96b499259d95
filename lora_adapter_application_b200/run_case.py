"""Run the grouping and lora_add_linear a few times on one synthetic workload
layer, for profilers (ncu, nsys) or a quick check on a new device.

    python -m lora_adapter_application_b200.run_case prefill --reps 3 --requests 16
    python -m lora_adapter_application_b200.run_case decode_qproj --min-run 0

Prints the tile counts and the device status word; exits non-zero on a
non-zero status.
"""
from __future__ import annotations

import argparse
import os
import sys

import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import lora_adapter_application_b200 as lora  # noqa: E402
import workloads  # noqa: E402


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("workload", choices=sorted(workloads.NAMES))
    ap.add_argument("--layer", type=int, default=0)
    ap.add_argument("--reps", type=int, default=3)
    ap.add_argument("--min-run", type=int, default=64, help="shortest run that becomes contiguous tiles (0 = none)")
    ap.add_argument("--rows-per-tile", type=int, default=lora.MAX_TILE_ROWS,
                    help="rows per gathered tile (1 .. 64)")
    ap.add_argument("--requests", type=int, default=0, help="prefill / mixed_70b: number of prompts (0 = default)")
    ap.add_argument("--seed", type=int, default=0)
    args = ap.parse_args(argv)

    kw = {"n_req": args.requests} if args.requests and args.workload in ("prefill", "mixed_70b") else {}
    w = workloads.make(args.workload, seed=args.seed, **kw)
    lay = w.layers[args.layer]
    dev = torch.device("cuda")
    x, y = lay.x.to(dev), lay.y0.to(dev)
    A, B = [a.to(dev) for a in lay.A], [b.to(dev) for b in lay.B]
    ids, ranks = w.ids.to(dev), w.ranks.to(dev)
    alphas = lora.alphas_full(w.alpha, w.N, dev)
    meta = lora.Meta(w.T, w.N, args.rows_per_tile, args.min_run, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    lora.lora_build_segments(ids, meta, status)
    for _ in range(args.reps):
        lora.lora_add_linear(y, x, A, B, lay.col_off, ranks, alphas, meta, status)
    torch.cuda.synchronize()
    code = int(status.item())
    print(f"{w.name}/{lay.name}: T={w.T} counts={meta.counts.cpu().tolist()} status={code}")
    return 0 if code == 0 else 1


if __name__ == "__main__":
    sys.exit(main())
